/*
 * mfa.h -- C ABI of libmfa.so: exact tiled scaled-dot-product attention on B200 (sm_100a).
 *
 * Operations:
 *   mfa_fwd            dense forward with online softmax: causal and sliding-window tile skip,
 *                      native GQA, optional tanh softcap, optional fp32 log-sum-exp output.
 *   mfa_fwd_varlen     the same forward over packed variable-length sequences (cu_seqlens).
 *   mfa_fwd_blocksparse the same forward restricted by a 128 x 128 block mask.
 *   mfa_fwd_paged      chunked prefill: packed query chunks over a paged KV cache.
 *   mfa_bwd            backward of mfa_fwd (dq, dk, dv from out and lse).
 *   mfa_decode_splitkv two-phase split-KV decode (N_q <= 4) over a paged KV cache
 *                      (mfa_decode_splitkv_window: with a left window).
 *
 * Sources (web pages, cited by title and section):
 *   [MLXBUN]  "mlx-bun 0.4.0 -> 1.0.0, src/model/flash-attention.ts" (diffend): forward shader
 *             (online softmax over K/V tiles, fp32 accumulation, saved m + log(l), kv_head =
 *             head / reps) and flashForward (q [B,Hq,Tq,D], k/v [B,Hkv,Tkv,D], o like q,
 *             log-sum-exp [B,Hq,Tq] fp32).
 *   [MFA252]  "mlx-mfa 2.5.2" (pypi.org): Features (causal tile-skip, window_size=(left,right)
 *             tile-skip, native GQA, tanh softcap, Flash Decode two-phase split-KV for N_q <= 4,
 *             paged KV with block_table), Usage (window (512,-1), softcap=50.0), Supported
 *             Configurations ([B,H,N,D] row-major, float16 / bfloat16).
 *   [MXFA15]  "mxflashattn 1.4.0 -> 1.5.0" (diffend), README: split-KV paged decode reading a
 *             paged KV cache, page_size 16, GQA 4; per-split (m, l) slots merged by a combine
 *             step; explicit errors instead of silent fallbacks.
 *   [MFA261]  "mlx-mfa 2.61.0" (PyPI package metadata): raw entry points carry the same guards
 *             as the wrappers (contiguity, paged capacity, zero-KV, GQA geometry).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers to contiguous row-major buffers owned by the
 *     caller. The library allocates nothing per call, never synchronises, and launches only on
 *     the stream it is given (a cudaStream_t passed as void*; NULL = legacy default stream).
 *   - Every tensor pointer must be 16-byte aligned.
 *   - Malformed arguments are rejected BEFORE any launch with a negative status; nothing is
 *     written then. There is no fallback path: an unsupported case is an error, never a slower
 *     or approximate answer.
 *   - Kernels bound every internal wait; a wait that runs out, or an out-of-range block_table
 *     entry, records a device status that mfa_device_status() returns.
 *   - The TMA tensor maps a launch needs are cached inside the library per device, keyed by
 *     (base pointer, data type, layout, extents), 256 of them with the least recently used one
 *     replaced; repeated calls over the same buffers encode no map (mfa_debug_tmap_stats).
 *   - Windows (win_l, win_r) at least as wide as every sequence of the call mean the same as -1
 *     and are treated as -1, so INT_MAX is a valid "unbounded" value; sequence lengths are below
 *     2^30.
 */
#ifndef MFA_H_
#define MFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types of q, k, v, out (and of the page pools). */
#define MFA_DTYPE_FP16 0
#define MFA_DTYPE_BF16 1

/* Status codes. */
#define MFA_OK                       0
#define MFA_ERR_NULL_POINTER        -1   /* a required pointer is NULL */
#define MFA_ERR_MISALIGNED          -2   /* a tensor pointer is not 16-byte aligned */
#define MFA_ERR_BAD_DTYPE           -3   /* dtype not MFA_DTYPE_FP16 / MFA_DTYPE_BF16 */
#define MFA_ERR_BAD_HEAD_DIM        -4   /* D not in {64, 128} (decode: {64, 128, 256}) */
#define MFA_ERR_BAD_SHAPE           -5   /* negative size, or a size whose element count overflows */
#define MFA_ERR_GQA_GEOMETRY        -6   /* Hkv < 1 or Hq not a multiple of Hkv */
#define MFA_ERR_BAD_WINDOW          -7   /* window bound below -1 */
#define MFA_ERR_BAD_SOFTCAP         -8   /* softcap negative or not finite */
#define MFA_ERR_BAD_SCALE           -9   /* scale not finite or not > 0 */
#define MFA_ERR_NQ_TOO_LARGE       -10   /* decode with N_q > 4 */
#define MFA_ERR_PAGE_SIZE          -11   /* page_size != 16 */
#define MFA_ERR_WORKSPACE          -12   /* workspace NULL, misaligned or smaller than required */
#define MFA_ERR_UNSUPPORTED        -13   /* decode with (Hq / Hkv) * N_q > 16 query rows per kv head, or a
                                            block-sparse call with more than 2048 key tiles */
#define MFA_ERR_CUDA               -20   /* a CUDA runtime/driver call or a launch failed */
#define MFA_ERR_DEVICE_TIMEOUT     -21   /* device status: a bounded wait inside a kernel ran out */
#define MFA_ERR_DEVICE_BAD_PAGE    -22   /* device status: a block_table entry was outside [0, num_pages) */
#define MFA_ERR_SCRATCH_TOO_SMALL  -23   /* mfa_decode_splitkv_noalloc: shape needs more than its fixed scratch */
#define MFA_ERR_DEVICE_BAD_SEQLENS -24   /* device status: a cu_seqlens entry was negative, decreasing or past
                                            the packed total, or a sequence was longer than max_seqlen_q */
#define MFA_ERR_DEVICE_TILE_LIST   -25   /* device status: a key-tile list exceeded its capacity (a host check failed) */

/*
 * mfa_fwd -- exact attention forward (prefill).
 *
 * Computes, for every batch b, query head h, query row i:
 *   g      = h / (Hq / Hkv)                          (contiguous GQA groups [MLXBUN] kv_head = head / reps)
 *   a      = i + (Nk - Nq)                           (bottom-right alignment of the query rows)
 *   vis(j) = (!causal || j <= a) && (win_l < 0 || j >= a - win_l) && (win_r < 0 || j <= a + win_r)
 *   s_j    = scale * <q[b,h,i,:], k[b,g,j,:]>;  if softcap > 0: s_j = softcap * tanh(s_j / softcap)
 *   out[b,h,i,:] = sum_{vis j} exp(s_j - m) v[b,g,j,:] / sum_{vis j} exp(s_j - m),  m = max_{vis j} s_j
 *   lse[b,h,i]   = m + ln(sum_{vis j} exp(s_j - m))
 * without materialising the score matrix ([MLXBUN] forward shader; [MFA252] Features). A row
 * with no visible key gets out = 0 and lse = -inf. Key tiles that no row of a block can see are
 * never loaded (causal and window tile skip, [MFA252] Features).
 *
 * Arguments
 *   q    [B, Hq,  Nq, D]  dtype        k, v [B, Hkv, Nk, D]  dtype       (read only)
 *   out  [B, Hq,  Nq, D]  dtype        lse  [B, Hq, Nq] float32, or NULL to skip it
 *   D in {64, 128}; Hq % Hkv == 0; win_l, win_r >= -1 (-1 = unbounded on that side);
 *   causal != 0 enables the causal predicate; softcap == 0 disables the cap;
 *   scale: the caller's float, used as given (typically 1/sqrt(D)).
 *   Sizes of 0 for B, Hq or Nq are a no-op; Nk == 0 gives out = 0, lse = -inf.
 * Returns MFA_OK after the launch was queued, or a negative status (nothing launched).
 */
int mfa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
            int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
            int causal, int win_l, int win_r, float softcap, int dtype, void* stream);

/*
 * mfa_fwd_host -- mfa_fwd with q, k, v, out and lse in HOST memory, for callers whose tensors
 * live on the host (the same operation as "mlx-mfa 2.5.2" Usage, flash_attention(q, k, v,
 * causal=...), whose arrays sit in memory the host and GPU share; here the copies to and from
 * the device are part of the call).
 *
 * q, k, v, out: host buffers, layouts as mfa_fwd; lse: host float buffer [B, Hq, Nq] or NULL.
 * Page-locked (pinned) host memory lets the copies run asynchronously; pageable memory works but
 * each copy then blocks the calling thread until it is done.
 * scratch: device buffer of at least mfa_fwd_host_scratch_size(...) bytes, 256-byte aligned,
 * owned by the caller; it holds the device copies of all five tensors.
 * The B * Hkv (batch, kv head) units are split into contiguous runs of about 12 MiB of input
 * each (at most 8; one for small problems). Run c's inputs are
 * copied in on an internal stream while run c - 1 computes on `stream` and run c - 2's outputs
 * are copied out on a second internal stream; the internal streams are ordered after the work
 * queued on `stream` before the call, and `stream` is ordered after the last copy out. The call
 * returns once everything is queued: out and lse are complete when `stream` reaches this point
 * (synchronize it, or record an event, before reading them). Results are bitwise those of
 * mfa_fwd on the same data. Argument checks and error codes as mfa_fwd, plus MFA_ERR_WORKSPACE
 * for a NULL, misaligned or too small scratch. Concurrent calls from several host threads on one
 * device are serialised by the library while they queue their work.
 */
size_t mfa_fwd_host_scratch_size(int B, int Hq, int Hkv, int Nq, int Nk, int D);
int mfa_fwd_host(const void* q, const void* k, const void* v, void* out, float* lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
                 int causal, int win_l, int win_r, float softcap, int dtype,
                 void* scratch, size_t scratch_bytes, void* stream);

/*
 * mfa_fwd_varlen -- the same forward over a packed batch of variable-length sequences
 * ([MFA252] Features "Variable-length -- packed sequences with cu_seqlens"; [MXFA15] README
 * public entry point flash_attn_varlen_func; [MFA261] 2.61.0 notes that varlen causal with
 * N_q < N_k was changed toward bottom-right alignment, which this call follows per sequence).
 *
 * Sequence b has Nq_b = cu_seqlens_q[b+1] - cu_seqlens_q[b] query rows, stored at rows
 * cu_seqlens_q[b] ... of q and out, and Nk_b = cu_seqlens_k[b+1] - cu_seqlens_k[b] keys at rows
 * cu_seqlens_k[b] ... of k and v. Every sequence is attended exactly as mfa_fwd attends one
 * batch entry with Nq = Nq_b, Nk = Nk_b (a = i + Nk_b - Nq_b; keys of other sequences are never
 * visible); a sequence with Nk_b = 0 gets out = 0, lse = -inf.
 *
 * Arguments
 *   q    [total_q, Hq, D]  dtype      k, v [total_k, Hkv, D]  dtype          (read only)
 *   out  [total_q, Hq, D]  dtype      lse  [Hq, total_q] float32, or NULL
 *   cu_seqlens_q, cu_seqlens_k: int32 [B + 1] device arrays, 4-byte aligned, starting at 0,
 *   non-decreasing, ending at total_q / total_k;
 *   max_seqlen_q >= every Nq_b (it sizes the grid); other arguments as mfa_fwd.
 * The offsets live on the device, so they are checked by the kernel: a malformed entry or a
 * sequence longer than max_seqlen_q records MFA_ERR_DEVICE_BAD_SEQLENS (mfa_device_status) and
 * the affected sequence's outputs are not written. Returns MFA_OK after the launch was queued,
 * or a negative status (nothing launched).
 */
int mfa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                   const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                   int B, int max_seqlen_q, int total_q, int total_k,
                   int Hq, int Hkv, int D, float scale,
                   int causal, int win_l, int win_r, float softcap, int dtype, void* stream);

/*
 * mfa_fwd_blocksparse -- the dense forward restricted by a block mask ([MFA252] Features
 * "Block-sparse attention -- block_mask tensor skips entire tiles"; Usage
 * flash_attention_sparse(q, k, v, block_mask, causal=True)).
 *
 * Query row i of (b, h) may attend key j only if block_mask[b][h][i / 128][j / 128] != 0, in
 * addition to the causal / window predicates of mfa_fwd: vis(j) becomes vis(j) && mask bit. A
 * 128 x 128 block is one tile of the kernel, so a zero entry is never loaded or computed for the
 * query tile it belongs to (when both 128-row tiles of a 256-row block have it off). Rows left
 * with no visible key get out = 0, lse = -inf.
 *
 * Arguments as mfa_fwd, plus
 *   block_mask  uint8 [B, Hq, ceil(Nq / 128), ceil(Nk / 128)], row-major   (device)
 *   ceil(Nk / 128) <= 2048 (Nk <= 262,144), else MFA_ERR_UNSUPPORTED.
 */
int mfa_fwd_blocksparse(const void* q, const void* k, const void* v, void* out, float* lse,
                        const uint8_t* block_mask,
                        int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
                        int causal, int win_l, int win_r, float softcap, int dtype, void* stream);

/*
 * mfa_fwd_paged -- chunked prefill over a paged KV cache: packed variable-length query chunks
 * attend the keys their sequences hold in the page pool ([MFA252] Features "Paged KV" and
 * "Variable-length"; [MFA261] notes paged causal with heterogeneous seq_lens corrected toward
 * the per-sequence bottom-right alignment used here).
 *
 * Sequence b has Nq_b = cu_seqlens_q[b+1] - cu_seqlens_q[b] query rows (rows of q / out) and
 * seq_lens[b] keys; key t is slot t % 16 of page block_table[b][t / 16]. The queries are the
 * last Nq_b positions (a = i + seq_lens[b] - Nq_b), and each sequence is attended exactly as
 * mfa_fwd attends one batch entry with Nq = Nq_b, Nk = seq_lens[b]. With Nq_b <= 4 this is
 * mfa_decode_splitkv's definition.
 *
 * Arguments
 *   q, out       [total_q, Hq, D] dtype; lse [Hq, total_q] float32 or NULL       (device)
 *   k_pages, v_pages [num_pages, 16, Hkv, D] dtype                                (device)
 *   block_table  int32 [B, max_pages_per_seq]: entries for t < ceil(seq_lens[b] / 16) must lie
 *                in [0, num_pages); later entries are never read                    (device)
 *   seq_lens     int32 [B], each in [0, max_pages_per_seq * 16]                   (device)
 *   cu_seqlens_q int32 [B + 1] as mfa_fwd_varlen; max_seqlen_q >= every Nq_b; page_size 16.
 * Page slots at or past a sequence's length may hold any bit pattern (NaN included). Entries
 * that break these rules are reported through mfa_device_status (MFA_ERR_DEVICE_BAD_PAGE or
 * MFA_ERR_DEVICE_BAD_SEQLENS); the affected pages read as zeros.
 */
int mfa_fwd_paged(const void* q, const void* k_pages, const void* v_pages,
                  const int32_t* block_table, const int32_t* seq_lens, const int32_t* cu_seqlens_q,
                  void* out, float* lse, int B, int max_seqlen_q, int total_q,
                  int Hq, int Hkv, int D, int page_size, int max_pages_per_seq, int num_pages,
                  float scale, int causal, int win_l, int win_r, float softcap, int dtype,
                  void* stream);

/*
 * mfa_bwd_workspace_size -- bytes of scratch mfa_bwd needs: one fp32 per query row
 * (rowsum(dO * O)), 256-byte rounded. Returns 0 for invalid arguments.
 */
size_t mfa_bwd_workspace_size(int B, int Hq, int Nq);

/*
 * mfa_bwd -- backward of mfa_fwd: the gradients of sum(out * dout) with respect to q, k, v,
 * given the forward's out and lse ([MLXBUN] Backward: three passes -- D-vec, dKV, dQ -- that
 * recompute the scores from the saved log-sum-exp).
 *
 * With p_ij = exp(c_ij - lse_i) for visible pairs (c the scaled, optionally capped score),
 *   D_i  = sum_d dout[i,d] out[i,d],   dp_ij = <dout_i, v_j>,
 *   ds_ij = p_ij (dp_ij - D_i) (times 1 - tanh^2(s_ij / softcap) when softcap > 0),
 *   dq_i = scale sum_j ds_ij k_j,  dk_j = scale sum_i ds_ij q_i,  dv_j = sum_i p_ij dout_i,
 * with dk, dv summed over the query heads of each kv group. Every output element is written
 * by exactly one thread (no atomics): repeated calls give bitwise the same result.
 *
 * Arguments
 *   q, out, dout, dq  [B, Hq, Nq, D] dtype     k, v, dk, dv [B, Hkv, Nk, D] dtype    (device)
 *   lse  [B, Hq, Nq] float32 as written by mfa_fwd for the same arguments              (device)
 *   workspace: device scratch of at least mfa_bwd_workspace_size(B, Hq, Nq) bytes, 256-byte
 *   aligned, caller-owned; other arguments as mfa_fwd. Nk == 0 gives dq = 0; Nq == 0 gives
 *   dk = dv = 0. Returns MFA_OK after the launches were queued.
 */
int mfa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
            const float* lse, void* dq, void* dk, void* dv,
            int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
            int causal, int win_l, int win_r, float softcap, int dtype,
            void* workspace, size_t workspace_bytes, void* stream);

/*
 * mfa_decode_workspace_size -- bytes of scratch mfa_decode_splitkv needs for this shape.
 * The split plan is a function of these arguments only (not of seq_lens), so one workspace
 * serves every call with the same shape. Returns 0 for invalid arguments.
 */
size_t mfa_decode_workspace_size(int B, int Nq, int Hq, int Hkv, int D,
                                 int max_pages_per_seq, int page_size);

/*
 * mfa_decode_plan -- the split plan mfa_decode_splitkv_window (win_l >= 0) or
 * mfa_decode_splitkv (win_l = -1) uses for this shape, computed on the host without a launch:
 * *kv_heads_per_cta kv heads per phase-1 CTA (the most that divide Hkv with a token row of at
 * most 1 KB), *pages_per_split 16-token pages per split and *max_splits splits per sequence
 * (the phase-1 grid is max_splits x B x Hkv / kv_heads_per_cta). Without a window the split
 * starts at 32 pages and halves (down to 4) while that grid would hold fewer than 296 CTAs (two
 * per SM); with a window it is the smallest halving of 32 whose grid over the window's page
 * span still fits in 296 CTAs, never more splits than without the window. The override of
 * mfa_debug_set_decode_split_pages applies. Any output pointer may be NULL. Returns MFA_OK, or
 * the error code the decode entry point would return for these arguments.
 */
int mfa_decode_plan(int B, int Nq, int Hq, int Hkv, int D, int max_pages_per_seq, int page_size,
                    int win_l, int* pages_per_split, int* max_splits, int* kv_heads_per_cta);

/*
 * mfa_decode_splitkv -- two-phase split-KV decode over a paged KV cache
 * ([MFA252] Features "Flash Decode -- two-phase split-KV for N_q <= 4" and "Paged KV";
 *  [MXFA15] README: paged decode with per-split (m, l) slots and a combine step).
 *
 * Sequence b holds seq_lens[b] tokens; its token t is stored in page block_table[b][t / 16],
 * slot t % 16. Query token t (of Nq) sits at position seq_lens[b] - Nq + t; with causal != 0 it
 * sees keys at positions <= its own. Phase 1 splits each sequence into runs of pages and
 * computes, per run, unnormalised partial outputs with their running max and sum; phase 2
 * merges the runs with max-rescaling. The result equals mfa_fwd's definition on the gathered
 * K/V (up to fp32 rounding order).
 *
 * Arguments
 *   q            [B, Hq, Nq, D] dtype, Nq in [1, 4]          (device)
 *   k_pages      [num_pages, 16, Hkv, D] dtype                (device)
 *   v_pages      [num_pages, 16, Hkv, D] dtype                (device)
 *   block_table  int32 [B, max_pages_per_seq]; entries for pages t < ceil(len/16) must lie in
 *                [0, num_pages); later entries are never read    (device)
 *   seq_lens     int32 [B], each in [0, max_pages_per_seq * 16]  (device)
 *   out          [B, Hq, Nq, D] dtype; lse float32 [B, Hq, Nq] or NULL   (device)
 *   page_size must be 16; (Hq / Hkv) * Nq <= 16; D in {64, 128, 256};
 *   workspace: device scratch of at least mfa_decode_workspace_size(...) bytes, 256-byte
 *   aligned, owned by the caller; its contents need no initialisation and are overwritten.
 * Page slots at or past a sequence's length are never used in the arithmetic, so they may hold
 * any bit pattern (NaN included). Returns MFA_OK after both launches were queued.
 */
int mfa_decode_splitkv(const void* q, const void* k_pages, const void* v_pages,
                       const int32_t* block_table, const int32_t* seq_lens,
                       void* out, float* lse,
                       int B, int Nq, int Hq, int Hkv, int D, int page_size,
                       int max_pages_per_seq, int num_pages,
                       float scale, int causal, float softcap, int dtype,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * mfa_decode_splitkv_window -- mfa_decode_splitkv with a left window ([MFA252] Features:
 * window_size=(left, right) for local-attention layers, here in decode): query token t (at
 * position a = seq_lens[b] - Nq + t) sees keys j with a - win_l <= j (and j <= a when causal);
 * win_l = -1 is mfa_decode_splitkv. Splits are counted from the first page that some query
 * token can see, so pages wholly left of every window are never read, and the split size is
 * chosen from the window's page span rather than max_pages_per_seq. Arguments as
 * mfa_decode_splitkv plus win_l >= -1 (MFA_ERR_BAD_WINDOW otherwise); the workspace that
 * mfa_decode_workspace_size reports (which has no window argument) is always sufficient.
 */
int mfa_decode_splitkv_window(const void* q, const void* k_pages, const void* v_pages,
                              const int32_t* block_table, const int32_t* seq_lens,
                              void* out, float* lse,
                              int B, int Nq, int Hq, int Hkv, int D, int page_size,
                              int max_pages_per_seq, int num_pages,
                              float scale, int causal, int win_l, float softcap, int dtype,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Human-readable text for a status code (static storage). */
const char* mfa_status_string(int code);

/*
 * Launch record of the last successful call on this host thread: which kernel ran and with
 * what schedule ([MXFA15] README keeps a per-dispatch record; this is the same idea).
 */
typedef struct mfa_launch_info {
    int kernel;                 /* 1 = prefill forward, 2 = decode phase 1 + combine, 3 = empty-key fill */
    int grid_x, grid_y, grid_z; /* grid of the main kernel */
    int block_threads;          /* threads per CTA of the main kernel */
    int smem_bytes;             /* dynamic shared memory per CTA of the main kernel */
    int tile_m, tile_n;         /* prefill: query rows per Q tile, keys per K/V tile */
    int q_tiles_per_cta;        /* prefill: Q tiles per CTA */
    int pages_per_split;        /* decode: pages per split */
    int max_splits;             /* decode: splits per sequence at max_pages_per_seq */
    int kv_heads_per_cta;       /* decode: kv heads handled by one CTA */
} mfa_launch_info;

int mfa_last_launch_info(mfa_launch_info* info);

/*
 * Device status: copies the kernels' status word to *code (MFA_OK or MFA_ERR_DEVICE_*) and
 * *detail (where it happened), then clears it. Synchronises `stream`. For tests and debugging.
 */
int mfa_device_status(void* stream, int* code, int* detail);

/*
 * Debug switches (process-wide; default 0). Bit 0: the forward visits every key tile and masks
 * element-wise instead of skipping tiles. Bit 1: count the key tiles each forward CTA visits
 * into a device counter read by mfa_debug_tiles_visited. Bit 2: the forward's MMA thread issues
 * nothing, so the softmax warps' first bounded wait runs out after 2 s; the kernel then records
 * MFA_ERR_DEVICE_TIMEOUT in the device status, writes out = 0 and lse = -inf, releases TMEM and
 * returns, leaving the context usable (for tests of the failure path). Returns the previous
 * flags.
 */
#define MFA_DEBUG_NO_TILE_SKIP 1
#define MFA_DEBUG_COUNT_TILES  2
#define MFA_DEBUG_WITHHOLD_MMA 4
int mfa_debug_set_flags(int flags);

/* Reads and resets the tile counter (synchronises `stream`). */
int mfa_debug_tiles_visited(void* stream, unsigned long long* count);

/*
 * mfa_decode_phase1 / mfa_decode_combine -- the two phases of mfa_decode_splitkv_window as
 * separate calls, for a decode whose splits are spread over several GPUs (each GPU holds the
 * pages of some splits of every sequence). Source: [MFA252] Features (Flash Decode: two-phase
 * split-KV) and [MXFA15] README (per-split (m, l) slots merged by a combine step); spreading the
 * splits over GPUs is this library's use of the same two phases.
 *
 * The split plan is mfa_decode_plan's for the shape and win_l: splits s = 0 .. max_splits - 1,
 * split s of a sequence covering pages [first + s * pages_per_split, first + (s + 1) *
 * pages_per_split) of it (first = 0 without a window).
 *
 * Partial results are split-major, so a range of splits is one contiguous block of each array:
 *   part_o   float [split_capacity][B][Hq * Nq][D]   unnormalised O of the split's keys
 *   part_ml  float [split_capacity][B][Hq * Nq][2]   (running max in log2 units, running sum)
 * (row index (h * Nq + t)); split_capacity >= max_splits; both 16-byte aligned device buffers
 * owned by the caller.
 *
 * mfa_decode_phase1 computes the partials of splits [split_lo, split_hi) (0 <= split_lo <=
 * split_hi <= max_splits) of every sequence and kv head into their slots; it reads only the
 * block_table entries and pages of those splits, so a GPU's pool need hold only those pages.
 * Slots of splits past a sequence's end are left untouched. Arguments as mfa_decode_splitkv_window.
 *
 * mfa_decode_combine merges, for every (sequence, query head, token), the slots of splits
 * 0 .. n_splits(b) - 1 of part_o / part_ml (every one must have been written, by some GPU's
 * phase 1, and be visible on this stream) into out and lse, as mfa_decode_splitkv does.
 *
 * Gathering: with the splits cut into equal ranges of c splits per GPU (split_capacity = c x
 * number of GPUs), GPU r's block of each array starts at split r * c, so one all-gather of the
 * blocks in rank order leaves every GPU with the arrays a single GPU computing all splits writes.
 * Returns MFA_OK after the launch was queued, or a negative status (MFA_ERR_WORKSPACE when
 * split_capacity < max_splits or a partial pointer is NULL).
 */
int mfa_decode_phase1(const void* q, const void* k_pages, const void* v_pages,
                      const int32_t* block_table, const int32_t* seq_lens, int B, int Nq, int Hq,
                      int Hkv, int D, int page_size, int max_pages_per_seq, int num_pages,
                      float scale, int causal, int win_l, float softcap, int dtype, int split_lo,
                      int split_hi, float* part_o, float* part_ml, int split_capacity,
                      void* stream);
int mfa_decode_combine(const int32_t* seq_lens, void* out, float* lse, int B, int Nq, int Hq,
                       int Hkv, int D, int page_size, int max_pages_per_seq, int win_l, int dtype,
                       const float* part_o, const float* part_ml, int split_capacity,
                       void* stream);

/*
 * Tensor-map cache counters: map lookups made by launches so far and how many of them had to
 * encode a map (cuTensorMapEncodeTiled) because no map of the same (device, base pointer, data
 * type, layout, extents) was cached. A second call over the same buffers encodes nothing.
 */
int mfa_debug_tmap_stats(unsigned long long* lookups, unsigned long long* encodes);

/*
 * Host-only check of the tensor-map cache (no GPU or driver needed): looks up the key (base,
 * kind 0 dense / 1 packed / 2 pages, dtype, outer, n, D) under a device number no launch uses,
 * encoding a placeholder map on a miss. *encoded = 1 on a miss, 0 on a hit; the counters of
 * mfa_debug_tmap_stats include these lookups. Returns MFA_OK, or MFA_ERR_CUDA if a hit returned
 * a map built for another key.
 */
int mfa_debug_tmap_probe(const void* base, int kind, int dtype, long long outer, long long n, int D,
                         int* encoded);

/*
 * Decode split size override in pages (0 = automatic, at most 64). It changes the split plan,
 * and with it mfa_decode_workspace_size. Returns the previous value.
 */
int mfa_debug_set_decode_split_pages(int pages);

/*
 * mfa_decode_splitkv_noalloc -- mfa_decode_splitkv for callers that cannot allocate device
 * memory. The paper has no counterpart of this entry point; it exists for this library's users.
 *
 * Some callers cannot call cudaMalloc when decode runs: a serving engine that reserves all of
 * HBM for its KV page pool up front and hands out nothing else, code running inside an
 * allocator or memory-pool callback (where re-entering the allocator is not allowed), and
 * latency-critical decode loops that cannot afford cudaMalloc's implicit device
 * synchronisation. They cannot provide mfa_decode_splitkv's workspace. This variant keeps that workspace in a fixed
 * device array inside the library instead of taking one from the caller; every other argument
 * has the meaning given for mfa_decode_splitkv, and the computation and result are the same.
 *
 *   - The array holds MFA_NOALLOC_SCRATCH_BYTES (64 MiB). A device takes it when the library's
 *     code is first used there (under CUDA's lazy module loading that can be this entry point's
 *     first call, whose address lookup loads the module) and holds it until the process exits.
 *     A shape whose workspace
 *     (mfa_decode_workspace_size) is larger is rejected with MFA_ERR_SCRATCH_TOO_SMALL before
 *     anything runs; the paged decode of 8 sequences x 131072 tokens with 32 query heads, 8 kv
 *     heads and D = 128 needs about 34 MB.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress with
 *     that device current; this can also load the module and take the array) and remembers it;
 *     make that first call before any stream capture.
 *   - No call allocates or frees memory.
 *   - All calls on a device share the one array and leave their partial results in it. Calls
 *     whose kernels overlap on the GPU (different streams without ordering, or concurrent
 *     host threads) race on it and give wrong results; order them on one stream. Nothing in the
 *     array needs to start at zero: each call writes every entry it later reads.
 * Returns MFA_OK after both launches were queued, or a negative status.
 */
#define MFA_NOALLOC_SCRATCH_BYTES (64u << 20)
int mfa_decode_splitkv_noalloc(const void* q, const void* k_pages, const void* v_pages,
                               const int32_t* block_table, const int32_t* seq_lens,
                               void* out, float* lse,
                               int B, int Nq, int Hq, int Hkv, int D, int page_size,
                               int max_pages_per_seq, int num_pages,
                               float scale, int causal, float softcap, int dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MFA_H_ */
