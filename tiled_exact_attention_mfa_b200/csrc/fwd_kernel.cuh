// fwd_kernel.cuh -- exact attention forward (prefill) for sm_100a.
//
// Algorithm: FlashAttention-2 style single pass over K/V tiles with an online softmax (running
// row max m, running sum l, fp32 accumulator O), as in the forward shader of "mlx-bun 0.4.0 ->
// 1.0.0, src/model/flash-attention.ts": S = scale * Q K^T per tile, m_new = max(m, rowmax(S)),
// alpha = exp(m - m_new), P = exp(S - m_new), l = alpha l + rowsum(P), O = alpha O + P V, and at
// the end O / l and LSE = m + ln l. A tile whose every score of a row is masked leaves that
// row untouched (the shader's m_new = -inf guard).
//
// B200 mapping, default shape (one CTA per SM, 384 threads, 2 Q tiles of 128 rows per CTA;
// setmaxnreg gives the softmax warpgroups 200 registers per thread and the producer / MMA
// warpgroup 104; the single-Q-tile shape that uncapped dense calls use is described at FwdShape):
//   warp 8      TMA producer: Q tiles once, then K and V tiles through 2-stage rings (128-byte
//               swizzled smem, 3-D tensor maps so tails are zero-filled per head).
//   warp 9      TMEM owner and single-thread tcgen05.mma issuer:
//                 S_t = Q_t K^T   (M=128, N=128, K=D; A and B K-major from smem)
//                 O_t += P_t V    (M=128, N=D, K=128; P_t from TMEM, V MN-major from smem)
//   warps 0-3   softmax for Q tile 0, warps 4-7 for Q tile 1: one TMEM lane = one query row =
//               one thread, so row max / row sum are thread-local. Scores are kept in the log2
//               domain (scale * log2 e folded into one FFMA). The running max is only moved when
//               it grows by more than 2^8 (rescaling is exact for any reference max; a stale one
//               only bounds P by 2^8), and then O is rescaled in TMEM by the owning warp.
//   TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,256+D) O_1 [256+D, 256+2D) (one Q tile:
//                 S [0,128), O [128,128+D)); P_t (16-bit, 2 per column) overwrites the first
//                 64 columns of S_t.
// Ordering: QK for tile j+1 of Q tile t overwrites S_t's columns, where PV for tile j reads P_t
// from. tcgen05 only orders MMAs that share an accumulator, so the MMA thread waits for that PV
// to complete before issuing the QK (issuing it right behind the PV would rely on an execution
// order the rules do not give; it measured ~2 % faster and is not built). The commit that
// signals S_t ready covers every earlier MMA, so when the softmax of tile j+1 starts, PV of tile
// j is done and O_t can be rescaled in place.
//
// Tile skip ("mlx-mfa 2.5.2", Features: causal tile-skip, window_size=(left,right) tile skip):
// each CTA visits only key tiles that intersect the union of its rows' visible ranges, and each
// of its Q tiles computes only those that intersect its own rows' range (the two differ by up to
// a tile at each end: the causal diagonal, the window's edges); inside, masking is applied per
// element only on tiles that are not fully visible to all 128 rows.
#pragma once
#include "sm100.cuh"

namespace mfa {

constexpr int kFwdBM = 128;       // query rows per Q tile (= TMEM lanes)
constexpr int kFwdBN = 128;       // keys per K/V tile
// Two CTA shapes. The default holds two Q tiles (384 threads: 8 softmax warps, then a
// warpgroup of producer + MMA + 2 idle warps; 512 TMEM columns; ~198 KB of shared memory at
// D = 128; one CTA per SM), whose softmax phases interleave on one tensor core. ONE holds a
// single Q tile (256 threads: 4 softmax warps, then the same control warpgroup; 256 TMEM
// columns; at D = 128 one K and one V stage, ~98 KB; two CTAs per SM): the two resident CTAs
// interleave the same way, and one CTA's start (Q load, first QK) and end (last PV, O store)
// overlap the other's key tiles. With the speculative reference max below, ONE is the faster
// shape for uncapped dense calls; capped, packed, block-sparse and paged calls use the default.
// setmaxnreg moves registers from the control warpgroup to the softmax warpgroups; each split
// adds up to the registers the CTA launches with (threads x launch-bound registers).
template <bool ONE>
struct FwdShape {
  static constexpr int kQT = ONE ? 1 : 2;                // Q tiles per CTA
  static constexpr int kThreads = ONE ? 256 : 384;
  static constexpr int kMinBlocks = ONE ? 2 : 1;          // CTAs per SM the launch bounds ask for
  static constexpr int kProducerWarp = ONE ? 4 : 8;
  static constexpr int kMmaWarp = ONE ? 5 : 9;
  static constexpr int kTmemCols = ONE ? 256 : 512;       // S of each Q tile, then O of each
  static constexpr int kRegsSoftmax = ONE ? 192 : 200;    // per thread after setmaxnreg
  static constexpr int kRegsControl = ONE ? 64 : 104;
  static constexpr int kRegsLaunch = ONE ? 128 : 168;     // 65,536 / (threads x CTAs per SM), rounded
  static_assert(kQT * 128 * kRegsSoftmax + 128 * kRegsControl == kThreads * kRegsLaunch,
                "the setmaxnreg split must use exactly the CTA's launch registers");
};
template <int D, bool ONE>
__host__ __device__ constexpr int fwd_stages() {  // K ring and V ring depth
  return (ONE && D == 128) ? 1 : 2;
}
constexpr float kRescaleLog2 = 8.0f;
constexpr int kFwdMaxSparseTiles = 2048;  // key tiles a block-sparse row may span (262,144 keys)
#ifndef MFA_POLY_MASK
#define MFA_POLY_MASK 0x0ull
#endif
// Pairs of P computed with the FMA-pipe exp2 (bit i of the mask = pair i of the 64 per row).
__host__ __device__ constexpr bool kPolyPair(int i) { return (MFA_POLY_MASK >> i) & 1ull; }

struct FwdParams {
  CUtensorMap tm_q;  // [B*Hq][Nq][D]
  CUtensorMap tm_k;  // [B*Hkv][Nk][D]
  CUtensorMap tm_v;
  CUtensorMap tm_o;  // out, laid out as q (the epilogue's TMA stores)
  void* out;
  float* lse;
  unsigned long long* tile_counter;
  // packed variable-length batches: sequence b holds rows [cu_q[b], cu_q[b+1]) of q / out and
  // [cu_k[b], cu_k[b+1]) of k / v (device arrays of B + 1 offsets); NULL for the dense layout
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  // block-sparse: uint8 [B, Hq, nqt, nkt], one entry per 128-row x 128-key block (0 = skip)
  const uint8_t* block_mask;
  int nqt, nkt;
  // paged keys (with packed queries): sequence b's key t is slot t % 16 of page
  // block_table[b * max_pages + t / 16] of the pools [num_pages, 16, Hkv, D]; seq_lens[b] keys
  const int* block_table;
  const int* seq_lens;
  int max_pages, num_pages;
  int B, Hq, Hkv, Nq, Nk, G;
  int causal, win_l, win_r;
  int n_qblk;       // number of 256-row query blocks per head
  int flags;        // bit 0: no tile skip; bit 1: count tiles; bit 2: withhold every MMA
  float c_log2;     // factor taking the stored score to the log2 domain
  float softcap;    // 0 = off
  float cap_in;     // scale / softcap
  float cap_out;    // softcap / scale
  float lse_mul;    // ln 2
};

template <int D, bool SPARSE, bool ONE = false>
struct FwdSmem {
  static constexpr int kTileBytes = kFwdBM * D * 2;  // one 128 x D tile of 16-bit values
  static constexpr int kSlabBytes = 128 * 128;       // 128 rows x 64 columns (128 B) slab
  static constexpr int kQT = FwdShape<ONE>::kQT;
  static constexpr int kNS = fwd_stages<D, ONE>();
  uint8_t q[kQT][kTileBytes];
  uint8_t k[kNS][kTileBytes];
  uint8_t v[kNS][kTileBytes];
  uint64_t bar_q;
  uint64_t bar_k_full[kNS], bar_k_empty[kNS];
  uint64_t bar_v_full[kNS], bar_v_empty[kNS];
  // P of a Q tile becomes ready in two halves (keys 0-63, 64-127), so the first half of PV can
  // run while the second half of the exponentials is computed
  uint64_t bar_s_full[kQT], bar_p_full[kQT][2], bar_o_done[kQT];
  uint64_t bar_final;
  uint32_t tmem_base;
  int abort;
  int n_act;                                  // block-sparse: key tiles this CTA visits
  uint16_t act_tile[SPARSE ? kFwdMaxSparseTiles : 1];  // ... their indices (from kt_lo), ascending
  uint8_t act_bits[SPARSE ? kFwdMaxSparseTiles : 1];   // ... bit t: Q tile t's block is on
};

template <int D, bool SPARSE, bool ONE = false>
constexpr int fwd_smem_bytes() {
  return (int)sizeof(FwdSmem<D, SPARSE, ONE>) + 1024;  // + alignment slack for the 1024-byte swizzle atoms
}

// Visible key range [lo, hi) of absolute query positions [a0, a1] (inclusive) among Nk keys.
__device__ __forceinline__ void key_range(const FwdParams& p, int Nk, int a0, int a1, int& lo, int& hi) {
  lo = 0;
  hi = Nk;
  if (p.causal) hi = min(hi, a1 + 1);
  if (p.win_r >= 0) hi = min(hi, a1 + p.win_r + 1);
  if (p.win_l >= 0) lo = max(lo, a0 - p.win_l);
}

// VARLEN: q / out are [total_q, Hq, D] and k / v [total_k, Hkv, D] with per-sequence offsets
// (cu_q, cu_k), read through tensor maps ordered (D, head, token); lse is [Hq, total_q]. Otherwise q / out are [B, Hq, Nq, D], k / v
// [B, Hkv, Nk, D] and lse [B, Hq, Nq].
// SPARSE: dense layout plus a block mask; a CTA visits only key tiles whose block is on for one
// of its Q tiles and which that Q tile's rows can see (causal / window); a Q tile takes no part
// (no MMA, no softmax) in a visited tile that is not its own, and its barriers count only the
// tiles it takes part in.
// SOFTCAP: compiled with the softcap transform (p.softcap > 0); without it the softmax carries
// no softcap code at all.
// PAGED (with VARLEN queries): K / V tiles are assembled from 16-token pages through the block
// table (8 TMA boxes per 128-key tile, maps ordered (D, head, pool token)); pages past the
// sequence are loaded from past the pool's end, which TMA fills with zeros. Value rows at or past
// the length inside the last page may hold anything, so before P of that tile is released the
// first softmax warpgroup zeroes them in shared memory (P is 0 there, but 0 x NaN is NaN).
// PART (dense layout): each Q tile computes only the key tiles its own rows can see, instead of
// every tile of the CTA's range; chosen for sliding windows, where the two Q tiles' ranges
// differ by a tile at each end (elsewhere the saving is one diagonal tile per CTA, less than what
// the extra bookkeeping costs the plain loop).
// ONE: the single-Q-tile CTA shape (FwdShape).
template <int D, bool BF16, bool VARLEN, bool SPARSE, bool SOFTCAP, bool PAGED, bool PART = false, bool ONE = false>
__global__ void __launch_bounds__(FwdShape<ONE>::kThreads, FwdShape<ONE>::kMinBlocks)
    mfa_fwd_kernel(const __grid_constant__ FwdParams p) {
  constexpr bool kRuns = PART && !SPARSE;  // Q tile t takes part in the run [jlo_t, jhi_t)
  constexpr bool kPart = SPARSE || kRuns;  // a Q tile may sit out some visited tiles
  constexpr int kFwdQT = FwdShape<ONE>::kQT;  // Q tiles of this CTA shape
  constexpr int kFwdStages = fwd_stages<D, ONE>();
  constexpr int kProd = FwdShape<ONE>::kProducerWarp;
  constexpr int kMma = FwdShape<ONE>::kMmaWarp;
  constexpr int kOCol = kFwdQT * kFwdBN;  // first TMEM column of O (after the S of each Q tile)
  using Smem = FwdSmem<D, SPARSE, ONE>;
  static_assert(!(VARLEN && SPARSE), "block masks are defined on the dense layout");
  static_assert(!PAGED || VARLEN, "paged keys come with packed queries");
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: heavy query blocks first (causal blocks near the end see the most keys)
  const int BH = p.B * p.Hq;
  const int qb = p.n_qblk - 1 - (int)(blockIdx.x / BH);
  const int bh = blockIdx.x % BH;
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int g = h / p.G;
  const int q0 = qb * (kFwdBM * kFwdQT);
  int Nq = p.Nq, Nk = p.Nk;  // this sequence's query and key counts
  int rq = 0, rk = 0;        // its first row in the packed q / k (VARLEN)
  if constexpr (VARLEN) {
    rq = p.cu_q[b];
    const int eq = p.cu_q[b + 1];
    int ek;
    if constexpr (PAGED) {
      rk = 0;
      ek = p.seq_lens[b];
      if (ek < 0 || ek > p.max_pages * 16) {
        if (threadIdx.x == 0 && qb == 0 && h == 0) record_status(-22, 0x40000000 + b);
        return;
      }
    } else {
      rk = p.cu_k[b];
      ek = p.cu_k[b + 1];
    }
    if (rq < 0 || eq < rq || eq > p.total_q || rk < 0 || ek < rk || (!PAGED && ek > p.total_k)) {
      if (threadIdx.x == 0 && qb == 0 && h == 0) record_status(-24, b);
      return;  // the whole CTA, before any barrier or TMEM allocation
    }
    Nq = eq - rq;
    Nk = ek - rk;
    // rows past the grid's query blocks would never be computed: report the short max_seqlen_q
    if (threadIdx.x == 0 && qb == p.n_qblk - 1 && h == 0 && Nq > p.n_qblk * kFwdBM * kFwdQT)
      record_status(-24, b);
    if (q0 >= Nq) return;  // a shorter sequence has fewer query blocks
  }
  const int off = Nk - Nq;
  const int q_last = min(q0 + kFwdBM * kFwdQT, Nq) - 1;

  int lo, hi;
  key_range(p, Nk, q0 + off, q_last + off, lo, hi);
  if (p.flags & 1) {
    lo = 0;
    hi = Nk;
  }
  const int kt_lo = lo / kFwdBN;
  const int n_tiles = (hi > lo) ? ((hi + kFwdBN - 1) / kFwdBN - kt_lo) : 0;
  // each Q tile's own visible key range: a key tile it cannot see at all is not its to visit
  // (the two Q tiles' ranges differ by up to a tile at each end: causal diagonal, window edges)
  int vlo0, vhi0, vlo1, vhi1;  // (scalars, not arrays: selected, never indexed)
  {
    int vlo[kFwdQT], vhi[kFwdQT];
#pragma unroll
    for (int t = 0; t < kFwdQT; ++t) {
      const int f = q0 + t * kFwdBM, l = min(f + kFwdBM, Nq) - 1;
      if (l < f) {
        vlo[t] = 1;
        vhi[t] = 0;
      } else if (p.flags & 1) {
        vlo[t] = 0;
        vhi[t] = Nk;
      } else {
        key_range(p, Nk, f + off, l + off, vlo[t], vhi[t]);
      }
    }
    vlo0 = vlo[0];
    vhi0 = vhi[0];
    vlo1 = kFwdQT > 1 ? vlo[kFwdQT - 1] : 1;  // (one Q tile: a second that sees nothing)
    vhi1 = kFwdQT > 1 ? vhi[kFwdQT - 1] : 0;
  }
  // bit t: Q tile t takes part in key tile kt (intersects its visible range)
  auto vis_bits = [&](int kt) -> uint32_t {
    const int k0 = kt * kFwdBN;
    return ((k0 < vhi0 && k0 + kFwdBN > vlo0) ? 1u : 0u) | ((k0 < vhi1 && k0 + kFwdBN > vlo1) ? 2u : 0u);
  };

  // ---- setup: the producer thread initialises the barriers and starts the Q load at once, so
  // the copy overlaps the TMEM allocation, the block-sparse tile list and the CTA barrier
  const bool q_early = n_tiles > 0;
  if (warp == kProd && lane == 0) {
    mbar_init(smem_u32(&sm.bar_q), 1);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(smem_u32(&sm.bar_k_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_k_empty[s]), 1);
      mbar_init(smem_u32(&sm.bar_v_full[s]), 1);
      mbar_init(smem_u32(&sm.bar_v_empty[s]), 1);
    }
    for (int t = 0; t < kFwdQT; ++t) {
      mbar_init(smem_u32(&sm.bar_s_full[t]), 1);
      mbar_init(smem_u32(&sm.bar_p_full[t][0]), kFwdBM / 32);  // one arrival per softmax warp
      mbar_init(smem_u32(&sm.bar_p_full[t][1]), kFwdBM / 32);
      mbar_init(smem_u32(&sm.bar_o_done[t]), 1);
    }
    mbar_init(smem_u32(&sm.bar_final), 1);
    sm.abort = 0;
    fence_barrier_init();
    if (q_early) {
      tma_prefetch_desc(&p.tm_q);
      const uint32_t bq = smem_u32(&sm.bar_q);
      mbar_expect_tx(bq, kFwdQT * (uint32_t)Smem::kTileBytes);
      for (int t = 0; t < kFwdQT; ++t)
        for (int sl = 0; sl < D / 64; ++sl)
          if constexpr (VARLEN)
            tma_load_3d(smem_u32(sm.q[t]) + sl * Smem::kSlabBytes, &p.tm_q, bq, sl * 64,
                        h, rq + q0 + t * kFwdBM);
          else
            tma_load_3d(smem_u32(sm.q[t]) + sl * Smem::kSlabBytes, &p.tm_q, bq, sl * 64,
                        q0 + t * kFwdBM, b * p.Hq + h);
    }
  }
  if (SPARSE && warp == 0) {
    // Active key tiles of the block mask rows of this CTA's two Q tiles, compacted in order:
    // 32 lanes read 8 tiles each per step (all loads issued before the ballots).
    const int qt0 = q0 / kFwdBM;
    const uint8_t* r0 = p.block_mask + ((size_t)(b * p.Hq + h) * p.nqt + qt0) * p.nkt + kt_lo;
    const uint8_t* r1 = (kFwdQT > 1 && qt0 + 1 < p.nqt) ? r0 + p.nkt : nullptr;
    int count = 0;
    for (int base = 0; base < n_tiles; base += 32 * 8) {
      uint8_t a0[8], a1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int jj = base + i * 32 + lane;
        const uint32_t vb = vis_bits(kt_lo + jj);
        a0[i] = (jj < n_tiles && (vb & 1u)) ? r0[jj] : 0;
        a1[i] = (r1 != nullptr && jj < n_tiles && (vb & 2u)) ? r1[jj] : 0;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool act = (a0[i] | a1[i]) != 0;
        const unsigned bal = __ballot_sync(0xffffffffu, act);
        if (act) {
          const int pos = count + __popc(bal & ((1u << lane) - 1u));
          if (pos < kFwdMaxSparseTiles) {  // the host keeps every list within the capacity
            sm.act_tile[pos] = (uint16_t)(base + i * 32 + lane);
            sm.act_bits[pos] = (uint8_t)((a0[i] != 0 ? 1 : 0) | (a1[i] != 0 ? 2 : 0));
          }
        }
        count += __popc(bal);
      }
    }
    if (lane == 0) {
      if (count > kFwdMaxSparseTiles) record_status(-25, count);
      sm.n_act = min(count, kFwdMaxSparseTiles);
    }
  }
  if (warp == kMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), FwdShape<ONE>::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProd && lane == 0) {
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // the key tiles every role walks: u-th visited tile = kt_lo + tile_of(u)
  const int n_act = SPARSE ? sm.n_act : n_tiles;
  auto tile_of = [&](int u) -> int {
    if constexpr (SPARSE) return sm.act_tile[u]; else return u;
  };
  // bit t of visited tile u: Q tile t takes part in it (block-sparse: its block is on as well)
  // Dense: Q tile t's visited tiles are the contiguous run [jlo_t, jhi_t) of the CTA's.
  const int jlo0 = min(n_tiles, max(0, vlo0 / kFwdBN - kt_lo));
  const int jhi0 = max(jlo0, min(n_tiles, (vhi0 + kFwdBN - 1) / kFwdBN - kt_lo));
  const int jlo1 = min(n_tiles, max(0, vlo1 / kFwdBN - kt_lo));
  const int jhi1 = max(jlo1, min(n_tiles, (vhi1 + kFwdBN - 1) / kFwdBN - kt_lo));
  auto bits_of = [&](int u) -> uint32_t {  // bit t: Q tile t takes part in visited tile u
    if constexpr (SPARSE) return sm.act_bits[u];
    else if constexpr (kRuns) return ((u >= jlo0 && u < jhi0) ? 1u : 0u) | ((u >= jlo1 && u < jhi1) ? 2u : 0u);
    else return kFwdQT > 1 ? 3u : 1u;
  };
  if (threadIdx.x == 0 && (p.flags & 2) && n_act > 0)
    atomicAdd(p.tile_counter, (unsigned long long)n_act);
  volatile int* abort = &sm.abort;

  constexpr int kSlabs = D / 64;
  constexpr uint32_t kTileBytes = Smem::kTileBytes;
  constexpr int kSlab = Smem::kSlabBytes;

  if (warp >= kProd) {
   regs_dec<FwdShape<ONE>::kRegsControl>();
   if (warp == kProd) {
    // ================================================================ TMA producer
    const uint32_t bq = smem_u32(&sm.bar_q);
    if (lane == 0 && n_act > 0) {  // (the Q tiles were requested during setup)
      int issued_k[kFwdStages] = {}, issued_v[kFwdStages] = {};
      for (int u = 0; u < n_act; ++u) {
        const int s = u % kFwdStages;
        const int use = u / kFwdStages;
        const int row = (kt_lo + tile_of(u)) * kFwdBN;
        if (use > 0 && !mbar_wait(smem_u32(&sm.bar_k_empty[s]), (use - 1) & 1, abort, 801)) break;
        // pool token of each of the tile's 8 pages (past the sequence: past the pool, zero-filled)
        int ptok[PAGED ? 8 : 1];
        if constexpr (PAGED) {
#pragma unroll
          for (int pi = 0; pi < 8; ++pi) {
            const int lp = row / 16 + pi;
            int tok = p.num_pages * 16;
            if (lp * 16 < Nk) {
              const int pg = p.block_table[(size_t)b * p.max_pages + lp];
              if (pg >= 0 && pg < p.num_pages) tok = pg * 16;
              else record_status(-22, b);
            }
            ptok[pi] = tok;
          }
        }
        const uint32_t bk = smem_u32(&sm.bar_k_full[s]);
        mbar_expect_tx(bk, kTileBytes);
        for (int sl = 0; sl < kSlabs; ++sl) {
          if constexpr (PAGED) {
#pragma unroll
            for (int pi = 0; pi < 8; ++pi)
              tma_load_3d(smem_u32(sm.k[s]) + sl * kSlab + pi * 16 * 128, &p.tm_k, bk, sl * 64, g, ptok[pi]);
          } else {
            tma_load_3d(smem_u32(sm.k[s]) + sl * kSlab, &p.tm_k, bk, sl * 64, VARLEN ? g : row,
                        VARLEN ? rk + row : b * p.Hkv + g);
          }
        }
        issued_k[s] = use + 1;
        if (use > 0 && !mbar_wait(smem_u32(&sm.bar_v_empty[s]), (use - 1) & 1, abort, 802)) break;
        const uint32_t bv = smem_u32(&sm.bar_v_full[s]);
        mbar_expect_tx(bv, kTileBytes);
        for (int sl = 0; sl < kSlabs; ++sl) {
          if constexpr (PAGED) {
#pragma unroll
            for (int pi = 0; pi < 8; ++pi)
              tma_load_3d(smem_u32(sm.v[s]) + sl * kSlab + pi * 16 * 128, &p.tm_v, bv, sl * 64, g, ptok[pi]);
          } else {
            tma_load_3d(smem_u32(sm.v[s]) + sl * kSlab, &p.tm_v, bv, sl * 64, VARLEN ? g : row,
                        VARLEN ? rk + row : b * p.Hkv + g);
          }
        }
        issued_v[s] = use + 1;
      }
      // Make sure no copy into this CTA's shared memory is still in flight when it exits.
      volatile int no_abort = 0;
      for (int s = 0; s < kFwdStages; ++s) {
        if (issued_k[s] > 0) mbar_wait(smem_u32(&sm.bar_k_full[s]), (issued_k[s] - 1) & 1, &no_abort, 804);
        if (issued_v[s] > 0) mbar_wait(smem_u32(&sm.bar_v_full[s]), (issued_v[s] - 1) & 1, &no_abort, 805);
      }
    }
    if (lane == 0 && q_early) {  // the Q copy, also when a block-sparse list came out empty
      volatile int no_abort = 0;
      mbar_wait(bq, 0, &no_abort, 803);
    }
  } else if (warp == kMma) {
    // ================================================================ MMA issuer
    if (lane == 0 && n_act > 0) {
      const uint32_t idesc_qk = idesc_f16(BF16 ? 1 : 0, kFwdBM, kFwdBN, 0);
      const uint32_t idesc_pv = idesc_f16(BF16 ? 1 : 0, kFwdBM, D, 1);
      // descriptors of the tiles' first bytes, built once (selected, not indexed, so they stay in
      // registers); each MMA adds a constant offset
      static_assert(kFwdQT <= 2 && kFwdStages <= 2, "descriptor selection assumes at most two of each");
      const SmemDesc dq0 = smem_desc_sw128_split(smem_u32(sm.q[0]), 16, 1024);
      const SmemDesc dq1 = smem_desc_sw128_split(smem_u32(sm.q[kFwdQT - 1]), 16, 1024);
      const SmemDesc dk0 = smem_desc_sw128_split(smem_u32(sm.k[0]), 16, 1024);
      const SmemDesc dk1 = smem_desc_sw128_split(smem_u32(sm.k[kFwdStages - 1]), 16, 1024);
      const SmemDesc dv0 = smem_desc_sw128_split(smem_u32(sm.v[0]), kSlab, 1024);
      const SmemDesc dv1 = smem_desc_sw128_split(smem_u32(sm.v[kFwdStages - 1]), kSlab, 1024);
      auto issue_qk = [&](int t, int s) {
        const SmemDesc a = t ? dq1 : dq0, bk = s ? dk1 : dk0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kSlab + (kk & 3) * 32) >> 4;
          if (kk == 0)
            tc_mma_ss_c<0>(tmem + t * kFwdBN, a.lo + off, a.hi, bk.lo + off, bk.hi, idesc_qk);
          else
            tc_mma_ss_c<1>(tmem + t * kFwdBN, a.lo + off, a.hi, bk.lo + off, bk.hi, idesc_qk);
        }
      };
      // half h covers keys 64h .. 64h + 63 (P columns 32h .. 32h + 31)
      auto issue_pv = [&](int t, int s, bool acc, int h) {
        const SmemDesc bv = s ? dv1 : dv0;
#pragma unroll
        for (int kk = h * 4; kk < h * 4 + 4; ++kk) {
          const uint32_t off = (kk * 16 * 128) >> 4;
          if (kk == 0 && !acc)
            tc_mma_ts_c<0>(tmem + kOCol + t * D, tmem + t * kFwdBN + kk * 8, bv.lo + off, bv.hi, idesc_pv);
          else
            tc_mma_ts_c<1>(tmem + kOCol + t * D, tmem + t * kFwdBN + kk * 8, bv.lo + off, bv.hi, idesc_pv);
        }
      };
      // Debug flag bit 2 (failure-detection tests): issue no MMA at all, so the softmax warps'
      // first wait for S runs out; the bounded waits then take the abort path below.
      const bool withhold = (p.flags & 4) != 0;
      bool ok = !withhold && mbar_wait(smem_u32(&sm.bar_q), 0, abort, 901);
      // Q tile t takes part in visited tile u only where its bit is on; its MMAs are skipped
      // elsewhere and its barriers count only the tiles it takes part in. The bits of tile j + 1
      // are taken at the top of iteration j, ahead of the waits, and carried into iteration j + 1
      // (a shared load after a wait would sit on the issue path).
      // (Dense: the runs [jlo_t, jhi_t) give the same answers in closed form.)
      uint32_t bits_cur = SPARSE ? sm.act_bits[0] : 0u, bits_next = 0u;
      int j = 0;
      auto act_cur = [&](int t) -> bool {  // Q tile t takes part in tile j
        if (t >= kFwdQT) return false;
        if constexpr (!kPart) return true;
        else if constexpr (SPARSE) return ((bits_cur >> t) & 1u) != 0;
        else return t ? (j >= jlo1 && j < jhi1) : (j >= jlo0 && j < jhi0);
      };
      auto act_next = [&](int t) -> bool {  // ... in tile j + 1
        if (t >= kFwdQT) return false;
        if constexpr (!kPart) return true;
        else if constexpr (SPARSE) return ((bits_next >> t) & 1u) != 0;
        else return t ? (j + 1 >= jlo1 && j + 1 < jhi1) : (j + 1 >= jlo0 && j + 1 < jhi0);
      };
      int npv0 = 0, npv1 = 0;  // PV groups issued so far per Q tile (block-sparse)
      // PV groups of Q tile t issued before tile j (dense: closed form; block-sparse: the count,
      // read before this tile's PV adds to it)
      auto pv_before = [&](int t) -> int {
        if constexpr (!kPart) return j;
        else if constexpr (SPARSE) return t ? npv1 : npv0;
        else return t ? max(0, min(j, jhi1) - jlo1) : max(0, min(j, jhi0) - jlo0);
      };
      // ... issued up to and including tile j (block-sparse: read after this tile's PV)
      auto pv_through = [&](int t) -> int {
        if constexpr (!kPart) return j + 1;
        else if constexpr (SPARSE) return t ? npv1 : npv0;
        else return t ? max(0, min(j + 1, jhi1) - jlo1) : max(0, min(j + 1, jhi0) - jlo0);
      };
      for (; ok && j < n_act; ++j) {  // j counts visited tiles
        const int s = j % kFwdStages;
        const uint32_t ph = (j / kFwdStages) & 1;
        const int s1 = (j + 1) % kFwdStages;
        const uint32_t ph1 = ((j + 1) / kFwdStages) & 1;
        const bool more = j + 1 < n_act;
        if constexpr (SPARSE) {
          if (j > 0) bits_cur = bits_next;
          bits_next = more ? sm.act_bits[j + 1] : 0u;
        }
        if (j == 0) {
          if (!(ok = mbar_wait(smem_u32(&sm.bar_k_full[s]), ph, abort, 902))) break;
          tc_fence_after();
          if (act_cur(0)) {
            issue_qk(0, s);
            tc_commit(smem_u32(&sm.bar_s_full[0]));
          }
          if (act_cur(1)) {
            issue_qk(1, s);
            tc_commit(smem_u32(&sm.bar_s_full[1]));
          }
          tc_commit(smem_u32(&sm.bar_k_empty[s]));
        }
        // Q tile 0: PV(j), then QK(j+1) once PV(j) is done (P_0 lives in S_0's columns)
        if (!(ok = mbar_wait(smem_u32(&sm.bar_v_full[s]), ph, abort, 903))) break;
        if (act_cur(0)) {
          const int c = pv_before(0);
          if (!(ok = mbar_wait(smem_u32(&sm.bar_p_full[0][0]), c & 1, abort, 904))) break;
          tc_fence_after();
          issue_pv(0, s, c > 0, 0);
          if (!(ok = mbar_wait(smem_u32(&sm.bar_p_full[0][1]), c & 1, abort, 914))) break;
          tc_fence_after();
          issue_pv(0, s, true, 1);
          tc_commit(smem_u32(&sm.bar_o_done[0]));
          ++npv0;
        }
        if (more) {
          if (!(ok = mbar_wait(smem_u32(&sm.bar_k_full[s1]), ph1, abort, 905))) break;
          if (act_next(0)) {
            // the latest PV of Q tile 0 read P_0 from S_0's columns
            const int n_pv = pv_through(0);
            if (n_pv > 0)
              if (!(ok = mbar_wait(smem_u32(&sm.bar_o_done[0]), (n_pv - 1) & 1, abort, 906))) break;
            tc_fence_after();
            issue_qk(0, s1);
            tc_commit(smem_u32(&sm.bar_s_full[0]));
          }
        }
        // Q tile 1
        if (act_cur(1)) {
          const int c = pv_before(1);
          if (!(ok = mbar_wait(smem_u32(&sm.bar_p_full[1][0]), c & 1, abort, 907))) break;
          tc_fence_after();
          issue_pv(1, s, c > 0, 0);
          if (!(ok = mbar_wait(smem_u32(&sm.bar_p_full[1][1]), c & 1, abort, 917))) break;
          tc_fence_after();
          issue_pv(1, s, true, 1);
          tc_commit(smem_u32(&sm.bar_o_done[1]));
          ++npv1;
        }
        tc_commit(smem_u32(&sm.bar_v_empty[s]));
        if (more) {
          if (act_next(1)) {
            const int n_pv = pv_through(1);
            if (n_pv > 0)
              if (!(ok = mbar_wait(smem_u32(&sm.bar_o_done[1]), (n_pv - 1) & 1, abort, 908))) break;
            tc_fence_after();
            issue_qk(1, s1);
            tc_commit(smem_u32(&sm.bar_s_full[1]));
          }
          tc_commit(smem_u32(&sm.bar_k_empty[s1]));
        }
      }
      // Drain: every MMA issued above has completed before TMEM is released.
      tc_commit(smem_u32(&sm.bar_final));
      volatile int no_abort = 0;
      mbar_wait(smem_u32(&sm.bar_final), 0, &no_abort, 909);
    }
   }
  } else {
    regs_inc<FwdShape<ONE>::kRegsSoftmax>();
    // ================================================================ softmax warps
    const int t = warp >> 2;                  // Q tile of this warpgroup
    const int quarter = warp & 3;             // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;        // row within the Q tile
    const int row = q0 + t * kFwdBM + r;      // query row
    const int a = row + off;                  // absolute position of the row
    const int a_lo = q0 + t * kFwdBM + off;   // first / last absolute position of the Q tile
    const int a_hi = a_lo + kFwdBM - 1;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_base + t * kFwdBN;
    const uint32_t t_o = tmem + lane_base + kOCol + t * D;
    const float c = p.c_log2;
    float m_run = -INFINITY;  // running max of the stored (scaled, capped) score
    float l_run = 0.f;

    // block-sparse: every visited tile, skipping those without this Q tile's bit; dense: the
    // contiguous run of tiles this Q tile takes part in
    const int j_first = kRuns ? (t ? jlo1 : jlo0) : 0;
    const int j_end = kRuns ? (t ? jhi1 : jhi0) : n_act;
    int nt = 0;  // tiles this Q tile took part in
    for (int j = j_first; j < j_end; ++j) {  // j counts visited tiles
      const uint32_t bj = bits_of(j);
      if (SPARSE && !((bj >> t) & 1u)) continue;  // not this Q tile's: no S, no P for it
      const int c_t = kPart ? nt : j;
      const bool got = mbar_wait(smem_u32(&sm.bar_s_full[t]), c_t & 1, abort, 1001 + t);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      uint32_t sraw[128];
      tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]));
      tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]));
      tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&sraw[64]));
      tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&sraw[96]));
      tmem_wait_ld(sraw);
      float* s = reinterpret_cast<float*>(sraw);

      const int k0 = (kt_lo + tile_of(j)) * kFwdBN;
      // Softcap: the capped score is cap * tanh(s * scale / cap); the value kept per key is that
      // divided by scale, so the exponent factor c = scale * log2 e is the same as without a cap.
      // When every |y| = |s| * scale / cap of this warp's rows is small, tanh(y) = y * q(y^2) is
      // evaluated inside the exponential loop below (FMA work that fills the issue slots left
      // while MUFU computes exponentials), and the row max is taken on the raw scores: tanh is
      // increasing, so the kept max is the transform of the raw max. Otherwise every score is
      // transformed here with tanh from exp2.
      bool poly = false;
      if (SOFTCAP && p.softcap > 0.f) {  // (the capped build keeps the run-time test: measured faster)
        float am8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) am8[i] = fmaxf(fabsf(s[i]), fabsf(s[i + 8]));
#pragma unroll
        for (int i = 16; i < 128; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) am8[k] = max3(am8[k], fabsf(s[i + k]), fabsf(s[i + 8 + k]));
        const float amax = max3(max3(am8[0], am8[1], am8[2]), max3(am8[3], am8[4], am8[5]),
                                fmaxf(am8[6], am8[7]));
        poly = __all_sync(0xffffffffu, amax * p.cap_in <= kTanhPolyMax);
        if (!poly) {
#pragma unroll
          for (int i = 0; i < 128; ++i) s[i] = p.cap_out * tanh_from_exp(s[i] * p.cap_in);
        }
      }
      // Element masks only where some row of this Q tile may not see some key of the tile.
      bool interior = (k0 + kFwdBN <= Nk);
      if (p.causal) interior = interior && (k0 + kFwdBN - 1 <= a_lo);
      if (p.win_r >= 0) interior = interior && (k0 + kFwdBN - 1 <= a_lo + p.win_r);
      if (p.win_l >= 0) interior = interior && (k0 >= a_hi - p.win_l);
      if (p.flags & 1) interior = false;
      if (!interior) {
        int jhi = Nk - k0;                                     // keys >= Nk
        if (p.causal) jhi = min(jhi, a - k0 + 1);
        if (p.win_r >= 0) jhi = min(jhi, a + p.win_r - k0 + 1);
        const int jlo = (p.win_l >= 0) ? (a - p.win_l - k0) : -1;
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = (i < jhi && i >= jlo) ? s[i] : -INFINITY;
      }
      // row max: 8 chains of 3-input max
      auto row_max = [&]() -> float {
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(s[i], s[i + 8]);
#pragma unroll
        for (int i = 16; i < 128; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = max3(m8[k], s[i + k], s[i + 8 + k]);
        float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        if (poly && mx > -INFINITY) {
          const float y = mx * p.cap_in;
          mx = p.cap_out * (y * tanh_q(y * y));
        }
        return mx;
      };
      // Lazy rescale: move the reference max only when it grew by more than 2^8 in exp2 terms.
      // Returns whether any row of the warp moves it (then alpha and m_run are updated).
      float alpha = 1.f;
      auto rescale_decision = [&](float mx) -> bool {
        const float m_new = fmaxf(m_run, mx);
        const bool need = (m_new > -INFINITY) && (m_run == -INFINITY || (m_new - m_run) * c > kRescaleLog2);
        const bool warp_rescale = __any_sync(0xffffffffu, need);
        if (warp_rescale) {
          if (m_new > m_run) {
            alpha = (m_run == -INFINITY) ? 0.f : fast_exp2((m_run - m_new) * c);
            m_run = m_new;
          }
        }
        return warp_rescale;
      };
      // O rescale before any PV of this tile reads P (only after the first tile: before it O
      // holds nothing). The previous PV of this Q tile has completed: its commit preceded S.
      auto rescale_o = [&]() {
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t o[32];
          tmem_ld32(t_o + cb, o);
          tmem_wait_ld(o);
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float lo, hi;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), a2), lo, hi);
            o[2 * i] = __float_as_uint(lo);
            o[2 * i + 1] = __float_as_uint(hi);
          }
          tmem_st32(t_o + cb, o);
        }
      };
      if constexpr (PAGED) {
        // the final tile: value rows at or past the length (inside the last page) become 0, by
        // the first Q tile taking part in it (each PV of the tile comes after that one's P)
        if (t == ((bj & 1u) ? 0 : 1) && k0 + kFwdBN > Nk) {
          const int vs = j % kFwdStages;
          const bool vok = mbar_wait(smem_u32(&sm.bar_v_full[vs]), (j / kFwdStages) & 1, abort, 1009);
          if (!__all_sync(0xffffffffu, vok)) break;
          if (r >= Nk - k0) {
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int sl = 0; sl < kSlabs; ++sl) {
              uint4* rowp = reinterpret_cast<uint4*>(sm.v[vs] + sl * kSlab + r * 128);
#pragma unroll
              for (int c16 = 0; c16 < 8; ++c16) rowp[c16] = z;
            }
          }
          fence_proxy_async_smem();  // generic stores, then the tensor core reads them after P
        }
      }
      // P = exp2(s * c - m * c) on fp32 pairs, packed to the input type and stored to TMEM 16
      // columns at a time (32 keys per chunk); a half of P (chunks 0-1, 2-3) is announced once it
      // is stored, when announcements are on.
      const uint64_t c2 = f2_pack(c, c);
      uint64_t acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = f2_pack(0.f, 0.f);
      auto announce = [&](int half) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.bar_p_full[t][half]));
      };
      // POLY: the kept value of a pair is tanh(y) * cap / scale with y = s * scale / cap, so
      // x = tanh(y) * (cap log2 e) - m c; a masked score (-inf) gives y = -inf, q = +inf and
      // x = -inf (the polynomial's leading coefficient is positive).
      auto exponentials = [&](auto poly_tag, auto ch_lo_tag, auto ch_hi_tag, bool announce_halves,
                              float neg_mc) {
        constexpr bool kPoly = decltype(poly_tag)::value;
        constexpr int kChLo = decltype(ch_lo_tag)::value, kChHi = decltype(ch_hi_tag)::value;
        const uint64_t ci2 = f2_pack(p.cap_in, p.cap_in);
        const float cc = p.softcap * 1.4426950408889634f;
        const uint64_t xc2 = kPoly ? f2_pack(cc, cc) : c2;
        const uint64_t nm2 = f2_pack(neg_mc, neg_mc);
#pragma unroll
        for (int ch = kChLo; ch < kChHi; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int ii = ch * 16 + i;
            uint64_t v = f2_pack(s[2 * ii], s[2 * ii + 1]);
            if constexpr (kPoly) {
              const uint64_t y = f2_mul(v, ci2);
              v = f2_mul(y, tanh_q2(f2_mul(y, y)));
            }
            const uint64_t x = f2_fma(v, xc2, nm2);
            uint64_t pp;
            if (kPolyPair(ii)) {
              pp = exp2_fma2(x);
            } else {
              float x0, x1;
              f2_unpack(x, x0, x1);
              pp = f2_pack(fast_exp2(x0), fast_exp2(x1));
            }
            acc[ii & 3] = f2_add(acc[ii & 3], pp);
            float p0, p1;
            f2_unpack(pp, p0, p1);
            pk[i] = pack2<BF16>(p0, p1);
          }
          tmem_st16(t_s + ch * 16, pk);
          if ((ch & 1) && announce_halves) announce(ch >> 1);
        }
      };
      using I0 = std::integral_constant<int, 0>;
      using I2 = std::integral_constant<int, 2>;
      using I4 = std::integral_constant<int, 4>;
      using PolyOff = std::integral_constant<bool, false>;
      using PolyOn = std::integral_constant<bool, true>;
      const float neg_mc_old = (m_run == -INFINITY) ? 0.f : -m_run * c;
      if (ONE && !SOFTCAP && c_t > 0) {
        // After the first tile the reference max rarely moves: compute the first half of P
        // with the current one while the row max of the whole tile is taken alongside, and
        // announce it unless some row of the warp moves the max, in which case the tile is
        // redone exactly as the ordinary path below does it (nothing of it was announced).
        // Bitwise the same results as the ordinary path. (Measured on the single-Q-tile shape:
        // causal N = 4096 6 %, windows 3-6 % faster; on the two-Q-tile shape it changed nothing
        // beyond noise.)
        exponentials(PolyOff(), I0(), I2(), false, neg_mc_old);
        const float mx = row_max();
        if (!rescale_decision(mx)) {
          announce(0);
          exponentials(PolyOff(), I2(), I4(), true, neg_mc_old);
        } else {
          rescale_o();
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = f2_pack(0.f, 0.f);
          exponentials(PolyOff(), I0(), I4(), true, (m_run == -INFINITY) ? 0.f : -m_run * c);
        }
      } else {
        const float mx = row_max();
        const bool warp_rescale = rescale_decision(mx);
        if (warp_rescale && c_t > 0) rescale_o();
        const float neg_mc = (m_run == -INFINITY) ? 0.f : -m_run * c;
        if (SOFTCAP && poly)
          exponentials(PolyOn(), I0(), I4(), true, neg_mc);
        else
          exponentials(PolyOff(), I0(), I4(), true, neg_mc);
      }
      float sa, sb;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), sa, sb);
      l_run = l_run * alpha + (sa + sb);
      ++nt;
    }

    // ---- epilogue: O / l, LSE
    bool have_o = false;
    const int n_t = kPart ? nt : n_act;  // PV groups of this Q tile
    if (n_t > 0 && !*abort) {
      have_o = mbar_wait(smem_u32(&sm.bar_o_done[t]), (n_t - 1) & 1, abort, 1003 + t);
      tc_fence_after();
    }
    have_o = __all_sync(0xffffffffu, have_o);
    {
    }
    const bool valid = row < Nq;
    const size_t orow = VARLEN ? (size_t)(rq + row) * p.Hq + h : (size_t)(b * p.Hq + h) * Nq + row;
    const size_t obase = orow * D;
    const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
    // The normalised tile goes to the Q tile's own buffer (free: its last QK completed before its
    // last scores were read) in the 128-byte-swizzled layout of the output tensor map, and one
    // thread writes it with TMA stores: whole 128-byte lines instead of a 16-byte piece of 32
    // rows per store instruction. Dense rows past Nq fall outside the map and are not written;
    // a packed tile that runs past its sequence's end is stored row by row instead.
    const bool tma_out = !VARLEN || (q0 + t * kFwdBM + kFwdBM <= Nq);
    const uint32_t stage = smem_u32(sm.q[t]);
    if (tma_out && q_early && n_t == 0) {
      // A Q tile that took part in no key tile never waited for S, so the Q load into the
      // buffer about to be overwritten may still be landing: wait for it first.
      volatile int no_abort = 0;
      mbar_wait(smem_u32(&sm.bar_q), 0, &no_abort, 1010);
    }
#pragma unroll
    for (int cb = 0; cb < D; cb += 32) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld32(t_o + cb, o);
        tmem_wait_ld(o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      uint4 w[4];
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        w[v4].x = pack2<BF16>(__uint_as_float(o[v4 * 8 + 0]) * inv_l, __uint_as_float(o[v4 * 8 + 1]) * inv_l);
        w[v4].y = pack2<BF16>(__uint_as_float(o[v4 * 8 + 2]) * inv_l, __uint_as_float(o[v4 * 8 + 3]) * inv_l);
        w[v4].z = pack2<BF16>(__uint_as_float(o[v4 * 8 + 4]) * inv_l, __uint_as_float(o[v4 * 8 + 5]) * inv_l);
        w[v4].w = pack2<BF16>(__uint_as_float(o[v4 * 8 + 6]) * inv_l, __uint_as_float(o[v4 * 8 + 7]) * inv_l);
      }
      if (tma_out) {
        // 16-byte chunk ch of row r in a slab sits at r * 128 + (ch ^ (r % 8)) * 16
        const uint32_t slab = stage + (cb / 64) * kSlab + r * 128;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const int ch = (cb % 64) / 8 + v4;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(slab + ((ch ^ (r & 7)) << 4)),
                       "r"(w[v4].x), "r"(w[v4].y), "r"(w[v4].z), "r"(w[v4].w)
                       : "memory");
        }
      } else if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + obase + cb);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) dst[v4] = w[v4];
      }
    }
    if (tma_out) {
      fence_proxy_async_smem();  // the staged tile, then the TMA engine reads it
      if (t == 0) named_bar_sync<1, kFwdBM>(); else named_bar_sync<2, kFwdBM>();
      if (r == 0) {
        for (int sl = 0; sl < kSlabs; ++sl) {
          if constexpr (VARLEN)
            tma_store_3d(&p.tm_o, stage + sl * kSlab, sl * 64, h, rq + q0 + t * kFwdBM);
          else
            tma_store_3d(&p.tm_o, stage + sl * kSlab, sl * 64, q0 + t * kFwdBM, b * p.Hq + h);
        }
        bulk_commit_group();
        bulk_wait_group_all();  // the staging buffer is read and the rows written before exit
      }
    }
    if (valid && p.lse != nullptr) {
      p.lse[VARLEN ? (size_t)h * p.total_q + rq + row : (size_t)(b * p.Hq + h) * Nq + row] =
          (l_run > 0.f) ? (m_run * c + log2f(l_run)) * p.lse_mul : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, FwdShape<ONE>::kTmemCols);
  }
}

// Nk == 0: every row sees no key.
template <bool BF16>
__global__ void mfa_fill_empty_kernel(void* out, float* lse, size_t rows, int D) {
  const size_t n = rows * (size_t)D;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    reinterpret_cast<uint16_t*>(out)[i] = 0;
  if (lse)
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < rows; i += (size_t)gridDim.x * blockDim.x)
      lse[i] = -INFINITY;
}

}  // namespace mfa
