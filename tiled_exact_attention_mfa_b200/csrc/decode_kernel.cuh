// decode_kernel.cuh -- two-phase split-KV decode over a paged KV cache (N_q <= 4).
//
// Source: "mlx-mfa 2.5.2" Features (Flash Decode: two-phase split-KV for N_q <= 4; paged KV
// with block_table) and "mxflashattn 1.4.0 -> 1.5.0" README (split-KV paged decode with page
// size 16, per-split (m, l) slots merged afterwards; a padded-row guard that once wrote into the
// neighbouring slot -- here every partial write is guarded by row < G * N_q).
//
// Phase 1 (one CTA per (split, sequence, group of kv heads)):
//   * a producer warp copies, page by page, the token rows of the CTA's kv heads from the
//     K and V pools into a 3-stage shared-memory ring with 1-D bulk copies (one per token row,
//     Hg * D * 2 contiguous bytes, padded by 16 bytes so that ldmatrix reads are conflict free).
//     Only tokens below the sequence length are copied; block_table entries are bounds-checked.
//   * one compute warp per kv head: its G * N_q query rows (<= 16) form one m16 MMA tile; per
//     16-token page it computes S = Q K^T with mma.sync m16n8k16 (fp32 accumulate), masks tokens
//     past the length and (causal) past the query's own position, runs the online softmax in
//     fp32 (row max / sum over the quad of lanes holding a row), rounds P to the input type and
//     accumulates O += P V with mma.sync. Value rows of tokens past the length are zeroed in
//     registers, so NaN in unused page slots never reaches the arithmetic.
//   * it writes unnormalised O, the running max (log2 domain) and the running sum per row.
//   * with a left window (local-attention layers, "mlx-mfa 2.5.2" Features, window_size) the
//     splits of a sequence start at the first page some query token can see, and tokens left of
//     a row's window are masked like those past its causal limit.
// Phase 2 (combine): per (sequence, query head, query token): M = max_s m_s,
//   O = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, LSE = ln 2 * (M + log2 sum_s 2^(m_s-M) l_s).
#pragma once
#include "sm100.cuh"

namespace mfa {

constexpr int kDecPage = 16;
constexpr int kDecMaxSplitPages = 64;  // pages per phase-1 split at most (two table entries per lane)
constexpr int kDecStages = 3;

struct DecodeParams {
  const uint16_t* q;
  const uint16_t* k_pages;
  const uint16_t* v_pages;
  const int32_t* block_table;
  const int32_t* seq_lens;
  void* out;
  float* lse;
  // partial results, split-major so that a range of splits is one contiguous block (the unit a
  // GPU contributes when the splits of a sequence are spread over GPUs):
  float* ws_o;    // [splits][B][Hq*Nq][D]  unnormalised O
  float* ws_ml;   // [splits][B][Hq*Nq][2]  (m in log2 units, l)
  int B, Nq, Hq, Hkv, G, max_pages, num_pages;
  int pages_per_split, max_splits, heads_per_cta;
  int split_lo;   // phase 1 computes splits split_lo + blockIdx.x
  int causal;
  int win_l;      // left window (query at position a sees keys >= a - win_l); -1: none
  float c_log2;   // scale * log2 e (no softcap) or log2 e (softcap)
  float softcap, cap_in;
};

// Sequence length clamped to [0, max_pages * 16]; an entry outside that range is reported.
__device__ __forceinline__ int checked_len(const DecodeParams& p, int b, bool report) {
  const int len = p.seq_lens[b];
  const int cap = p.max_pages * kDecPage;
  if (len < 0 || len > cap) {
    if (report) record_status(-22, 0x40000000 + b);
    return len < 0 ? 0 : cap;
  }
  return len;
}

// First page holding a key that some query token of the sequence can see: with a left window,
// tokens before len - Nq - win_l are invisible to every query token. Splits are counted from this
// page, so pages wholly left of the window are neither read nor given a split.
__device__ __forceinline__ int dec_first_page(const DecodeParams& p, int len) {
  if (p.win_l < 0) return 0;
  // 64-bit: a window near INT_MAX over a sequence shorter than Nq must not wrap around
  const long long first = (long long)len - p.Nq - p.win_l;
  return first > 0 ? (int)(first / kDecPage) : 0;
}

// kv heads per phase-1 CTA at most: a token row of all of them fits in 1 KB
template <int D>
constexpr int kDecMaxHeads = 1024 / (2 * D);

template <int D>
__host__ __device__ constexpr int dec_row_bytes(int hg) {
  return hg * D * 2 + 16;
}
template <int D>
__host__ __device__ constexpr int dec_smem_bytes(int hg) {
  // per stage: K and V, 16 token rows each; + barriers
  return kDecStages * 2 * kDecPage * dec_row_bytes<D>(hg) + 2 * kDecStages * 8 + 64;
}

template <int D, bool BF16>
__global__ void __launch_bounds__((kDecMaxHeads<D> + 1) * 32) mfa_decode_phase1_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int hg = p.heads_per_cta;
  const int row_bytes = dec_row_bytes<D>(hg);
  const int stage_bytes = 2 * kDecPage * row_bytes;
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + kDecStages * stage_bytes);
  uint64_t* bar_empty = bar_full + kDecStages;
  int* abort_flag = reinterpret_cast<int*>(bar_empty + kDecStages);

  // every CTA of this grid is resident (or done) once all have passed here, so the combine grid
  // may be launched now; it waits for this grid's completion before reading the workspace
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int split = p.split_lo + blockIdx.x;
  const int b = blockIdx.y;
  const int h0 = blockIdx.z * hg;  // first kv head of this CTA
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int len = checked_len(p, b, split == 0 && blockIdx.z == 0 && threadIdx.x == 0);
  const int n_pages = (len + kDecPage - 1) / kDecPage;
  const int pg0 = dec_first_page(p, len) + split * p.pages_per_split;
  if (pg0 >= n_pages) return;  // nothing of this sequence falls in this split
  const int pg1 = min(n_pages, pg0 + p.pages_per_split);
  const int np = pg1 - pg0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), hg);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = abort_flag;

  if (warp == hg) {
    // ====================================================== producer warp
    // block_table entries of this split, two per lane (pages_per_split <= kDecMaxSplitPages)
    int page_lo = -1, page_hi = -1;  // entries pg0 + lane and pg0 + 32 + lane
    if (lane < np) page_lo = p.block_table[(size_t)b * p.max_pages + pg0 + lane];
    if (32 + lane < np) page_hi = p.block_table[(size_t)b * p.max_pages + pg0 + 32 + lane];
    if (lane < np && (page_lo < 0 || page_lo >= p.num_pages)) record_status(-22, b * 65536 + pg0 + lane);
    if (32 + lane < np && (page_hi < 0 || page_hi >= p.num_pages))
      record_status(-22, b * 65536 + pg0 + 32 + lane);
    int issued[kDecStages] = {0, 0, 0};
    for (int i = 0; i < np; ++i) {
      const int s = i % kDecStages;
      const int use = i / kDecStages;
      const int pid = __shfl_sync(0xffffffffu, i < 32 ? page_lo : page_hi, i & 31);
      const bool pid_ok = pid >= 0 && pid < p.num_pages;
      const int valid = min(kDecPage, len - (pg0 + i) * kDecPage);
      bool ok = true;
      if (lane == 0 && use > 0) ok = mbar_wait(smem_u32(&bar_empty[s]), (use - 1) & 1, abort, 1101);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const uint32_t kdst = smem_u32(smem + s * stage_bytes);
      const uint32_t vdst = kdst + kDecPage * row_bytes;
      const uint32_t bar = smem_u32(&bar_full[s]);
      const uint32_t chunk = (uint32_t)(hg * D * 2);
      if (lane == 0) mbar_expect_tx(bar, pid_ok ? 2u * chunk * (uint32_t)valid : 0u);
      __syncwarp();
      if (pid_ok && lane < valid) {
        const size_t src = (((size_t)pid * kDecPage + lane) * p.Hkv + h0) * D;
        // K / V are read once: evict them first, so the partials written below stay in L2
        // for the combine
        const uint64_t pol = l2_policy_evict_first();
        bulk_load_hint(kdst + lane * row_bytes, p.k_pages + src, chunk, bar, pol);
        bulk_load_hint(vdst + lane * row_bytes, p.v_pages + src, chunk, bar, pol);
      }
      issued[s] = use + 1;
    }
    if (lane == 0) {
      volatile int no_abort = 0;
      for (int s = 0; s < kDecStages; ++s)
        if (issued[s] > 0) mbar_wait(smem_u32(&bar_full[s]), (issued[s] - 1) & 1, &no_abort, 1102);
    }
    return;
  }
  if (warp > hg) return;

  // ====================================================== compute warp: kv head h0 + warp
  const int kvh = h0 + warp;
  const int R = p.G * p.Nq;       // query rows of this kv head (<= 16)
  const int qr = lane >> 2;       // fragment row (and qr + 8)
  const int qc = (lane & 3) * 2;  // fragment column pair
  const float c = p.c_log2;

  // Q fragments (A operand, rows r = hl * Nq + t), kept for the whole split.
  uint32_t qa[D / 16][4];
  {
    auto qval = [&](int r, int d) -> uint32_t {
      if (r >= R) return 0u;
      const int hl = r / p.Nq, t = r % p.Nq;
      const size_t off = (((size_t)b * p.Hq + (size_t)kvh * p.G + hl) * p.Nq + t) * D + d;
      return *reinterpret_cast<const uint32_t*>(p.q + off);
    };
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qa[kk][0] = qval(qr, kk * 16 + qc);
      qa[kk][1] = qval(qr + 8, kk * 16 + qc);
      qa[kk][2] = qval(qr, kk * 16 + 8 + qc);
      qa[kk][3] = qval(qr + 8, kk * 16 + 8 + qc);
    }
  }
  // visible tokens [low, lim] of this thread's two rows: causal limit, left window, length
  int lim[2], low[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = qr + 8 * e;
    const int t = (r < R) ? (r % p.Nq) : 0;
    lim[e] = p.causal ? (len - p.Nq + t) : (len - 1);
    lim[e] = min(lim[e], len - 1);
    low[e] = (p.win_l >= 0) ? (int)max(-1ll, (long long)len - p.Nq + t - p.win_l) : 0;
  }

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  // ldmatrix row addresses (per lane) inside a stage
  const uint32_t head_off = (uint32_t)(warp * D * 2);
  const int k_tok = ((lane >> 4) << 3) + (lane & 7);   // K: matrices (t0-7,d0) (t0-7,d8) (t8-15,d0) (t8-15,d8)
  const int k_dof = ((lane >> 3) & 1) * 8;
  const int v_tok = (((lane >> 3) & 1) << 3) + (lane & 7);  // V: (t0-7,d0) (t8-15,d0) (t0-7,d8) (t8-15,d8)
  const int v_dof = (lane >> 4) * 8;
  const int row_bytes_c = row_bytes;

  for (int i = 0; i < np; ++i) {
    const int s = i % kDecStages;
    bool ok = mbar_wait(smem_u32(&bar_full[s]), (i / kDecStages) & 1, abort, 1201);
    if (!__all_sync(0xffffffffu, ok)) break;
    const uint32_t kbase = smem_u32(smem + s * stage_bytes) + head_off;
    const uint32_t vbase = kbase + kDecPage * row_bytes_c;
    const int tok0 = (pg0 + i) * kDecPage;
    const int valid = min(kDecPage, len - tok0);

    // ---- S = Q K^T : 16 rows x 16 tokens (two n8 tiles)
    float sc[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kbase + k_tok * row_bytes_c + (kk * 16 + k_dof) * 2, b0, b1, b2, b3);
      mma_16816<BF16>(sc[0], qa[kk], b0, b1);
      mma_16816<BF16>(sc[1], qa[kk], b2, b3);
    }
    // ---- scale / softcap / mask, row max
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tok0 + n * 8 + qc + (e & 1);
        const int ri = e >> 1;
        float x = sc[n][e];
        if (p.softcap > 0.f) x = p.softcap * tanh_from_exp(x * p.cap_in);
        x = (tok <= lim[ri] && tok >= low[ri]) ? x : -INFINITY;
        sc[n][e] = x;
        mx[ri] = fmaxf(mx[ri], x);
      }
    float alpha[2], neg_mc[2];
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      mx[ri] = fmaxf(mx[ri], __shfl_xor_sync(0xffffffffu, mx[ri], 1));
      mx[ri] = fmaxf(mx[ri], __shfl_xor_sync(0xffffffffu, mx[ri], 2));
      const float m_new = fmaxf(m_run[ri], mx[ri]);
      alpha[ri] = (m_new == -INFINITY || m_run[ri] == -INFINITY) ? (m_run[ri] == -INFINITY ? 0.f : 1.f)
                                                                  : fast_exp2((m_run[ri] - m_new) * c);
      m_run[ri] = m_new;
      neg_mc[ri] = (m_new == -INFINITY) ? 0.f : -m_new * c;
    }
    float sum[2] = {0.f, 0.f};
    uint32_t pa[4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const float p0 = fast_exp2(fmaf(sc[n][0], c, neg_mc[0]));
      const float p1 = fast_exp2(fmaf(sc[n][1], c, neg_mc[0]));
      const float p2 = fast_exp2(fmaf(sc[n][2], c, neg_mc[1]));
      const float p3 = fast_exp2(fmaf(sc[n][3], c, neg_mc[1]));
      sum[0] += p0 + p1;
      sum[1] += p2 + p3;
      pa[2 * n + 0] = pack2<BF16>(p0, p1);   // row qr,   tokens n*8 + qc..
      pa[2 * n + 1] = pack2<BF16>(p2, p3);   // row qr+8
    }
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      sum[ri] += __shfl_xor_sync(0xffffffffu, sum[ri], 1);
      sum[ri] += __shfl_xor_sync(0xffffffffu, sum[ri], 2);
      l_run[ri] = l_run[ri] * alpha[ri] + sum[ri];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // ---- O += P V : A = P (16 x 16 tokens), B = V (16 tokens x 8 d) per n tile
    const uint32_t a_frag[4] = {pa[0], pa[1], pa[2], pa[3]};
    // token indices held by this lane in a B fragment: qc, qc+1 (b0) and qc+8, qc+9 (b1)
    const bool tail = valid < kDecPage;
    const uint32_t keep0 = (qc < valid ? 0x0000FFFFu : 0u) | (qc + 1 < valid ? 0xFFFF0000u : 0u);
    const uint32_t keep1 = (qc + 8 < valid ? 0x0000FFFFu : 0u) | (qc + 9 < valid ? 0xFFFF0000u : 0u);
#pragma unroll
    for (int nn = 0; nn < D / 16; ++nn) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vbase + v_tok * row_bytes_c + (nn * 16 + v_dof) * 2, b0, b1, b2, b3);
      if (tail) {
        b0 &= keep0;
        b1 &= keep1;
        b2 &= keep0;
        b3 &= keep1;
      }
      mma_16816<BF16>(o[2 * nn], a_frag, b0, b1);
      mma_16816<BF16>(o[2 * nn + 1], a_frag, b2, b3);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bar_empty[s]));
  }

  // ---- partial results (rows < R only)
  const size_t rows_all = (size_t)p.Hq * p.Nq;
  const size_t slot = ((size_t)split * p.B + b) * rows_all;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = qr + 8 * e;
    if (r >= R) continue;
    const size_t row = (size_t)kvh * p.G * p.Nq + r;  // = (kvh*G + hl) * Nq + t
    float* dst = p.ws_o + (slot + row) * D;
    // the combine reads these back soon: keep them in L2 ahead of the streamed K / V lines
    const uint64_t pol = l2_policy_evict_last();
#pragma unroll
    for (int n = 0; n < D / 8; ++n) st_global_f2_hint(dst + n * 8 + qc, o[n][2 * e], o[n][2 * e + 1], pol);
    if ((lane & 3) == 0)
      st_global_f2_hint(p.ws_ml + (slot + row) * 2, m_run[e] == -INFINITY ? -INFINITY : m_run[e] * c,
                        l_run[e], pol);
  }
}

// Threads per combine CTA. Each thread owns 4 consecutive output columns (one 16-byte load per
// split), so a group of D / 4 threads covers a row and there are G = 4 * kCombineThreads / D
// groups; group g takes splits g, g + G, g + 2G, ... At 256 threads two CTAs share an SM, so one
// CTA's merge and store overlap the other's loads (with 512 threads, one CTA per SM, the SM had
// no load in flight between CTAs: 32 us for the 1,024 rows of the 4-token verify workload).
constexpr int kCombineThreads = 256;
// Splits a thread loads before folding them into its running statistics: all their loads are
// issued together, so a sequence of n splits costs about n / (G * kCombineBatch) memory round trips.
constexpr int kCombineBatch = 8;

// One CTA per (query row, sequence). Every group merges its own splits with the usual softmax
// rescale, a batch of loads at a time, into (m_g, l_g, acc_g), all in log2 units; the G group
// partials are merged in shared memory. A split with m = -inf (no visible key) weighs zero.
// Launched as a programmatic dependent of phase 1: griddepcontrol.wait holds every thread until
// phase 1 has completed and its workspace writes are visible (a no-op on a plain launch).
template <int D, bool BF16>
__global__ void __launch_bounds__(kCombineThreads) mfa_decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kRowThreads = D / 4;
  constexpr int G = kCombineThreads / kRowThreads;
  __shared__ __align__(16) float part[G][D];
  __shared__ float part_m[G], part_l[G];
  const int row = blockIdx.x;  // h * Nq + t
  const int b = blockIdx.y;
  const int dq = threadIdx.x % kRowThreads;  // columns 4 dq .. 4 dq + 3
  const int grp = threadIdx.x / kRowThreads;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int len = checked_len(p, b, false);
  const int n_pages = (len + kDecPage - 1) / kDecPage;
  const int n_splits = (n_pages - dec_first_page(p, len) + p.pages_per_split - 1) / p.pages_per_split;
  const size_t rows_all = (size_t)p.Hq * p.Nq;
  const size_t slot0 = (size_t)b * rows_all + row;  // slot of split s: slot0 + s * B * rows_all
  const size_t split_step = (size_t)p.B * rows_all;
  const float2* ml = reinterpret_cast<const float2*>(p.ws_ml);
  const float4* o = reinterpret_cast<const float4*>(p.ws_o + slot0 * D) + dq;
  const size_t stride = split_step * (D / 4);  // float4 steps from one split's row to the next

  float m_g = -INFINITY, l_g = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = grp; s0 < n_splits; s0 += G * kCombineBatch) {
    float2 st[kCombineBatch];
    float4 ov[kCombineBatch];
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) {
      const int s = s0 + j * G;
      st[j] = make_float2(-INFINITY, 0.f);
      ov[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s < n_splits) {
        st[j] = ml[slot0 + (size_t)s * split_step];
        ov[j] = o[(size_t)s * stride];
      }
    }
    float m_new = m_g;
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) m_new = fmaxf(m_new, st[j].x);
    if (m_new == -INFINITY) continue;
    const float r = (m_g == -INFINITY) ? 0.f : fast_exp2(m_g - m_new);
    l_g *= r;
    acc.x *= r;
    acc.y *= r;
    acc.z *= r;
    acc.w *= r;
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) {
      const float w = (st[j].x == -INFINITY) ? 0.f : fast_exp2(st[j].x - m_new);
      l_g = fmaf(w, st[j].y, l_g);
      acc.x = fmaf(w, ov[j].x, acc.x);
      acc.y = fmaf(w, ov[j].y, acc.y);
      acc.z = fmaf(w, ov[j].z, acc.z);
      acc.w = fmaf(w, ov[j].w, acc.w);
    }
    m_g = m_new;
  }
  *reinterpret_cast<float4*>(&part[grp][4 * dq]) = acc;
  if (dq == 0) {
    part_m[grp] = m_g;
    part_l[grp] = l_g;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int d = threadIdx.x;
    float M = part_m[0];
#pragma unroll
    for (int g = 1; g < G; ++g) M = fmaxf(M, part_m[g]);
    float L = 0.f, sum = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float w = (part_m[g] == -INFINITY) ? 0.f : fast_exp2(part_m[g] - M);
        L = fmaf(w, part_l[g], L);
        sum = fmaf(w, part[g][d], sum);
      }
    }
    const float val = (L > 0.f) ? sum / L : 0.f;
    const size_t orow = (size_t)b * rows_all + row;
    uint16_t bits;
    if constexpr (BF16) {
      bits = __bfloat16_as_ushort(__float2bfloat16_rn(val));
    } else {
      bits = __half_as_ushort(__float2half_rn(val));
    }
    reinterpret_cast<uint16_t*>(p.out)[orow * D + d] = bits;
    if (d == 0 && p.lse != nullptr) p.lse[orow] = (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace mfa
