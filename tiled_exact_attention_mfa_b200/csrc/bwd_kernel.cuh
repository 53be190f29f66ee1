// bwd_kernel.cuh -- exact attention backward for sm_100a: dQ, dK, dV of sum(O * dO).
//
// Algorithm: the three-pass FlashAttention-2 backward of "mlx-bun 0.4.0 -> 1.0.0,
// src/model/flash-attention.ts" (Backward: D-vec, dKV and dQ dispatches that recompute the scores
// from the saved log-sum-exp L): D_i = rowsum(dO_i * O_i); for a visible pair (i, j)
// p = exp(c_ij - L_i) with c the (capped) scaled score, dp = dO_i . v_j, ds = p (dp - D_i)
// (times 1 - tanh^2(s / cap) with a cap), dV_j += p dO_i, dK_j += scale ds q_i,
// dQ_i += scale ds k_j. No pass writes another pass's output, so every output is computed by
// one CTA and the result is deterministic (no atomics).
//
// B200 mapping. Both main passes run one CTA of 384 threads per 128-row tile:
//   warps 0-7  elementwise: a TMEM lane is a row of the CTA's tile (a key row in the dKV pass,
//              a query row in the dQ pass) and two warps share each row, one per 64-column half
//              of the 128 scores and 128 dP values; P and dS are packed to the input type.
//   warp 8     producer: TMA loads of the streamed tiles through a 2-stage ring (plus, in the
//              dKV pass, the 128 L and D values of each query tile, bounds-checked loads).
//   warp 9     TMEM owner and single-thread tcgen05.mma issuer.
// dKV pass (CTA = 128 keys of one kv head; loops over the query heads of its group and the
//   query tiles that can see the keys): S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 128
//   queries, K = D, operands K-major in smem), then dV += P^T dO and dK += dS^T Q (P^T, dS^T
//   from TMEM; dO, Q read MN-major from the same smem tiles). TMEM: S^T [0,128), dP^T
//   [128,256), dV [256,256+D), dK [256+D,256+2D); P^T and dS^T are packed over the dP^T
//   columns, so S^T of the next query tile is computed while the warps work on this one.
// dQ pass (CTA = 128 query rows of one head; loops over the key tiles the rows can see):
//   S = Q K^T, dP = dO V^T, then dQ += dS K (dS from TMEM, K MN-major). TMEM: S [0,128),
//   dP [128,256), dQ [256,256+D).
// The next step's S / dP MMAs overwrite the columns that hold P / dS, so the MMA thread waits
// for the previous step's consuming MMAs to complete before issuing them (tcgen05 orders only
// MMAs that share an accumulator).
#pragma once
#include "sm100.cuh"

namespace mfa {

constexpr int kBwdBM = 128;          // rows per tile (TMEM lanes), keys or queries
constexpr int kBwdStages = 2;
// setmaxnreg split of both main passes (384 threads): two elementwise warpgroups grow to 216
// registers, the producer / MMA warpgroup shrinks to 72; 256 x 216 + 128 x 72 = 384 x 168.
constexpr int kBwdQRegsElem = 216;
constexpr int kBwdQRegsCtl = 72;

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // [B*H][N][D] maps, 64 x 128 boxes, 128-byte swizzle
  const uint16_t* o;                    // [B, Hq, Nq, D] forward output
  const uint16_t* dout;                 // [B, Hq, Nq, D]
  const float* lse;                     // [B, Hq, Nq] natural-log LSE from the forward
  float* dvec;                          // [B, Hq, Nq] workspace: rowsum(dO * O)
  void* dq;                             // [B, Hq, Nq, D]
  void* dk;                             // [B, Hkv, Nk, D]
  void* dv;                             // [B, Hkv, Nk, D]
  int B, Hq, Hkv, Nq, Nk, G;
  int causal, win_l, win_r;
  int n_qt, n_kt;                       // 128-row query / key tiles per head
  float scale;
  float c_log2;                         // scale * log2 e
  float softcap, cap_in;                // cap, scale / cap (softcap = 0: off)
};

// ---------------------------------------------------------------- D-vec pass
// D_i = sum_d dO[i, d] * O[i, d] in fp32, one warp per row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) mfa_bwd_dvec_kernel(const __grid_constant__ BwdParams p) {
  const size_t rows = (size_t)p.B * p.Hq * p.Nq;
  const int lane = threadIdx.x & 31;
  const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t r = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const uint16_t* o = p.o + r * D;
    const uint16_t* g = p.dout + r * D;
    float acc = 0.f;
#pragma unroll
    for (int d = lane * 2; d < D; d += 64) {
      const uint32_t ov = *reinterpret_cast<const uint32_t*>(o + d);
      const uint32_t gv = *reinterpret_cast<const uint32_t*>(g + d);
      float o0, o1, g0, g1;
      unpack2<BF16>(ov, o0, o1);
      unpack2<BF16>(gv, g0, g1);
      acc = fmaf(o0, g0, fmaf(o1, g1, acc));
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (lane == 0) p.dvec[r] = acc;
  }
}

// Visible query rows [i_lo, i_hi] (inclusive, possibly empty) of key j: query i at absolute
// position a = i + Nk - Nq sees j iff (!causal || j <= a) && (win_l < 0 || j >= a - win_l) &&
// (win_r < 0 || j <= a + win_r).
__device__ __forceinline__ void bwd_rows_of_key(const BwdParams& p, int j, int& i_lo, int& i_hi) {
  const int off = p.Nk - p.Nq;
  int a_lo = -0x3fffffff, a_hi = 0x3fffffff;
  if (p.causal) a_lo = max(a_lo, j);
  if (p.win_r >= 0) a_lo = max(a_lo, j - p.win_r);
  if (p.win_l >= 0) a_hi = min(a_hi, j + p.win_l);
  i_lo = max(0, a_lo - off);
  i_hi = min(p.Nq - 1, a_hi - off);
}

// Visible keys [j_lo, j_hi] (inclusive, possibly empty) of query row i.
__device__ __forceinline__ void bwd_keys_of_row(const BwdParams& p, int i, int& j_lo, int& j_hi) {
  const int a = i + p.Nk - p.Nq;
  j_lo = 0;
  j_hi = p.Nk - 1;
  if (p.causal) j_hi = min(j_hi, a);
  if (p.win_r >= 0) j_hi = min(j_hi, a + p.win_r);
  if (p.win_l >= 0) j_lo = max(j_lo, a - p.win_l);
}

// tanh(y) for the softcap derivative and value: the small-argument polynomial when the whole
// warp's arguments allow it, else 1 - 2 / (2^(2|y| log2 e) + 1) with the sign restored.
__device__ __forceinline__ float bwd_tanh(float y, bool poly) {
  return poly ? y * tanh_q(y * y) : tanh_from_exp(y);
}

// ---------------------------------------------------------------- dKV pass
// 384 threads: warps 0-7 elementwise (warp w: key rows on TMEM lanes 32 (w % 4) .., query
// columns 64 (w / 4) .. of each query tile), warp 8 producer, warp 9 MMA issuer, warps 10-11
// idle; setmaxnreg as in the dQ pass. Each warp first reads its S^T values of both 32-column
// chunks (after which S^T of the next query tile may overwrite them), then per chunk reads the
// chunk's 32 dP^T columns and writes the chunk's packed P^T and dS^T (16 columns each) over
// them, so the two halves of a row never touch each other's columns; the dV / dK MMAs take
// query steps 2 ch + {0, 1} of half hf from columns 128 + 64 hf + 32 ch (+ 16 for dS^T).
constexpr int kBwdKvThreads = 384;

template <int D>
struct BwdKvSmem {
  static constexpr int kTile = kBwdBM * D * 2;
  uint8_t k[kTile];
  uint8_t v[kTile];
  uint8_t q[kBwdStages][kTile];
  uint8_t dout[kBwdStages][kTile];
  float nl[kBwdStages][kBwdBM];  // -L_i log2 e of the stage's query rows (0 past Nq / no key)
  float dd[kBwdStages][kBwdBM];  // D_i of the stage's query rows
  uint64_t bar_kv, bar_full[kBwdStages], bar_empty[kBwdStages];
  // bar_sfree: every elementwise warp has read its S^T (both chunks); bar_ds[ch]: chunk ch of
  // every warp stored; bar_sp: S^T and dP^T of the step ready; bar_mm: dV / dK of the step done
  uint64_t bar_sp, bar_sfree, bar_ds[2], bar_mm, bar_final;
  uint32_t tmem_base;
  int abort;
};

template <int D>
constexpr int bwd_kv_smem_bytes() {
  return (int)sizeof(BwdKvSmem<D>) + 1024;
}

// 128 x D tile of 16-bit values at smem address a as a K-major operand, K step kk (16 columns).
__device__ __forceinline__ uint64_t bwd_desc_k(uint32_t a, int kk) {
  return smem_desc_sw128(a + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
}
// The same tile as an MN-major B operand (rows = K dimension), K step kk (16 rows).
__device__ __forceinline__ uint64_t bwd_desc_mn(uint32_t a, int kk) {
  return smem_desc_sw128(a + kk * 16 * 128, 128 * 128, 1024);
}

template <int D, bool BF16, bool SOFTCAP>
__global__ void __launch_bounds__(kBwdKvThreads, 1) mfa_bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  BwdKvSmem<D>& sm = *reinterpret_cast<BwdKvSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: key tile kt of (b, kv head g); early key tiles (seen by the most causal rows) first
  const int BK = p.B * p.Hkv;
  const int kt = (int)(blockIdx.x / BK);
  const int b = (int)(blockIdx.x % BK) / p.Hkv;
  const int g = (int)(blockIdx.x % BK) % p.Hkv;
  const int k0 = kt * kBwdBM;
  const int k_last = min(k0 + kBwdBM, p.Nk) - 1;
  // Query rows that see some key of the tile: the first key's lowest row to the last key's
  // highest (both bounds grow with the key index).
  int r_lo, r_hi, t0, t1;
  bwd_rows_of_key(p, k0, r_lo, t0);
  bwd_rows_of_key(p, k_last, t1, r_hi);
  const int qt_lo = r_lo / kBwdBM;
  const int n_qt = (r_hi >= r_lo) ? r_hi / kBwdBM - qt_lo + 1 : 0;
  const int n_steps = n_qt * p.G;  // query heads of the group x query tiles, head-major

  constexpr int kSlabs = D / 64;
  constexpr uint32_t kTile = BwdKvSmem<D>::kTile;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.bar_kv), 1);
    for (int st = 0; st < kBwdStages; ++st) {
      mbar_init(smem_u32(&sm.bar_full[st]), 1);
      mbar_init(smem_u32(&sm.bar_empty[st]), 1);
    }
    mbar_init(smem_u32(&sm.bar_sp), 1);
    mbar_init(smem_u32(&sm.bar_sfree), 8);
    mbar_init(smem_u32(&sm.bar_ds[0]), 8);
    mbar_init(smem_u32(&sm.bar_ds[1]), 8);
    mbar_init(smem_u32(&sm.bar_mm), 1);
    mbar_init(smem_u32(&sm.bar_final), 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    tma_prefetch_desc(&p.tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp >= 8) {
   regs_dec<kBwdQRegsCtl>();
   if (warp == 8) {
    // ================================================================ producer
    if (n_steps > 0) {
      if (lane == 0) {
        const uint32_t bkv = smem_u32(&sm.bar_kv);
        mbar_expect_tx(bkv, 2 * kTile);
        for (int sl = 0; sl < kSlabs; ++sl) {
          tma_load_3d(smem_u32(sm.k) + sl * 128 * 128, &p.tm_k, bkv, sl * 64, k0, b * p.Hkv + g);
          tma_load_3d(smem_u32(sm.v) + sl * 128 * 128, &p.tm_v, bkv, sl * 64, k0, b * p.Hkv + g);
        }
      }
      int issued[kBwdStages] = {};
      for (int u = 0; u < n_steps; ++u) {
        const int st = u % kBwdStages;
        const int use = u / kBwdStages;
        const int h = g * p.G + u / n_qt;
        const int row0 = (qt_lo + u % n_qt) * kBwdBM;
        const bool ok = use == 0 || mbar_wait(smem_u32(&sm.bar_empty[st]), (use - 1) & 1, abort, 1101);
        if (!__all_sync(0xffffffffu, ok)) break;
        // -L log2 e and D of the tile's rows, 0 past Nq or where L = -inf (no visible key)
        const size_t base = (size_t)(b * p.Hq + h) * p.Nq;
#pragma unroll
        for (int rr = 0; rr < kBwdBM; rr += 32) {
          const int i = row0 + rr + lane;
          float l = 0.f, d = 0.f;
          if (i < p.Nq) {
            l = p.lse[base + i];
            d = p.dvec[base + i];
            if (!(l > -INFINITY)) l = 0.f;
          }
          sm.nl[st][rr + lane] = l * -1.4426950408889634f;
          sm.dd[st][rr + lane] = d;
        }
        __syncwarp();
        if (lane == 0) {
          const uint32_t bf = smem_u32(&sm.bar_full[st]);
          mbar_expect_tx(bf, 2 * kTile);
          for (int sl = 0; sl < kSlabs; ++sl) {
            tma_load_3d(smem_u32(sm.q[st]) + sl * 128 * 128, &p.tm_q, bf, sl * 64, row0, b * p.Hq + h);
            tma_load_3d(smem_u32(sm.dout[st]) + sl * 128 * 128, &p.tm_do, bf, sl * 64, row0, b * p.Hq + h);
          }
          issued[st] = use + 1;
        }
      }
      if (lane == 0) {  // no copy into this CTA's shared memory may outlive it
        volatile int no_abort = 0;
        mbar_wait(smem_u32(&sm.bar_kv), 0, &no_abort, 1102);
        for (int st = 0; st < kBwdStages; ++st)
          if (issued[st] > 0) mbar_wait(smem_u32(&sm.bar_full[st]), (issued[st] - 1) & 1, &no_abort, 1103);
      }
    }
   } else if (warp == 9) {
    // ================================================================ MMA issuer
    if (lane == 0 && n_steps > 0) {
      const uint32_t id_s = idesc_f16(BF16 ? 1 : 0, kBwdBM, kBwdBM, 0);  // S^T, dP^T: 128 x 128
      const uint32_t id_o = idesc_f16(BF16 ? 1 : 0, kBwdBM, D, 1);       // dV, dK: B MN-major
      const uint32_t ka = smem_u32(sm.k), va = smem_u32(sm.v);
      // S^T = K Q^T of the tile in stage st into columns [0, 128); dP^T = V dO^T into [128, 256)
      auto issue_s = [&](int st) {
        const uint32_t qa = smem_u32(sm.q[st]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma_ss(tmem + 0, bwd_desc_k(ka, kk), bwd_desc_k(qa, kk), id_s, kk > 0 ? 1u : 0u);
      };
      auto issue_dp = [&](int st) {
        const uint32_t oa = smem_u32(sm.dout[st]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma_ss(tmem + 128, bwd_desc_k(va, kk), bwd_desc_k(oa, kk), id_s, kk > 0 ? 1u : 0u);
      };
      // Per step u: dV / dK of step u chunk by chunk; S^T of step u + 1 between the two chunks
      // when its Q tile has landed (every warp has read S^T of step u by then, and P^T / dS^T of
      // step u go to the dP^T columns, so the S^T columns are free): it runs while the warps
      // compute the second chunk; otherwise right after the second chunk's dV / dK. Then, once
      // dV / dK have read P^T / dS^T, dP^T of step u + 1 and the commit that releases the warps
      // into step u + 1.
      bool ok = mbar_wait(smem_u32(&sm.bar_kv), 0, abort, 1201) &&
                mbar_wait(smem_u32(&sm.bar_full[0]), 0, abort, 1202);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        tc_commit(smem_u32(&sm.bar_sp));
      }
      for (int u = 0; ok && u < n_steps; ++u) {
        const int st = u % kBwdStages;
        const int st1 = (u + 1) % kBwdStages;
        const bool more = u + 1 < n_steps;
        const uint32_t qa = smem_u32(sm.q[st]), oa = smem_u32(sm.dout[st]);
        const uint32_t ph1 = ((u + 1) / kBwdStages) & 1;
        bool s_next = false;  // S^T of step u + 1 issued
        // packed P^T / dS^T of query step kk (16 queries) of half hf = kk / 4, chunk ch =
        // (kk / 2) % 2: P^T at column 128 + 64 hf + 32 ch + 8 (kk % 2), dS^T 16 columns further
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          if (!(ok = mbar_wait(smem_u32(&sm.bar_ds[ch]), u & 1, abort, 1204 + ch))) break;
          tc_fence_after();
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int kk = hf * 4 + ch * 2 + k2;
              tc_mma_ts(tmem + 256, tmem + 128 + hf * 64 + ch * 32 + k2 * 8, bwd_desc_mn(oa, kk),
                        id_o, (u > 0 || kk > 0) ? 1u : 0u);
            }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int kk = hf * 4 + ch * 2 + k2;
              tc_mma_ts(tmem + 256 + D, tmem + 128 + hf * 64 + ch * 32 + 16 + k2 * 8,
                        bwd_desc_mn(qa, kk), id_o, (u > 0 || kk > 0) ? 1u : 0u);
            }
          if (ch == 0 && more && mbar_test_wait(smem_u32(&sm.bar_full[st1]), ph1)) {
            // (every warp arrived on bar_sfree before its chunk-0 arrival: no real wait)
            if (!(ok = mbar_wait(smem_u32(&sm.bar_sfree), u & 1, abort, 1206))) break;
            tc_fence_after();
            issue_s(st1);
            s_next = true;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&sm.bar_mm));
        tc_commit(smem_u32(&sm.bar_empty[st]));
        if (more) {
          if (!s_next) {
            if (!(ok = mbar_wait(smem_u32(&sm.bar_full[st1]), ph1, abort, 1202))) break;
            if (!(ok = mbar_wait(smem_u32(&sm.bar_sfree), u & 1, abort, 1206))) break;
            tc_fence_after();
            issue_s(st1);
          }
          // dP^T of step u + 1 overwrites the packed P^T / dS^T that dV / dK of step u read
          if (!(ok = mbar_wait(smem_u32(&sm.bar_mm), u & 1, abort, 1203))) break;
          tc_fence_after();
          issue_dp(st1);
          tc_commit(smem_u32(&sm.bar_sp));  // also covers S^T of step u + 1
        }
      }
      tc_commit(smem_u32(&sm.bar_final));
      volatile int no_abort = 0;
      mbar_wait(smem_u32(&sm.bar_final), 0, &no_abort, 1205);
    }
   }
  } else {
    regs_inc<kBwdQRegsElem>();
    // ================================================================ elementwise (key rows)
    const int quarter = warp & 3;
    const int half = warp >> 2;  // query columns 64 half .. 64 half + 63 of each query tile
    const int j = k0 + quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    int ilo, ihi;
    bwd_rows_of_key(p, j, ilo, ihi);
    if (j >= p.Nk) {
      ilo = 1;
      ihi = 0;
    }
    const float c = p.c_log2;
    const float cc = p.softcap * 1.4426950408889634f;
    for (int u = 0; u < n_steps; ++u) {
      const int st = u % kBwdStages;
      const int col0 = (qt_lo + u % n_qt) * kBwdBM + half * 64;  // query row of this warp's column 0
      const bool got = mbar_wait(smem_u32(&sm.bar_sp), u & 1, abort, 1301);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const bool interior = __all_sync(0xffffffffu, ilo <= col0 && col0 + 63 <= ihi);
      const float* nlp = &sm.nl[st][half * 64];
      const float* ddp = &sm.dd[st][half * 64];
      // S^T of both chunks first: once every warp has it, S^T of the next step may be computed
      // into these columns while the warps work on this one
      uint32_t sr0[32], sr1[32];
      tmem_ld32(tmem + lane_base + half * 64, sr0);
      tmem_ld32(tmem + lane_base + half * 64 + 32, sr1);
      tmem_wait_ld(sr0, sr1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.bar_sfree));
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {  // 32 query columns at a time
        uint32_t(&sr)[32] = ch ? sr1 : sr0;
        uint32_t dr[32];
        tmem_ld32(tmem + lane_base + 128 + half * 64 + ch * 32, dr);
        tmem_wait_ld(dr);
        bool poly = false;
        if (SOFTCAP) {
          float am = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) am = fmaxf(am, fabsf(__uint_as_float(sr[e])));
          poly = __all_sync(0xffffffffu, am * p.cap_in <= kTanhPolyMax);
        }
        uint32_t pk[16], dk[16];
        // P^T = 2^(s c - L log2 e) (scores past the row / column limits are 0 on boundary tiles)
        // and dS^T = P^T (dP^T - D) [(1 - tanh^2) with a cap], two columns per packed f32x2 step
        auto chunk = [&](auto interior_c) {
          constexpr bool kInterior = decltype(interior_c)::value;
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const ulonglong2 n2 = *reinterpret_cast<const ulonglong2*>(nlp + ch * 32 + e4 * 4);
            const ulonglong2 d2 = *reinterpret_cast<const ulonglong2*>(ddp + ch * 32 + e4 * 4);
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
              const int e = e4 * 4 + hp * 2;
              const uint64_t nn = hp ? n2.y : n2.x;
              const uint64_t dd2 = hp ? d2.y : d2.x;
              float p0, p1;
              uint64_t fac2 = 0;
              if constexpr (SOFTCAP) {
                const float t0 = bwd_tanh(__uint_as_float(sr[e]) * p.cap_in, poly);
                const float t1 = bwd_tanh(__uint_as_float(sr[e + 1]) * p.cap_in, poly);
                const uint64_t t2 = f2_pack(t0, t1);
                f2_unpack(f2_fma(t2, f2_pack(cc, cc), nn), p0, p1);
                // 1 - t^2 with one rounding, as fmaf(-t, t, 1)
                fac2 = f2_fma(f2_mul(t2, f2_pack(-1.f, -1.f)), t2, f2_pack(1.f, 1.f));
              } else {
                f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])),
                                 f2_pack(c, c), nn), p0, p1);
              }
              p0 = fast_exp2(p0);
              p1 = fast_exp2(p1);
              if constexpr (!kInterior) {
                const int i = col0 + ch * 32 + e;
                if (i < ilo || i > ihi) p0 = 0.f;
                if (i + 1 < ilo || i + 1 > ihi) p1 = 0.f;
              }
              uint64_t ds2 = f2_mul(f2_pack(p0, p1),
                                    f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), dd2));
              if constexpr (SOFTCAP) ds2 = f2_mul(ds2, fac2);
              float s0, s1;
              f2_unpack(ds2, s0, s1);
              pk[e >> 1] = pack2<BF16>(p0, p1);
              dk[e >> 1] = pack2<BF16>(s0, s1);
            }
          }
        };
        if (interior) chunk(std::true_type{});
        else chunk(std::false_type{});
        // P^T and dS^T of the chunk (16 packed columns each) go over the chunk's own 32 dP^T
        // columns, which this warp has just read
        tmem_st16(tmem + lane_base + 128 + half * 64 + ch * 32, pk);
        tmem_st16(tmem + lane_base + 128 + half * 64 + ch * 32 + 16, dk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.bar_ds[ch]));
      }
    }
    // ---- epilogue: lower-column warps write dV, upper-column warps scale * dK, of their key rows
    bool have = false;
    if (n_steps > 0 && !*abort) {
      // bar_final: one commit after the MMA thread's last MMA, so a single-phase wait
      have = mbar_wait(smem_u32(&sm.bar_final), 0, abort, 1302);
      tc_fence_after();
    }
    have = __all_sync(0xffffffffu, have);
    const size_t obase = ((size_t)(b * p.Hkv + g) * p.Nk + (size_t)j) * D;
    const float mul = half ? p.scale : 1.f;
    uint16_t* dst_base = reinterpret_cast<uint16_t*>(half ? p.dk : p.dv);
#pragma unroll
    for (int cb = 0; cb < D; cb += 32) {
      uint32_t o[32];
      if (have) {
        tmem_ld32(tmem + lane_base + 256 + half * D + cb, o);
        tmem_wait_ld(o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (j < p.Nk) {
        uint4* dst = reinterpret_cast<uint4*>(dst_base + obase + cb);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          w.x = pack2<BF16>(__uint_as_float(o[v4 * 8 + 0]) * mul, __uint_as_float(o[v4 * 8 + 1]) * mul);
          w.y = pack2<BF16>(__uint_as_float(o[v4 * 8 + 2]) * mul, __uint_as_float(o[v4 * 8 + 3]) * mul);
          w.z = pack2<BF16>(__uint_as_float(o[v4 * 8 + 4]) * mul, __uint_as_float(o[v4 * 8 + 5]) * mul);
          w.w = pack2<BF16>(__uint_as_float(o[v4 * 8 + 6]) * mul, __uint_as_float(o[v4 * 8 + 7]) * mul);
          dst[v4] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dQ pass
// 384 threads: warps 0-7 elementwise (warp w: TMEM lanes 32 (w % 4) .., key columns
// 64 (w / 4) ..), warp 8 producer, warp 9 MMA issuer, warps 10-11 idle (setmaxnreg works on
// whole warpgroups: the elementwise warpgroups grow to 216 registers, the rest shrink to 72;
// 256 x 216 + 128 x 72 = 384 x 168 is the pool the CTA launches with).
// dS goes to two spare TMEM buffers [384, 448) and [448, 512), so S / dP of key tile u + 1 are
// computed while the elementwise warps work on tile u: the MMA thread issues them as soon as
// every elementwise warp has read S / dP of tile u (bar_ld), then dQ += dS K for tile u.
// K and V have rings of their own: V of tile u is read only by dP of tile u, so its slot is
// released as soon as S / dP of tile u complete; K is read again by dQ of tile u, so its ring has
// a third stage, and K of tile u + 1 is already in flight while dQ of tile u - 1 still reads its
// slot (with one shared 2-stage ring the copy of tile u + 1 started only after dQ of tile u - 1
// and sat on the critical path).
constexpr int kBwdQThreads = 384;
constexpr int kBwdQKStages = 3;
constexpr int kBwdQVStages = 2;

template <int D>
struct BwdQSmem {
  static constexpr int kTile = kBwdBM * D * 2;
  uint8_t q[kTile];
  uint8_t dout[kTile];
  uint8_t k[kBwdQKStages][kTile];
  uint8_t v[kBwdQVStages][kTile];
  uint64_t bar_qo, bar_kfull[kBwdQKStages], bar_kempty[kBwdQKStages];
  uint64_t bar_vfull[kBwdQVStages], bar_vempty[kBwdQVStages];
  // bar_ds[u % 2]: every elementwise warp stored dS of key tile u. S / dP of tile u + 1 are
  // issued once every warp has loaded tile u, so a fast warp can finish tile u + 1 before a slow
  // one finishes tile u; alternating barriers keep its arrival out of tile u's phase (it cannot
  // get two tiles ahead: S / dP of tile u + 2 wait for every warp to load tile u + 1).
  uint64_t bar_sp, bar_ld, bar_ds[2], bar_final;
  uint32_t tmem_base;
  int abort;
};

template <int D>
constexpr int bwd_q_smem_bytes() {
  return (int)sizeof(BwdQSmem<D>) + 1024;
}

template <int D, bool BF16, bool SOFTCAP>
__global__ void __launch_bounds__(kBwdQThreads, 1) mfa_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  BwdQSmem<D>& sm = *reinterpret_cast<BwdQSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: query tile qt of (b, h); late query tiles (most keys under causal) first
  const int BH = p.B * p.Hq;
  const int qt = p.n_qt - 1 - (int)(blockIdx.x / BH);
  const int b = (int)(blockIdx.x % BH) / p.Hq;
  const int h = (int)(blockIdx.x % BH) % p.Hq;
  const int g = h / p.G;
  const int q0 = qt * kBwdBM;
  const int q_last = min(q0 + kBwdBM, p.Nq) - 1;
  // keys seen by some row of the tile: the first row's lowest key to the last row's highest
  int j_lo, j_hi, t0, t1;
  bwd_keys_of_row(p, q0, j_lo, t0);
  bwd_keys_of_row(p, q_last, t1, j_hi);
  const int kt_lo = max(j_lo, 0) / kBwdBM;
  const int n_kt = (j_hi >= j_lo && j_hi >= 0) ? j_hi / kBwdBM - kt_lo + 1 : 0;

  constexpr int kSlabs = D / 64;
  constexpr uint32_t kTile = BwdQSmem<D>::kTile;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.bar_qo), 1);
    for (int st = 0; st < kBwdQKStages; ++st) {
      mbar_init(smem_u32(&sm.bar_kfull[st]), 1);
      mbar_init(smem_u32(&sm.bar_kempty[st]), 1);
    }
    for (int st = 0; st < kBwdQVStages; ++st) {
      mbar_init(smem_u32(&sm.bar_vfull[st]), 1);
      mbar_init(smem_u32(&sm.bar_vempty[st]), 1);
    }
    mbar_init(smem_u32(&sm.bar_sp), 1);
    mbar_init(smem_u32(&sm.bar_ld), 8);
    mbar_init(smem_u32(&sm.bar_ds[0]), 8);
    mbar_init(smem_u32(&sm.bar_ds[1]), 8);
    mbar_init(smem_u32(&sm.bar_final), 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    tma_prefetch_desc(&p.tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp >= 8) {
   regs_dec<kBwdQRegsCtl>();
   if (warp == 8) {
    // ================================================================ producer
    if (lane == 0 && n_kt > 0) {
      const uint32_t bqo = smem_u32(&sm.bar_qo);
      mbar_expect_tx(bqo, 2 * kTile);
      for (int sl = 0; sl < kSlabs; ++sl) {
        tma_load_3d(smem_u32(sm.q) + sl * 128 * 128, &p.tm_q, bqo, sl * 64, q0, b * p.Hq + h);
        tma_load_3d(smem_u32(sm.dout) + sl * 128 * 128, &p.tm_do, bqo, sl * 64, q0, b * p.Hq + h);
      }
      int issued_k[kBwdQKStages] = {}, issued_v[kBwdQVStages] = {};
      for (int u = 0; u < n_kt; ++u) {
        const int sk = u % kBwdQKStages, uk = u / kBwdQKStages;
        const int sv = u % kBwdQVStages, uv = u / kBwdQVStages;
        const int row = (kt_lo + u) * kBwdBM;
        if (uk > 0 && !mbar_wait(smem_u32(&sm.bar_kempty[sk]), (uk - 1) & 1, abort, 1401)) break;
        const uint32_t bk = smem_u32(&sm.bar_kfull[sk]);
        mbar_expect_tx(bk, kTile);
        for (int sl = 0; sl < kSlabs; ++sl)
          tma_load_3d(smem_u32(sm.k[sk]) + sl * 128 * 128, &p.tm_k, bk, sl * 64, row, b * p.Hkv + g);
        issued_k[sk] = uk + 1;
        if (uv > 0 && !mbar_wait(smem_u32(&sm.bar_vempty[sv]), (uv - 1) & 1, abort, 1404)) break;
        const uint32_t bv = smem_u32(&sm.bar_vfull[sv]);
        mbar_expect_tx(bv, kTile);
        for (int sl = 0; sl < kSlabs; ++sl)
          tma_load_3d(smem_u32(sm.v[sv]) + sl * 128 * 128, &p.tm_v, bv, sl * 64, row, b * p.Hkv + g);
        issued_v[sv] = uv + 1;
      }
      volatile int no_abort = 0;
      mbar_wait(bqo, 0, &no_abort, 1402);
      for (int st = 0; st < kBwdQKStages; ++st)
        if (issued_k[st] > 0) mbar_wait(smem_u32(&sm.bar_kfull[st]), (issued_k[st] - 1) & 1, &no_abort, 1403);
      for (int st = 0; st < kBwdQVStages; ++st)
        if (issued_v[st] > 0) mbar_wait(smem_u32(&sm.bar_vfull[st]), (issued_v[st] - 1) & 1, &no_abort, 1405);
    }
   } else if (warp == 9) {
    // ================================================================ MMA issuer
    if (lane == 0 && n_kt > 0) {
      const uint32_t id_s = idesc_f16(BF16 ? 1 : 0, kBwdBM, kBwdBM, 0);  // S, dP: 128 x 128
      const uint32_t id_o = idesc_f16(BF16 ? 1 : 0, kBwdBM, D, 1);       // dQ: B MN-major
      const uint32_t qa = smem_u32(sm.q), oa = smem_u32(sm.dout);
      auto issue_sdp = [&](int u) -> bool {
        const int sk = u % kBwdQKStages, sv = u % kBwdQVStages;
        if (!mbar_wait(smem_u32(&sm.bar_kfull[sk]), (u / kBwdQKStages) & 1, abort, 1502)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(sm.k[sk]), va = smem_u32(sm.v[sv]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma_ss(tmem + 0, bwd_desc_k(qa, kk), bwd_desc_k(ka, kk), id_s, kk > 0 ? 1u : 0u);
        if (!mbar_wait(smem_u32(&sm.bar_vfull[sv]), (u / kBwdQVStages) & 1, abort, 1506)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma_ss(tmem + 128, bwd_desc_k(oa, kk), bwd_desc_k(va, kk), id_s, kk > 0 ? 1u : 0u);
        tc_commit(smem_u32(&sm.bar_sp));  // also covers every earlier dQ MMA
        tc_commit(smem_u32(&sm.bar_vempty[sv]));  // V of tile u is not read again
        return true;
      };
      bool ok = mbar_wait(smem_u32(&sm.bar_qo), 0, abort, 1501) && issue_sdp(0);
      for (int u = 0; ok && u < n_kt; ++u) {
        if (u + 1 < n_kt) {
          // S / dP of tile u + 1 overwrite S / dP of tile u once every elementwise warp has read them
          if (!(ok = mbar_wait(smem_u32(&sm.bar_ld), u & 1, abort, 1503))) break;
          if (!(ok = issue_sdp(u + 1))) break;
        }
        if (!(ok = mbar_wait(smem_u32(&sm.bar_ds[u & 1]), (u >> 1) & 1, abort, 1504))) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(sm.k[u % kBwdQKStages]);
        const uint32_t ds_col = 384 + (u & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < kBwdBM / 16; ++kk)
          tc_mma_ts(tmem + 256, tmem + ds_col + kk * 8, bwd_desc_mn(ka, kk), id_o, (u > 0 || kk > 0) ? 1u : 0u);
        tc_commit(smem_u32(&sm.bar_kempty[u % kBwdQKStages]));
      }
      tc_commit(smem_u32(&sm.bar_final));
      volatile int no_abort = 0;
      mbar_wait(smem_u32(&sm.bar_final), 0, &no_abort, 1505);
    }
   }
  } else {
    regs_inc<kBwdQRegsElem>();
    // ================================================================ elementwise (query rows)
    const int quarter = warp & 3;
    const int half = warp >> 2;                 // key columns 64 half .. 64 half + 63 of each tile
    const int i = q0 + quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    int klo, khi;
    bwd_keys_of_row(p, i, klo, khi);
    float nl = 0.f, dd = 0.f;
    if (i < p.Nq) {
      const size_t idx = (size_t)(b * p.Hq + h) * p.Nq + i;
      nl = p.lse[idx];
      dd = p.dvec[idx];
      if (!(nl > -INFINITY)) nl = 0.f;
      nl *= -1.4426950408889634f;  // -L log2 e
    } else {
      klo = 1;
      khi = 0;
    }
    const float c = p.c_log2;
    const float cc = p.softcap * 1.4426950408889634f;
    for (int u = 0; u < n_kt; ++u) {
      const int kc0 = (kt_lo + u) * kBwdBM + half * 64;  // first key of this warp's columns
      const bool got = mbar_wait(smem_u32(&sm.bar_sp), u & 1, abort, 1601);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      uint32_t sr[64], dr[64];
      tmem_ld32(tmem + lane_base + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tmem + lane_base + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tmem + lane_base + 128 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
      tmem_ld32(tmem + lane_base + 128 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
      tmem_wait_ld(sr, dr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.bar_ld));  // S / dP columns may be overwritten now
      const bool interior = __all_sync(0xffffffffu, klo <= kc0 && kc0 + 63 <= khi);
      bool poly = false;
      if (SOFTCAP) {
        float am = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) am = fmaxf(am, fabsf(__uint_as_float(sr[e])));
        poly = __all_sync(0xffffffffu, am * p.cap_in <= kTanhPolyMax);
      }
      uint32_t dk[32];
      // dS = 2^(s c - L log2 e) (dP - D) [(1 - tanh^2) with a cap], zero past the row's key limits
      // on boundary tiles; two columns per packed f32x2 step
      const uint64_t nl2 = f2_pack(nl, nl), dd2 = f2_pack(dd, dd);
      auto tile = [&](auto interior_c) {
        constexpr bool kInterior = decltype(interior_c)::value;
#pragma unroll
        for (int e2 = 0; e2 < 32; ++e2) {
          const int e = 2 * e2;
          float p0, p1;
          uint64_t fac2 = 0;
          if constexpr (SOFTCAP) {
            const float t0 = bwd_tanh(__uint_as_float(sr[e]) * p.cap_in, poly);
            const float t1 = bwd_tanh(__uint_as_float(sr[e + 1]) * p.cap_in, poly);
            const uint64_t t2 = f2_pack(t0, t1);
            f2_unpack(f2_fma(t2, f2_pack(cc, cc), nl2), p0, p1);
            // 1 - t^2 with one rounding, as fmaf(-t, t, 1)
            fac2 = f2_fma(f2_mul(t2, f2_pack(-1.f, -1.f)), t2, f2_pack(1.f, 1.f));
          } else {
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])),
                             f2_pack(c, c), nl2), p0, p1);
          }
          p0 = fast_exp2(p0);
          p1 = fast_exp2(p1);
          if constexpr (!kInterior) {
            const int j = kc0 + e;
            if (j < klo || j > khi) p0 = 0.f;
            if (j + 1 < klo || j + 1 > khi) p1 = 0.f;
          }
          uint64_t ds2 = f2_mul(f2_pack(p0, p1),
                                f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), dd2));
          if constexpr (SOFTCAP) ds2 = f2_mul(ds2, fac2);
          float s0, s1;
          f2_unpack(ds2, s0, s1);
          dk[e2] = pack2<BF16>(s0, s1);
        }
      };
      if (interior) tile(std::true_type{});
      else tile(std::false_type{});
      // dS of tile u into buffer u % 2; the dQ MMA of tile u - 2 that read it is complete (the
      // commit that signalled S of tile u came after it)
      const uint32_t ds_col = 384 + (u & 1) * 64 + half * 32;
      tmem_st16(tmem + lane_base + ds_col, *reinterpret_cast<uint32_t(*)[16]>(&dk[0]));
      tmem_st16(tmem + lane_base + ds_col + 16, *reinterpret_cast<uint32_t(*)[16]>(&dk[16]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.bar_ds[u & 1]));
    }
    // ---- epilogue: scale * dQ of this query row, this warp's half of the columns
    bool have = false;
    if (n_kt > 0 && !*abort) {
      // bar_final: one commit after the MMA thread's last dQ MMA. (A parity wait on a barrier
      // committed once per key tile would be ambiguous here: when these warps finish their last
      // tile the MMA thread may not yet have issued dQ of the tile before it.)
      have = mbar_wait(smem_u32(&sm.bar_final), 0, abort, 1602);
      tc_fence_after();
    }
    have = __all_sync(0xffffffffu, have);
    const size_t obase = ((size_t)(b * p.Hq + h) * p.Nq + (size_t)i) * D + half * (D / 2);
#pragma unroll
    for (int cb = 0; cb < D / 2; cb += 32) {
      uint32_t o[32];
      if (have) {
        tmem_ld32(tmem + lane_base + 256 + half * (D / 2) + cb, o);
        tmem_wait_ld(o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (i < p.Nq) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.dq) + obase + cb);
        const float m = p.scale;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          w.x = pack2<BF16>(__uint_as_float(o[v4 * 8 + 0]) * m, __uint_as_float(o[v4 * 8 + 1]) * m);
          w.y = pack2<BF16>(__uint_as_float(o[v4 * 8 + 2]) * m, __uint_as_float(o[v4 * 8 + 3]) * m);
          w.z = pack2<BF16>(__uint_as_float(o[v4 * 8 + 4]) * m, __uint_as_float(o[v4 * 8 + 5]) * m);
          w.w = pack2<BF16>(__uint_as_float(o[v4 * 8 + 6]) * m, __uint_as_float(o[v4 * 8 + 7]) * m);
          dst[v4] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mfa
