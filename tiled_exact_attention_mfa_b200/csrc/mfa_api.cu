// mfa_api.cu -- the C ABI of libmfa.so (declared in include/mfa.h): argument validation, the
// split plan, TMA tensor maps and kernel launches. All kernels live in this translation unit so
// that the device status word is one symbol.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "fwd_kernel.cuh"
#include "mfa.h"

namespace {

thread_local mfa_launch_info g_last = {};
int g_debug_flags = 0;
// Debug override of the decode split size (0 = the plan's own). Every entry point reads it once
// and passes that value down, so the size check and the launched plan of one call agree even
// while another thread changes it.
std::atomic<int> g_split_pages_override{0};
std::mutex g_mutex;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// ------------------------------------------------------------------ driver entry point
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Encodes one 3-D map over a 16-bit tensor with a 128-byte swizzle:
//   kind 0: [outer][n][D] (dense q / k / v / out), box 64 x 128 x 1: one box is one 128-row x
//           128-byte slab of one head, so tails past n are zero-filled per head;
//   kind 1: packed variable-length [n = total][outer = H][D], ordered (D, head, token), box
//           64 x 1 x 128: the same 128-row x 128-byte slab as kind 0;
//   kind 2: page pools [num_pages * 16 = n tokens][outer = H][D], ordered (D, head, token), box
//           64 x 1 x 16: one box is one page of one head, 16 rows of a slab.
bool encode_map(CUtensorMap* m, const void* base, int dtype, int kind, long long outer, long long n, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3];
  if (kind == 0) {
    dims[0] = (cuuint64_t)D; dims[1] = (cuuint64_t)n; dims[2] = (cuuint64_t)outer;
    strides[0] = (cuuint64_t)D * 2; strides[1] = (cuuint64_t)n * D * 2;
    box[0] = 64; box[1] = 128; box[2] = 1;
  } else {
    dims[0] = (cuuint64_t)D; dims[1] = (cuuint64_t)outer; dims[2] = (cuuint64_t)n;
    strides[0] = (cuuint64_t)D * 2; strides[1] = (cuuint64_t)outer * D * 2;
    box[0] = 64; box[1] = 1; box[2] = kind == 1 ? 128 : 16;
  }
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dtype == MFA_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ tensor-map cache
// A map depends only on (base pointer, data type, layout kind, extents); repeated calls over the
// same buffers (a serving loop, a training step) would re-encode identical maps every time, each
// a driver call of about a microsecond on the host. Encoded maps are therefore kept per device
// under that key: kTmapCacheEntries entries, the least recently used one replaced, one mutex
// (calls may come from several host threads). A map stays correct for any later allocation at
// the same address with the same extents, since it describes addresses, not an allocation.
struct TmapKey {
  int dev, kind, dtype, D;
  const void* base;
  long long outer, n;
  bool operator==(const TmapKey& o) const {
    return dev == o.dev && kind == o.kind && dtype == o.dtype && D == o.D && base == o.base &&
           outer == o.outer && n == o.n;
  }
};

constexpr int kTmapCacheEntries = 256;
// Keys of the fake encoder of mfa_debug_tmap_probe live under this device number, so they never
// match a key of a real launch.
constexpr int kTmapFakeDevice = -2;

struct TmapCache {
  struct Entry {
    CUtensorMap map;
    TmapKey key;
    unsigned long long stamp;  // 0 = empty
  };
  std::mutex mu;
  Entry e[kTmapCacheEntries] = {};
  unsigned long long clock = 0, lookups = 0, encodes = 0;

  // Copies the map of `k` into *out, encoding (and inserting) it on a miss. `encoded` tells which.
  template <typename Enc>
  bool get(const TmapKey& k, CUtensorMap* out, Enc&& encode, bool* encoded) {
    std::lock_guard<std::mutex> lk(mu);
    ++lookups;
    int victim = 0;
    for (int i = 0; i < kTmapCacheEntries; ++i) {
      if (e[i].stamp != 0 && e[i].key == k) {
        e[i].stamp = ++clock;
        *out = e[i].map;
        if (encoded) *encoded = false;
        return true;
      }
      if (e[i].stamp < e[victim].stamp) victim = i;
    }
    CUtensorMap m;
    if (!encode(&m)) return false;
    ++encodes;
    e[victim].map = m;
    e[victim].key = k;
    e[victim].stamp = ++clock;
    *out = m;
    if (encoded) *encoded = true;
    return true;
  }
};
TmapCache g_tmaps;

bool cached_map(CUtensorMap* m, const void* base, int dtype, int kind, long long outer, long long n, int D) {
  const int dev = current_device();
  if (dev < 0) return false;
  const TmapKey k = {dev, kind, dtype, D, base, outer, n};
  return g_tmaps.get(k, m, [&](CUtensorMap* dst) { return encode_map(dst, base, dtype, kind, outer, n, D); },
                     nullptr);
}

// 3-D map over a [rows_outer][n][D] 16-bit tensor (kind 0).
bool make_map(CUtensorMap* m, const void* base, int dtype, long long outer, long long n, int D) {
  return cached_map(m, base, dtype, 0, outer, n, D);
}

// Packed variable-length layout [total, H, D] (kind 1).
bool make_map_packed(CUtensorMap* m, const void* base, int dtype, long long total, int H, int D) {
  return cached_map(m, base, dtype, 1, H, total, D);
}

// Page pools [num_pages, 16, H, D] seen as [num_pages * 16 tokens, H, D] (kind 2).
bool make_map_pages(CUtensorMap* m, const void* base, int dtype, long long tokens, int H, int D) {
  return cached_map(m, base, dtype, 2, H, tokens, D);
}

// Opt a kernel into its dynamic shared memory size once per device.
template <typename K>
bool ensure_smem(K kernel, int bytes, bool (&done)[kMaxDevices]) {
  int dev = current_device();
  if (dev < 0) return false;
  if (done[dev]) return true;
  std::lock_guard<std::mutex> lk(g_mutex);
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

// ------------------------------------------------------------------ decode split plan
struct DecodePlan {
  int pages_per_split;
  int max_splits;
  int heads_per_cta;
  int groups;
};

// With a left window (win_l >= 0) splits are counted from each sequence's first visible page,
// so a sequence spans at most win_pages pages. Such a grid is small and each CTA pays a fixed
// start-up latency (block table, Q and first page in flight), so the split is halved only while
// the halved grid still fits one wave of two CTAs per SM, and never past the split count of the
// unwindowed plan, so the workspace that mfa_decode_workspace_size reports stays sufficient.
DecodePlan decode_plan(int B, int Hkv, int D, int max_pages, int Nq, int win_l, int override_pages) {
  DecodePlan pl;
  // kv heads per CTA: the largest divisor of Hkv whose token row (heads x D x 2 bytes) fits in
  // 1 KB, so that a 3-stage K+V page ring stays near 100 KB and two CTAs share an SM (one
  // streams pages while the other starts up or drains).
  pl.heads_per_cta = 1;
  for (int h = 8; h >= 1; --h)
    if (Hkv % h == 0 && h * D * 2 <= 1024) {
      pl.heads_per_cta = h;
      break;
    }
  pl.groups = Hkv / pl.heads_per_cta;
  const int s0 = 32;
  int s = s0;
  if (override_pages > 0) {
    s = std::min(override_pages, mfa::kDecMaxSplitPages);
  } else {
    // halve the split while the grid would hold fewer than two CTAs per SM (148 SMs)
    while (s > 4 && (long long)B * ((max_pages + s - 1) / s) * pl.groups < 296) s /= 2;
  }
  pl.pages_per_split = s;
  pl.max_splits = (max_pages + s - 1) / s;
  if (win_l >= 0) {
    const long long win_pages = ((long long)win_l + Nq + mfa::kDecPage - 1) / mfa::kDecPage + 1;
    const int span = (int)std::min<long long>(max_pages, win_pages);
    const int cap = pl.max_splits;
    if (override_pages <= 0) {
      s = s0;
      while (s > 4 && (long long)B * ((span + s / 2 - 1) / (s / 2)) * pl.groups <= 296 &&
             (span + s / 2 - 1) / (s / 2) <= cap)
        s /= 2;
    }
    pl.pages_per_split = s;
    pl.max_splits = (span + s - 1) / s;
  }
  return pl;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_sizes(long long a, long long b, long long c, long long d) {
  // element counts must fit comfortably in 63 bits and TMA coordinates in 31 bits
  if (a < 0 || b < 0 || c < 0 || d < 0) return MFA_ERR_BAD_SHAPE;
  long double n = (long double)a * b * c * d;
  if (n > 4.0e18L) return MFA_ERR_BAD_SHAPE;
  return MFA_OK;
}

// Arguments of one forward launch (dense, or packed variable-length when cu_q != NULL; then Nq
// is the longest sequence's query count, which sizes the grid).
struct FwdCall {
  const void *q, *k, *v;
  void* out;
  float* lse;
  int B, Hq, Hkv, Nq, Nk;
  float scale;
  int causal, win_l, win_r;
  float softcap;
  int dtype;
  const int32_t *cu_q, *cu_k;
  int total_q, total_k;
  const uint8_t* block_mask;  // block-sparse: [B, Hq, ceil(Nq/128), ceil(Nk/128)]
  const int32_t *block_table, *seq_lens;  // paged keys
  int max_pages, num_pages;
};

// ONE: the single-Q-tile CTA shape (two CTAs per SM); see mfa::FwdShape.
template <int D, bool BF16, bool VARLEN, bool SPARSE, bool SOFTCAP, bool PAGED, bool PART, bool ONE = false>
int launch_fwd(const FwdCall& c, cudaStream_t st) {
  const int B = c.B, Hq = c.Hq, Hkv = c.Hkv, Nq = c.Nq, Nk = c.Nk, dtype = c.dtype;
  const float scale = c.scale, softcap = c.softcap;
  using Shape = mfa::FwdShape<ONE>;
  static bool smem_done[kMaxDevices] = {};
  static bool regs_ok[kMaxDevices] = {};
  constexpr int smem = mfa::fwd_smem_bytes<D, SPARSE, ONE>();
  static_assert(!ONE || 2 * (smem + 1024) <= 233472, "two single-Q-tile CTAs must fit one SM");
  auto kernel = mfa::mfa_fwd_kernel<D, BF16, VARLEN, SPARSE, SOFTCAP, PAGED, PART, ONE>;
  if (!ensure_smem(kernel, smem, smem_done)) return MFA_ERR_CUDA;
  {
    // setmaxnreg redistributes the registers the CTA launched with; refuse to launch if the
    // split does not fit that pool (the growing warpgroups would wait forever).
    const int dev = current_device();
    if (dev < 0) return MFA_ERR_CUDA;
    if (!regs_ok[dev]) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return MFA_ERR_CUDA;
      if (fa.numRegs * Shape::kThreads <
          Shape::kQT * 128 * Shape::kRegsSoftmax + 128 * Shape::kRegsControl)
        return MFA_ERR_CUDA;
      regs_ok[dev] = true;
    }
  }
  mfa::FwdParams p;
  std::memset(&p, 0, sizeof(p));
  if (PAGED) {
    if (!make_map_packed(&p.tm_q, c.q, dtype, c.total_q, Hq, D)) return MFA_ERR_CUDA;
    if (!make_map_packed(&p.tm_o, c.out, dtype, c.total_q, Hq, D)) return MFA_ERR_CUDA;
    if (!make_map_pages(&p.tm_k, c.k, dtype, (long long)c.num_pages * 16, Hkv, D)) return MFA_ERR_CUDA;
    if (!make_map_pages(&p.tm_v, c.v, dtype, (long long)c.num_pages * 16, Hkv, D)) return MFA_ERR_CUDA;
    p.cu_q = c.cu_q;
    p.total_q = c.total_q;
    p.block_table = c.block_table;
    p.seq_lens = c.seq_lens;
    p.max_pages = c.max_pages;
    p.num_pages = c.num_pages;
  } else if (VARLEN) {
    if (!make_map_packed(&p.tm_q, c.q, dtype, c.total_q, Hq, D)) return MFA_ERR_CUDA;
    if (!make_map_packed(&p.tm_o, c.out, dtype, c.total_q, Hq, D)) return MFA_ERR_CUDA;
    if (!make_map_packed(&p.tm_k, c.k, dtype, c.total_k, Hkv, D)) return MFA_ERR_CUDA;
    if (!make_map_packed(&p.tm_v, c.v, dtype, c.total_k, Hkv, D)) return MFA_ERR_CUDA;
    p.cu_q = c.cu_q;
    p.cu_k = c.cu_k;
    p.total_q = c.total_q;
    p.total_k = c.total_k;
  } else {
    if (!make_map(&p.tm_q, c.q, dtype, (long long)B * Hq, Nq, D)) return MFA_ERR_CUDA;
    if (!make_map(&p.tm_o, c.out, dtype, (long long)B * Hq, Nq, D)) return MFA_ERR_CUDA;
    if (!make_map(&p.tm_k, c.k, dtype, (long long)B * Hkv, Nk, D)) return MFA_ERR_CUDA;
    if (!make_map(&p.tm_v, c.v, dtype, (long long)B * Hkv, Nk, D)) return MFA_ERR_CUDA;
  }
  p.out = c.out;
  p.lse = c.lse;
  if (SPARSE) {
    p.block_mask = c.block_mask;
    p.nqt = (Nq + mfa::kFwdBM - 1) / mfa::kFwdBM;
    p.nkt = (Nk + mfa::kFwdBN - 1) / mfa::kFwdBN;
  }
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.causal = c.causal ? 1 : 0;
  p.win_l = c.win_l;
  p.win_r = c.win_r;
  const int rows_per_cta = mfa::kFwdBM * Shape::kQT;
  p.n_qblk = (Nq + rows_per_cta - 1) / rows_per_cta;
  p.flags = g_debug_flags;
  if (p.flags & MFA_DEBUG_COUNT_TILES) {
    void* ctr = nullptr;
    if (cudaGetSymbolAddress(&ctr, mfa::g_tile_counter) != cudaSuccess) return MFA_ERR_CUDA;
    p.tile_counter = static_cast<unsigned long long*>(ctr);
  }
  const float log2e = 1.4426950408889634f;
  // the kernel keeps (capped score) / scale per key, so the exponent factor is scale * log2 e
  // with or without a cap
  p.c_log2 = scale * log2e;
  if (softcap > 0.f) {
    p.softcap = softcap;
    p.cap_in = scale / softcap;
    p.cap_out = softcap / scale;
  } else {
    p.softcap = 0.f;
    p.cap_in = 0.f;
    p.cap_out = 0.f;
  }
  p.lse_mul = 0.69314718055994531f;
  const long long grid = (long long)p.n_qblk * B * Hq;
  if (grid > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  kernel<<<(unsigned)grid, Shape::kThreads, smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  mfa_launch_info li = {};
  li.kernel = 1;
  li.grid_x = (int)grid;
  li.grid_y = li.grid_z = 1;
  li.block_threads = Shape::kThreads;
  li.smem_bytes = smem;
  li.tile_m = mfa::kFwdBM;
  li.tile_n = mfa::kFwdBN;
  li.q_tiles_per_cta = Shape::kQT;
  g_last = li;
  return MFA_OK;
}

// Parts of the decode a launch runs.
constexpr int kDecPhase1 = 1;
constexpr int kDecCombine = 2;

// Phase 1 over splits [p.split_lo, split_hi) and / or the combine. With both, the combine is a
// programmatic dependent of phase 1: it is launched while the last phase-1 CTAs still run and
// waits in griddepcontrol.wait until their workspace writes are visible. Alone, it is a plain
// launch ordered after earlier work on the stream (its wait is then a no-op).
template <int D, bool BF16>
int launch_decode(const mfa::DecodeParams& p, const DecodePlan& pl, int split_hi, int parts,
                  cudaStream_t st) {
  static bool smem_done[kMaxDevices] = {};
  const int smem = mfa::dec_smem_bytes<D>(pl.heads_per_cta);
  mfa_launch_info li = {};
  li.kernel = 2;
  const bool phase1 = (parts & kDecPhase1) && split_hi > p.split_lo;
  if (phase1) {
    // the largest plan (1024 / (2 D) heads per CTA) sets the attribute for all
    auto k1 = mfa::mfa_decode_phase1_kernel<D, BF16>;
    if (!ensure_smem(k1, mfa::dec_smem_bytes<D>(mfa::kDecMaxHeads<D>), smem_done)) return MFA_ERR_CUDA;
    dim3 g1(split_hi - p.split_lo, p.B, pl.groups);
    k1<<<g1, (pl.heads_per_cta + 1) * 32, smem, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
    li.grid_x = g1.x;
    li.grid_y = g1.y;
    li.grid_z = g1.z;
    li.block_threads = (pl.heads_per_cta + 1) * 32;
    li.smem_bytes = smem;
  }
  if (parts & kDecCombine) {
    dim3 g2(p.Hq * p.Nq, p.B, 1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = g2;
    cfg.blockDim = dim3(mfa::kCombineThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = phase1 ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, mfa::mfa_decode_combine_kernel<D, BF16>, p) != cudaSuccess)
      return MFA_ERR_CUDA;
  }
  li.pages_per_split = pl.pages_per_split;
  li.max_splits = pl.max_splits;
  li.kv_heads_per_cta = pl.heads_per_cta;
  g_last = li;
  return MFA_OK;
}

template <int D>
int dispatch_decode_d(const mfa::DecodeParams& p, const DecodePlan& pl, int split_hi, int parts,
                      bool bf, cudaStream_t st) {
  return bf ? launch_decode<D, true>(p, pl, split_hi, parts, st)
            : launch_decode<D, false>(p, pl, split_hi, parts, st);
}

int dispatch_decode(const mfa::DecodeParams& p, const DecodePlan& pl, int D, int split_hi, int parts,
                    bool bf, cudaStream_t st) {
  if (D == 256) return dispatch_decode_d<256>(p, pl, split_hi, parts, bf, st);
  if (D == 128) return dispatch_decode_d<128>(p, pl, split_hi, parts, bf, st);
  return dispatch_decode_d<64>(p, pl, split_hi, parts, bf, st);
}

// Checks shared by the dense and the packed forward.
int validate_fwd_common(int Hq, int Hkv, int D, int dtype, int win_l, int win_r,
                               float softcap, float scale) {
  if (dtype != MFA_DTYPE_FP16 && dtype != MFA_DTYPE_BF16) return MFA_ERR_BAD_DTYPE;
  if (D != 64 && D != 128) return MFA_ERR_BAD_HEAD_DIM;
  if (Hq < 0) return MFA_ERR_BAD_SHAPE;
  if (Hkv < 1 || Hq % Hkv != 0) return MFA_ERR_GQA_GEOMETRY;
  if (win_l < -1 || win_r < -1) return MFA_ERR_BAD_WINDOW;
  if (!std::isfinite(softcap) || softcap < 0.f) return MFA_ERR_BAD_SOFTCAP;
  if (!std::isfinite(scale) || !(scale > 0.f)) return MFA_ERR_BAD_SCALE;
  return MFA_OK;
}

// A window wider than any sequence of the call is the same as no bound on that side; it is
// replaced by -1 before launch, so the kernels' 32-bit position arithmetic (a - win_l,
// a + win_r + 1, with positions below 2^30) cannot wrap around for windows near INT_MAX.
// max_k bounds every key count of the call and max_q every query count.
void clamp_window(int& win_l, int& win_r, long long max_k, long long max_q) {
  if (win_l >= max_k) win_l = -1;
  if (win_r >= max_q) win_r = -1;
}

// Sequence lengths the kernels index with 32-bit positions.
constexpr long long kMaxTokens = 0x3fffffffLL;

// Every row sees no key: out = 0, lse = -inf (rows = number of (query, head) pairs).
int launch_fill_empty(void* out, float* lse, size_t rows, int D, int dtype, cudaStream_t st) {
  if (dtype == MFA_DTYPE_BF16)
    mfa::mfa_fill_empty_kernel<true><<<148, 256, 0, st>>>(out, lse, rows, D);
  else
    mfa::mfa_fill_empty_kernel<false><<<148, 256, 0, st>>>(out, lse, rows, D);
  if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  mfa_launch_info li = {};
  li.kernel = 3;
  li.grid_x = 148;
  li.grid_y = li.grid_z = 1;
  li.block_threads = 256;
  g_last = li;
  return MFA_OK;
}

template <bool VARLEN, bool SPARSE, bool SOFTCAP, bool PAGED, bool PART, bool ONE>
int dispatch_fwd_d(const FwdCall& c, int D, cudaStream_t st) {
  const bool bf = c.dtype == MFA_DTYPE_BF16;
  if (D == 128)
    return bf ? launch_fwd<128, true, VARLEN, SPARSE, SOFTCAP, PAGED, PART, ONE>(c, st)
              : launch_fwd<128, false, VARLEN, SPARSE, SOFTCAP, PAGED, PART, ONE>(c, st);
  return bf ? launch_fwd<64, true, VARLEN, SPARSE, SOFTCAP, PAGED, PART, ONE>(c, st)
            : launch_fwd<64, false, VARLEN, SPARSE, SOFTCAP, PAGED, PART, ONE>(c, st);
}

// PART: each Q tile of a CTA computes only the key tiles its own rows see; ONE: one Q tile per
// CTA, two CTAs per SM (dense sliding windows)
template <bool VARLEN, bool SPARSE, bool PAGED = false, bool PART = false, bool ONE = false>
int dispatch_fwd(const FwdCall& c, int D, cudaStream_t st) {
  return c.softcap > 0.f ? dispatch_fwd_d<VARLEN, SPARSE, true, PAGED, PART, ONE>(c, D, st)
                         : dispatch_fwd_d<VARLEN, SPARSE, false, PAGED, PART, ONE>(c, D, st);
}

template <int D, bool BF16, bool SOFTCAP>
int launch_bwd(mfa::BwdParams& p, const void* q, const void* k, const void* v, const void* dout,
               int dtype, cudaStream_t st) {
  static bool smem_kv[kMaxDevices] = {}, smem_q[kMaxDevices] = {};
  auto kdkv = mfa::mfa_bwd_dkv_kernel<D, BF16, SOFTCAP>;
  auto kdq = mfa::mfa_bwd_dq_kernel<D, BF16, SOFTCAP>;
  if (!ensure_smem(kdkv, mfa::bwd_kv_smem_bytes<D>(), smem_kv)) return MFA_ERR_CUDA;
  if (!ensure_smem(kdq, mfa::bwd_q_smem_bytes<D>(), smem_q)) return MFA_ERR_CUDA;
  {
    // the dQ pass redistributes its launch registers with setmaxnreg: refuse a launch whose
    // register count would not cover the split (the growing warpgroups would wait forever)
    static bool regs_ok[kMaxDevices] = {};
    const int dev = current_device();
    if (dev < 0) return MFA_ERR_CUDA;
    if (!regs_ok[dev]) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kdq) != cudaSuccess) return MFA_ERR_CUDA;
      if (fa.numRegs * mfa::kBwdQThreads < 256 * mfa::kBwdQRegsElem + 128 * mfa::kBwdQRegsCtl)
        return MFA_ERR_CUDA;
      if (cudaFuncGetAttributes(&fa, kdkv) != cudaSuccess) return MFA_ERR_CUDA;
      if (fa.numRegs * mfa::kBwdKvThreads < 256 * mfa::kBwdQRegsElem + 128 * mfa::kBwdQRegsCtl)
        return MFA_ERR_CUDA;
      regs_ok[dev] = true;
    }
  }
  if (!make_map(&p.tm_q, q, dtype, (long long)p.B * p.Hq, p.Nq, D)) return MFA_ERR_CUDA;
  if (!make_map(&p.tm_do, dout, dtype, (long long)p.B * p.Hq, p.Nq, D)) return MFA_ERR_CUDA;
  if (!make_map(&p.tm_k, k, dtype, (long long)p.B * p.Hkv, p.Nk, D)) return MFA_ERR_CUDA;
  if (!make_map(&p.tm_v, v, dtype, (long long)p.B * p.Hkv, p.Nk, D)) return MFA_ERR_CUDA;
  const long long rows = (long long)p.B * p.Hq * p.Nq;
  long long g0 = (rows + 7) / 8;
  if (g0 > 148 * 16) g0 = 148 * 16;
  mfa::mfa_bwd_dvec_kernel<D, BF16><<<(unsigned)g0, 256, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  const long long g1 = (long long)p.n_kt * p.B * p.Hkv;
  const long long g2 = (long long)p.n_qt * p.B * p.Hq;
  if (g1 > 0x7FFFFFFFLL || g2 > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  kdkv<<<(unsigned)g1, mfa::kBwdKvThreads, mfa::bwd_kv_smem_bytes<D>(), st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  kdq<<<(unsigned)g2, mfa::kBwdQThreads, mfa::bwd_q_smem_bytes<D>(), st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  mfa_launch_info li = {};
  li.kernel = 4;
  li.grid_x = (int)g1;
  li.grid_y = (int)g2;
  li.grid_z = 1;
  li.block_threads = mfa::kBwdKvThreads;
  li.smem_bytes = mfa::bwd_kv_smem_bytes<D>();
  li.tile_m = mfa::kBwdBM;
  li.tile_n = mfa::kBwdBM;
  g_last = li;
  return MFA_OK;
}

}  // namespace

extern "C" {

int mfa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
            int Hkv, int Nq, int Nk, int D, float scale, int causal, int win_l, int win_r,
            float softcap, int dtype, void* stream) {
  int rc = validate_fwd_common(Hq, Hkv, D, dtype, win_l, win_r, softcap, scale);
  if (rc != MFA_OK) return rc;
  if (B < 0 || Nq < 0 || Nk < 0) return MFA_ERR_BAD_SHAPE;
  if ((rc = check_sizes(B, Hq, Nq, D)) != MFA_OK) return rc;
  if ((rc = check_sizes(B, Hkv, Nk, D)) != MFA_OK) return rc;
  if ((long long)B * Hq > 0x7FFFFFFFLL || (long long)B * Hkv > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  if (Nq > kMaxTokens || Nk > kMaxTokens) return MFA_ERR_BAD_SHAPE;
  if (B == 0 || Hq == 0 || Nq == 0) return MFA_OK;
  if (!q || !out || (Nk > 0 && (!k || !v))) return MFA_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || (Nk > 0 && (!aligned16(k) || !aligned16(v))))
    return MFA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (Nk == 0) return launch_fill_empty(out, lse, (size_t)B * Hq * Nq, D, dtype, st);
  clamp_window(win_l, win_r, Nk, Nq);
  FwdCall c = {q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, scale, causal, win_l, win_r, softcap, dtype,
               nullptr, nullptr, 0, 0, nullptr, nullptr, nullptr, 0, 0};
  // Uncapped: the single-Q-tile shape (two CTAs per SM, which hide each other's start and end;
  // measured faster on causal, non-causal and windowed workloads). With a cap its softmax needs
  // more registers than that shape's split gives, so capped calls keep two Q tiles per CTA (under
  // a window each computing only its own run of key tiles).
  if (c.softcap <= 0.f) return dispatch_fwd_d<false, false, false, false, false, true>(c, D, st);
  if (win_l >= 0 || win_r >= 0) return dispatch_fwd_d<false, false, true, false, true, false>(c, D, st);
  return dispatch_fwd_d<false, false, true, false, false, false>(c, D, st);
}

int mfa_fwd_blocksparse(const void* q, const void* k, const void* v, void* out, float* lse,
                        const uint8_t* block_mask, int B, int Hq, int Hkv, int Nq, int Nk, int D,
                        float scale, int causal, int win_l, int win_r, float softcap, int dtype,
                        void* stream) {
  int rc = validate_fwd_common(Hq, Hkv, D, dtype, win_l, win_r, softcap, scale);
  if (rc != MFA_OK) return rc;
  if (B < 0 || Nq < 0 || Nk < 0) return MFA_ERR_BAD_SHAPE;
  if ((rc = check_sizes(B, Hq, Nq, D)) != MFA_OK) return rc;
  if ((rc = check_sizes(B, Hkv, Nk, D)) != MFA_OK) return rc;
  if ((long long)B * Hq > 0x7FFFFFFFLL || (long long)B * Hkv > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  if ((long long)(Nk + mfa::kFwdBN - 1) / mfa::kFwdBN > mfa::kFwdMaxSparseTiles) return MFA_ERR_UNSUPPORTED;
  if (Nq > kMaxTokens || Nk > kMaxTokens) return MFA_ERR_BAD_SHAPE;
  if (B == 0 || Hq == 0 || Nq == 0) return MFA_OK;
  if (!q || !out || !block_mask || (Nk > 0 && (!k || !v))) return MFA_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || (Nk > 0 && (!aligned16(k) || !aligned16(v))))
    return MFA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (Nk == 0) return launch_fill_empty(out, lse, (size_t)B * Hq * Nq, D, dtype, st);
  clamp_window(win_l, win_r, Nk, Nq);
  FwdCall c = {q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, scale, causal, win_l, win_r, softcap, dtype,
               nullptr, nullptr, 0, 0, block_mask, nullptr, nullptr, 0, 0};
  return dispatch_fwd<false, true>(c, D, st);
}

int mfa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                   const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int max_seqlen_q,
                   int total_q, int total_k, int Hq, int Hkv, int D, float scale, int causal,
                   int win_l, int win_r, float softcap, int dtype, void* stream) {
  int rc = validate_fwd_common(Hq, Hkv, D, dtype, win_l, win_r, softcap, scale);
  if (rc != MFA_OK) return rc;
  if (B < 0 || max_seqlen_q < 0 || total_q < 0 || total_k < 0) return MFA_ERR_BAD_SHAPE;
  if (max_seqlen_q > total_q) return MFA_ERR_BAD_SHAPE;
  if ((rc = check_sizes(total_q, Hq, D, 1)) != MFA_OK) return rc;
  if ((rc = check_sizes(total_k, Hkv, D, 1)) != MFA_OK) return rc;
  if ((long long)B * Hq > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  if (total_q > kMaxTokens || total_k > kMaxTokens) return MFA_ERR_BAD_SHAPE;
  if (B == 0 || Hq == 0 || total_q == 0 || max_seqlen_q == 0) return MFA_OK;
  if (!q || !out || !cu_seqlens_q || !cu_seqlens_k || (total_k > 0 && (!k || !v)))
    return MFA_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(out) || !aligned16(lse) ||
      (total_k > 0 && (!aligned16(k) || !aligned16(v))) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return MFA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (total_k == 0) return launch_fill_empty(out, lse, (size_t)total_q * Hq, D, dtype, st);
  clamp_window(win_l, win_r, total_k, total_q);
  FwdCall c = {q, k, v, out, lse, B, Hq, Hkv, max_seqlen_q, 0, scale, causal, win_l, win_r, softcap,
               dtype, cu_seqlens_q, cu_seqlens_k, total_q, total_k, nullptr, nullptr, nullptr, 0, 0};
  return dispatch_fwd<true, false>(c, D, st);
}

int mfa_fwd_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                  const int32_t* seq_lens, const int32_t* cu_seqlens_q, void* out, float* lse, int B,
                  int max_seqlen_q, int total_q, int Hq, int Hkv, int D, int page_size,
                  int max_pages_per_seq, int num_pages, float scale, int causal, int win_l, int win_r,
                  float softcap, int dtype, void* stream) {
  int rc = validate_fwd_common(Hq, Hkv, D, dtype, win_l, win_r, softcap, scale);
  if (rc != MFA_OK) return rc;
  if (page_size != mfa::kDecPage) return MFA_ERR_PAGE_SIZE;
  if (B < 0 || max_seqlen_q < 0 || total_q < 0 || max_pages_per_seq < 1 || num_pages < 1)
    return MFA_ERR_BAD_SHAPE;
  if (max_seqlen_q > total_q) return MFA_ERR_BAD_SHAPE;
  if ((rc = check_sizes(total_q, Hq, D, 1)) != MFA_OK) return rc;
  if ((rc = check_sizes(num_pages, page_size, Hkv, D)) != MFA_OK) return rc;
  if ((long long)max_pages_per_seq * 16 > 0x3fffffffLL || (long long)num_pages * 16 > 0x3fffffffLL)
    return MFA_ERR_BAD_SHAPE;
  if ((long long)B * Hq > 0x7FFFFFFFLL || total_q > kMaxTokens) return MFA_ERR_BAD_SHAPE;
  if (B == 0 || Hq == 0 || total_q == 0 || max_seqlen_q == 0) return MFA_OK;
  if (!q || !out || !k_pages || !v_pages || !block_table || !seq_lens || !cu_seqlens_q)
    return MFA_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || !aligned16(k_pages) || !aligned16(v_pages) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u))
    return MFA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  clamp_window(win_l, win_r, (long long)max_pages_per_seq * 16, total_q);
  FwdCall c = {q, k_pages, v_pages, out, lse, B, Hq, Hkv, max_seqlen_q, 0, scale, causal, win_l, win_r,
               softcap, dtype, cu_seqlens_q, nullptr, total_q, 0, nullptr, block_table, seq_lens,
               max_pages_per_seq, num_pages};
  return dispatch_fwd<true, false, true>(c, D, st);
}

static int validate_decode(int B, int Nq, int Hq, int Hkv, int D, int page_size, int max_pages) {
  if (D != 64 && D != 128 && D != 256) return MFA_ERR_BAD_HEAD_DIM;
  if (B < 0 || Hq < 0) return MFA_ERR_BAD_SHAPE;
  if (Nq < 1 || Nq > 4) return Nq < 1 ? MFA_ERR_BAD_SHAPE : MFA_ERR_NQ_TOO_LARGE;
  if (Hkv < 1 || Hq % Hkv != 0 || Hq < 1) return MFA_ERR_GQA_GEOMETRY;
  if (page_size != mfa::kDecPage) return MFA_ERR_PAGE_SIZE;
  if (max_pages < 1) return MFA_ERR_BAD_SHAPE;
  if ((Hq / Hkv) * Nq > 16) return MFA_ERR_UNSUPPORTED;
  if ((long long)max_pages * mfa::kDecPage > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  return MFA_OK;
}

size_t mfa_bwd_workspace_size(int B, int Hq, int Nq) {
  if (B < 0 || Hq < 0 || Nq < 0) return 0;
  if (check_sizes(B, Hq, Nq, 1) != MFA_OK) return 0;
  return align256((size_t)B * Hq * Nq * sizeof(float));
}

int mfa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
            const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
            int D, float scale, int causal, int win_l, int win_r, float softcap, int dtype,
            void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_fwd_common(Hq, Hkv, D, dtype, win_l, win_r, softcap, scale);
  if (rc != MFA_OK) return rc;
  if (B < 0 || Nq < 0 || Nk < 0) return MFA_ERR_BAD_SHAPE;
  if ((rc = check_sizes(B, Hq, Nq, D)) != MFA_OK) return rc;
  if ((rc = check_sizes(B, Hkv, Nk, D)) != MFA_OK) return rc;
  if ((long long)B * Hq > 0x7FFFFFFFLL || (long long)B * Hkv > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  if (Nq > kMaxTokens || Nk > kMaxTokens) return MFA_ERR_BAD_SHAPE;
  if (B == 0 || Hq == 0 || (Nq == 0 && Nk == 0)) return MFA_OK;
  clamp_window(win_l, win_r, Nk, Nq);
  const bool need_q = Nq > 0, need_k = Nk > 0;
  if ((need_q && (!q || !out || !dout || !lse || !dq)) || (need_k && (!k || !v || !dk || !dv)))
    return MFA_ERR_NULL_POINTER;
  if ((need_q && (!aligned16(q) || !aligned16(out) || !aligned16(dout) || !aligned16(lse) || !aligned16(dq))) ||
      (need_k && (!aligned16(k) || !aligned16(v) || !aligned16(dk) || !aligned16(dv))))
    return MFA_ERR_MISALIGNED;
  const size_t need = mfa_bwd_workspace_size(B, Hq, Nq);
  if (need_q && need_k &&
      (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need))
    return MFA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!need_k) {  // no keys: every query row sees nothing, so dQ = 0
    return cudaMemsetAsync(dq, 0, (size_t)B * Hq * Nq * D * 2, st) == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
  }
  if (!need_q) {  // no queries: no key receives a gradient
    if (cudaMemsetAsync(dk, 0, (size_t)B * Hkv * Nk * D * 2, st) != cudaSuccess) return MFA_ERR_CUDA;
    return cudaMemsetAsync(dv, 0, (size_t)B * Hkv * Nk * D * 2, st) == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
  }
  mfa::BwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.o = static_cast<const uint16_t*>(out);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.dvec = static_cast<float*>(workspace);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.G = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.win_l = win_l;
  p.win_r = win_r;
  p.n_qt = (Nq + mfa::kBwdBM - 1) / mfa::kBwdBM;
  p.n_kt = (Nk + mfa::kBwdBM - 1) / mfa::kBwdBM;
  p.scale = scale;
  p.c_log2 = scale * 1.4426950408889634f;
  p.softcap = softcap > 0.f ? softcap : 0.f;
  p.cap_in = softcap > 0.f ? scale / softcap : 0.f;
  const bool bf = dtype == MFA_DTYPE_BF16;
  const bool cap = p.softcap > 0.f;
#define MFA_BWD_CAP(DD, BB) \
  (cap ? launch_bwd<DD, BB, true>(p, q, k, v, dout, dtype, st) : launch_bwd<DD, BB, false>(p, q, k, v, dout, dtype, st))
  if (D == 128) return bf ? MFA_BWD_CAP(128, true) : MFA_BWD_CAP(128, false);
  return bf ? MFA_BWD_CAP(64, true) : MFA_BWD_CAP(64, false);
#undef MFA_BWD_CAP
}

int mfa_decode_plan(int B, int Nq, int Hq, int Hkv, int D, int max_pages_per_seq, int page_size,
                    int win_l, int* pages_per_split, int* max_splits, int* kv_heads_per_cta) {
  if (win_l < -1) return MFA_ERR_BAD_WINDOW;
  const int rc = validate_decode(B, Nq, Hq, Hkv, D, page_size, max_pages_per_seq);
  if (rc != MFA_OK) return rc;
  const DecodePlan pl = decode_plan(B, Hkv, D, max_pages_per_seq, Nq, win_l, g_split_pages_override.load());
  if (pages_per_split) *pages_per_split = pl.pages_per_split;
  if (max_splits) *max_splits = pl.max_splits;
  if (kv_heads_per_cta) *kv_heads_per_cta = pl.heads_per_cta;
  return MFA_OK;
}

}  // extern "C"

namespace {

size_t decode_workspace_size(int B, int Nq, int Hq, int Hkv, int D, int max_pages_per_seq,
                             int page_size, int override_pages) {
  if (validate_decode(B, Nq, Hq, Hkv, D, page_size, max_pages_per_seq) != MFA_OK) return 0;
  DecodePlan pl = decode_plan(B, Hkv, D, max_pages_per_seq, Nq, -1, override_pages);
  const size_t rows = (size_t)B * pl.max_splits * Hq * Nq;
  return align256(rows * D * sizeof(float)) + align256(rows * 2 * sizeof(float));
}

// Checks every argument of a decode call that phase 1 needs (pointers may be NULL only where
// the caller passes nullptr for `need_kv`), derives the plan and fills the kernel parameters
// (partial-result pointers left to the caller).
int decode_params(mfa::DecodeParams& p, DecodePlan& pl, const void* q, const void* k_pages,
                  const void* v_pages, const int32_t* block_table, const int32_t* seq_lens,
                  void* out, float* lse, int B, int Nq, int Hq, int Hkv, int D, int page_size,
                  int max_pages_per_seq, int num_pages, float scale, int causal, int win_l,
                  float softcap, int dtype, int override_pages, bool need_kv, bool need_out) {
  if (dtype != MFA_DTYPE_FP16 && dtype != MFA_DTYPE_BF16) return MFA_ERR_BAD_DTYPE;
  if (win_l < -1) return MFA_ERR_BAD_WINDOW;
  int rc = validate_decode(B, Nq, Hq, Hkv, D, page_size, max_pages_per_seq);
  if (rc != MFA_OK) return rc;
  if (need_kv && num_pages < 1) return MFA_ERR_BAD_SHAPE;
  if (!std::isfinite(softcap) || softcap < 0.f) return MFA_ERR_BAD_SOFTCAP;
  if (!std::isfinite(scale) || !(scale > 0.f)) return MFA_ERR_BAD_SCALE;
  if (need_kv && (rc = check_sizes(num_pages, page_size, Hkv, D)) != MFA_OK) return rc;
  if ((rc = check_sizes(B, Hq, Nq, D)) != MFA_OK) return rc;
  if (B == 0) return MFA_OK;
  if (!seq_lens || (need_kv && (!q || !k_pages || !v_pages || !block_table)) || (need_out && !out))
    return MFA_ERR_NULL_POINTER;
  if (!aligned16(seq_lens) || (need_kv && (!aligned16(q) || !aligned16(k_pages) ||
                                           !aligned16(v_pages) || !aligned16(block_table))) ||
      (need_out && (!aligned16(out) || !aligned16(lse))))
    return MFA_ERR_MISALIGNED;
  pl = decode_plan(B, Hkv, D, max_pages_per_seq, Nq, win_l, override_pages);
  if (pl.max_splits > 0x7FFFFFFF || B > 65535 || pl.groups > 65535) return MFA_ERR_BAD_SHAPE;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const uint16_t*>(q);
  p.k_pages = static_cast<const uint16_t*>(k_pages);
  p.v_pages = static_cast<const uint16_t*>(v_pages);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.Nq = Nq;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.max_pages = max_pages_per_seq;
  p.num_pages = num_pages;
  p.pages_per_split = pl.pages_per_split;
  p.max_splits = pl.max_splits;
  p.heads_per_cta = pl.heads_per_cta;
  p.causal = causal ? 1 : 0;
  p.win_l = win_l;
  const float log2e = 1.4426950408889634f;
  if (softcap > 0.f) {
    p.softcap = softcap;
    p.cap_in = scale / softcap;
    p.c_log2 = log2e;
  } else {
    p.c_log2 = scale * log2e;
  }
  return MFA_OK;
}

// The decode entry points after their override read: override_pages is the split-size override
// this call uses for both the workspace check and the launched plan.
int decode_splitkv(const void* q, const void* k_pages, const void* v_pages,
                   const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                   int B, int Nq, int Hq, int Hkv, int D, int page_size, int max_pages_per_seq,
                   int num_pages, float scale, int causal, int win_l, float softcap, int dtype,
                   void* workspace, size_t workspace_bytes, cudaStream_t st, int override_pages) {
  mfa::DecodeParams p;
  DecodePlan pl;
  int rc = decode_params(p, pl, q, k_pages, v_pages, block_table, seq_lens, out, lse, B, Nq, Hq,
                         Hkv, D, page_size, max_pages_per_seq, num_pages, scale, causal, win_l,
                         softcap, dtype, override_pages, true, true);
  if (rc != MFA_OK || B == 0) return rc;
  const size_t need = decode_workspace_size(B, Nq, Hq, Hkv, D, max_pages_per_seq, page_size, override_pages);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return MFA_ERR_WORKSPACE;
  // the unwindowed plan sizes the workspace; a window's plan never has more splits
  const DecodePlan full = decode_plan(B, Hkv, D, max_pages_per_seq, Nq, -1, override_pages);
  const size_t rows = (size_t)B * full.max_splits * Hq * Nq;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(rows * D * sizeof(float)));
  p.split_lo = 0;
  return dispatch_decode(p, pl, D, pl.max_splits, kDecPhase1 | kDecCombine,
                         dtype == MFA_DTYPE_BF16, st);
}

}  // namespace

extern "C" {

size_t mfa_decode_workspace_size(int B, int Nq, int Hq, int Hkv, int D, int max_pages_per_seq,
                                 int page_size) {
  return decode_workspace_size(B, Nq, Hq, Hkv, D, max_pages_per_seq, page_size,
                               g_split_pages_override.load());
}

int mfa_decode_splitkv_window(const void* q, const void* k_pages, const void* v_pages,
                              const int32_t* block_table, const int32_t* seq_lens, void* out,
                              float* lse, int B, int Nq, int Hq, int Hkv, int D, int page_size,
                              int max_pages_per_seq, int num_pages, float scale, int causal,
                              int win_l, float softcap, int dtype, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return decode_splitkv(q, k_pages, v_pages, block_table, seq_lens, out, lse, B, Nq, Hq, Hkv, D,
                        page_size, max_pages_per_seq, num_pages, scale, causal, win_l, softcap,
                        dtype, workspace, workspace_bytes, static_cast<cudaStream_t>(stream),
                        g_split_pages_override.load());
}

int mfa_decode_phase1(const void* q, const void* k_pages, const void* v_pages,
                      const int32_t* block_table, const int32_t* seq_lens, int B, int Nq, int Hq,
                      int Hkv, int D, int page_size, int max_pages_per_seq, int num_pages,
                      float scale, int causal, int win_l, float softcap, int dtype, int split_lo,
                      int split_hi, float* part_o, float* part_ml, int split_capacity,
                      void* stream) {
  const int ovr = g_split_pages_override.load();
  mfa::DecodeParams p;
  DecodePlan pl;
  int rc = decode_params(p, pl, q, k_pages, v_pages, block_table, seq_lens, nullptr, nullptr, B,
                         Nq, Hq, Hkv, D, page_size, max_pages_per_seq, num_pages, scale, causal,
                         win_l, softcap, dtype, ovr, true, false);
  if (rc != MFA_OK || B == 0) return rc;
  if (split_lo < 0 || split_hi < split_lo || split_hi > pl.max_splits) return MFA_ERR_BAD_SHAPE;
  if (split_capacity < pl.max_splits || !part_o || !part_ml) return MFA_ERR_WORKSPACE;
  if (!aligned16(part_o) || !aligned16(part_ml)) return MFA_ERR_MISALIGNED;
  p.ws_o = part_o;
  p.ws_ml = part_ml;
  p.split_lo = split_lo;
  return dispatch_decode(p, pl, D, split_hi, kDecPhase1, dtype == MFA_DTYPE_BF16,
                         static_cast<cudaStream_t>(stream));
}

int mfa_decode_combine(const int32_t* seq_lens, void* out, float* lse, int B, int Nq, int Hq,
                       int Hkv, int D, int page_size, int max_pages_per_seq, int win_l, int dtype,
                       const float* part_o, const float* part_ml, int split_capacity,
                       void* stream) {
  const int ovr = g_split_pages_override.load();
  mfa::DecodeParams p;
  DecodePlan pl;
  int rc = decode_params(p, pl, nullptr, nullptr, nullptr, nullptr, seq_lens, out, lse, B, Nq, Hq,
                         Hkv, D, page_size, max_pages_per_seq, 1, 1.0f, 1, win_l, 0.f, dtype, ovr,
                         false, true);
  if (rc != MFA_OK || B == 0) return rc;
  if (split_capacity < pl.max_splits || !part_o || !part_ml) return MFA_ERR_WORKSPACE;
  if (!aligned16(part_o) || !aligned16(part_ml)) return MFA_ERR_MISALIGNED;
  p.ws_o = const_cast<float*>(part_o);
  p.ws_ml = const_cast<float*>(part_ml);
  return dispatch_decode(p, pl, D, 0, kDecCombine, dtype == MFA_DTYPE_BF16,
                         static_cast<cudaStream_t>(stream));
}

int mfa_decode_splitkv(const void* q, const void* k_pages, const void* v_pages,
                       const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                       int B, int Nq, int Hq, int Hkv, int D, int page_size, int max_pages_per_seq,
                       int num_pages, float scale, int causal, float softcap, int dtype,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return mfa_decode_splitkv_window(q, k_pages, v_pages, block_table, seq_lens, out, lse, B, Nq, Hq,
                                   Hkv, D, page_size, max_pages_per_seq, num_pages, scale, causal,
                                   -1, softcap, dtype, workspace, workspace_bytes, stream);
}

const char* mfa_status_string(int code) {
  switch (code) {
    case MFA_OK: return "ok";
    case MFA_ERR_NULL_POINTER: return "a required pointer is NULL";
    case MFA_ERR_MISALIGNED: return "a tensor pointer is not 16-byte aligned";
    case MFA_ERR_BAD_DTYPE: return "dtype must be MFA_DTYPE_FP16 or MFA_DTYPE_BF16";
    case MFA_ERR_BAD_HEAD_DIM: return "head dim D must be 64 or 128";
    case MFA_ERR_BAD_SHAPE: return "invalid or overflowing size";
    case MFA_ERR_GQA_GEOMETRY: return "Hkv must be >= 1 and divide Hq";
    case MFA_ERR_BAD_WINDOW: return "window bounds must be >= -1";
    case MFA_ERR_BAD_SOFTCAP: return "softcap must be finite and >= 0";
    case MFA_ERR_BAD_SCALE: return "scale must be finite and > 0";
    case MFA_ERR_NQ_TOO_LARGE: return "split-KV decode takes at most 4 query tokens";
    case MFA_ERR_PAGE_SIZE: return "page_size must be 16";
    case MFA_ERR_WORKSPACE: return "workspace is NULL, not 256-byte aligned or too small";
    case MFA_ERR_UNSUPPORTED: return "decode supports at most 16 query rows ((Hq/Hkv)*Nq) per kv head";
    case MFA_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case MFA_ERR_DEVICE_TIMEOUT: return "device: a bounded wait inside a kernel ran out";
    case MFA_ERR_DEVICE_BAD_PAGE: return "device: block_table or seq_lens entry out of range";
    case MFA_ERR_DEVICE_BAD_SEQLENS: return "device: cu_seqlens entry negative, decreasing, past the packed total, or a sequence longer than max_seqlen_q";
    case MFA_ERR_DEVICE_TILE_LIST: return "device: a key-tile list exceeded its capacity (tiles past it were not visited)";
    case MFA_ERR_SCRATCH_TOO_SMALL: return "decode shape needs more workspace than the fixed 64 MiB scratch of mfa_decode_splitkv_noalloc";
    default: return "unknown status";
  }
}

int mfa_last_launch_info(mfa_launch_info* info) {
  if (!info) return MFA_ERR_NULL_POINTER;
  *info = g_last;
  return MFA_OK;
}

int mfa_device_status(void* stream, int* code, int* detail) {
  if (!code || !detail) return MFA_ERR_NULL_POINTER;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h[2] = {0, 0};
  if (cudaMemcpyFromSymbolAsync(h, mfa::g_status, sizeof(h), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MFA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MFA_ERR_CUDA;
  int zero[2] = {0, 0};
  if (cudaMemcpyToSymbolAsync(mfa::g_status, zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MFA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MFA_ERR_CUDA;
  *code = h[0];
  *detail = h[1];
  return MFA_OK;
}

int mfa_debug_set_flags(int flags) {
  int old = g_debug_flags;
  g_debug_flags = flags;
  return old;
}

int mfa_debug_tiles_visited(void* stream, unsigned long long* count) {
  if (!count) return MFA_ERR_NULL_POINTER;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned long long h = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&h, mfa::g_tile_counter, sizeof(h), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MFA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MFA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(mfa::g_tile_counter, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MFA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MFA_ERR_CUDA;
  *count = h;
  return MFA_OK;
}

int mfa_debug_tmap_stats(unsigned long long* lookups, unsigned long long* encodes) {
  if (!lookups || !encodes) return MFA_ERR_NULL_POINTER;
  std::lock_guard<std::mutex> lk(g_tmaps.mu);
  *lookups = g_tmaps.lookups;
  *encodes = g_tmaps.encodes;
  return MFA_OK;
}

int mfa_debug_tmap_probe(const void* base, int kind, int dtype, long long outer, long long n, int D,
                         int* encoded) {
  if (!encoded) return MFA_ERR_NULL_POINTER;
  if (kind < 0 || kind > 2) return MFA_ERR_BAD_SHAPE;
  const TmapKey k = {kTmapFakeDevice, kind, dtype, D, base, outer, n};
  CUtensorMap m;
  bool enc = false;
  // the fake encoder writes the key's fields into the map and needs no driver
  auto fake = [&](CUtensorMap* dst) {
    std::memset(dst, 0, sizeof(*dst));
    long long f[4] = {(long long)(uintptr_t)base, outer, n, (long long)kind * 1000 + D};
    std::memcpy(dst, f, sizeof(f));
    return true;
  };
  if (!g_tmaps.get(k, &m, fake, &enc)) return MFA_ERR_CUDA;
  long long f[4];
  std::memcpy(f, &m, sizeof(f));
  if (f[0] != (long long)(uintptr_t)base || f[1] != outer || f[2] != n || f[3] != (long long)kind * 1000 + D)
    return MFA_ERR_CUDA;  // a hit returned another key's map
  *encoded = enc ? 1 : 0;
  return MFA_OK;
}

int mfa_debug_set_decode_split_pages(int pages) {
  return g_split_pages_override.exchange(pages < 0 ? 0 : pages);
}

}  // extern "C"

// ----------------------------------------------------------------------------------------------
// Allocation-free decode: the workspace lives in a fixed device array of this file.
namespace {

constexpr size_t kNoAllocScratchBytes = MFA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device. In host code the array's name only stands in
// for the device symbol; kernels must be given the address cudaGetSymbolAddress returns.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

void* noalloc_scratch(int dev) {
  std::lock_guard<std::mutex> lk(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int mfa_decode_splitkv_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                          const int32_t* block_table, const int32_t* seq_lens,
                                          void* out, float* lse, int B, int Nq, int Hq, int Hkv,
                                          int D, int page_size, int max_pages_per_seq,
                                          int num_pages, float scale, int causal, float softcap,
                                          int dtype, void* stream) {
  // one read of the split-size override serves the size check and the launch
  const int ovr = g_split_pages_override.load();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Every argument check of the decode runs first; with no workspace it returns before any
  // launch, and MFA_ERR_WORKSPACE then means that everything else is valid.
  int rc = decode_splitkv(q, k_pages, v_pages, block_table, seq_lens, out, lse, B, Nq, Hq, Hkv, D,
                          page_size, max_pages_per_seq, num_pages, scale, causal, -1, softcap,
                          dtype, nullptr, 0, st, ovr);
  if (rc != MFA_ERR_WORKSPACE) return rc;
  const size_t need = decode_workspace_size(B, Nq, Hq, Hkv, D, max_pages_per_seq, page_size, ovr);
  if (need > kNoAllocScratchBytes) return MFA_ERR_SCRATCH_TOO_SMALL;
  const int dev = current_device();
  if (dev < 0) return MFA_ERR_CUDA;
  void* scratch = noalloc_scratch(dev);
  if (scratch == nullptr) return MFA_ERR_CUDA;
  return decode_splitkv(q, k_pages, v_pages, block_table, seq_lens, out, lse, B, Nq, Hq, Hkv, D,
                        page_size, max_pages_per_seq, num_pages, scale, causal, -1, softcap, dtype,
                        scratch, kNoAllocScratchBytes, st, ovr);
}

// ----------------------------------------------------------------------------------------------
// Forward over host buffers: the batch x kv-head units are cut into up to kHostChunks contiguous
// runs of about 12 MiB of input each; run c's inputs are copied in on an internal stream while
// run c - 1 computes on the caller's stream and run c - 2's outputs are copied out on a second
// internal stream, so the PCIe copies in the two directions and the kernels overlap. Each run of units [u0, u1) is the
// forward problem B' = u1 - u0, Hq' = Hq / Hkv, Hkv' = 1 over the same memory layout.
namespace {

constexpr int kHostChunks = 8;

struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t entry = nullptr, done = nullptr;
  cudaEvent_t in_done[kHostChunks] = {}, comp_done[kHostChunks] = {};
};
HostPipe g_host_pipe[kMaxDevices];
std::mutex g_host_mutex[kMaxDevices];

bool host_pipe_init(HostPipe& hp) {
  if (hp.ready) return true;
  const unsigned ev = cudaEventDisableTiming;
  if (cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaEventCreateWithFlags(&hp.entry, ev) != cudaSuccess) return false;
  if (cudaEventCreateWithFlags(&hp.done, ev) != cudaSuccess) return false;
  for (int c = 0; c < kHostChunks; ++c) {
    if (cudaEventCreateWithFlags(&hp.in_done[c], ev) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&hp.comp_done[c], ev) != cudaSuccess) return false;
  }
  hp.ready = true;
  return true;
}

struct HostLayout {
  size_t q_bytes, kv_bytes, lse_bytes;
  size_t off_k, off_v, off_out, off_lse, total;
};
HostLayout host_layout(int B, int Hq, int Hkv, int Nq, int Nk, int D) {
  HostLayout L;
  L.q_bytes = (size_t)B * Hq * Nq * D * 2;
  L.kv_bytes = (size_t)B * Hkv * Nk * D * 2;
  L.lse_bytes = (size_t)B * Hq * Nq * sizeof(float);
  L.off_k = align256(L.q_bytes);
  L.off_v = L.off_k + align256(L.kv_bytes);
  L.off_out = L.off_v + align256(L.kv_bytes);
  L.off_lse = L.off_out + align256(L.q_bytes);
  L.total = L.off_lse + align256(L.lse_bytes);
  return L;
}

}  // namespace

extern "C" size_t mfa_fwd_host_scratch_size(int B, int Hq, int Hkv, int Nq, int Nk, int D) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Nq < 0 || Nk < 0 || Hq % Hkv != 0) return 0;
  if (D != 64 && D != 128) return 0;
  if (check_sizes(B, Hq, Nq, D) != MFA_OK || check_sizes(B, Hkv, Nk, D) != MFA_OK) return 0;
  return host_layout(B, Hq, Hkv, Nq, Nk, D).total;
}

extern "C" int mfa_fwd_host(const void* q, const void* k, const void* v, void* out, float* lse,
                            int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale, int causal,
                            int win_l, int win_r, float softcap, int dtype, void* scratch,
                            size_t scratch_bytes, void* stream) {
  int rc = validate_fwd_common(Hq, Hkv, D, dtype, win_l, win_r, softcap, scale);
  if (rc != MFA_OK) return rc;
  if (B < 0 || Nq < 0 || Nk < 0) return MFA_ERR_BAD_SHAPE;
  if ((rc = check_sizes(B, Hq, Nq, D)) != MFA_OK) return rc;
  if ((rc = check_sizes(B, Hkv, Nk, D)) != MFA_OK) return rc;
  if ((long long)B * Hq > 0x7FFFFFFFLL || (long long)B * Hkv > 0x7FFFFFFFLL) return MFA_ERR_BAD_SHAPE;
  if (B == 0 || Hq == 0 || Nq == 0) return MFA_OK;
  if (!q || !out || (Nk > 0 && (!k || !v))) return MFA_ERR_NULL_POINTER;
  const HostLayout L = host_layout(B, Hq, Hkv, Nq, Nk, D);
  if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 255u) || scratch_bytes < L.total)
    return MFA_ERR_WORKSPACE;
  const int dev = current_device();
  if (dev < 0) return MFA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_host_mutex[dev]);
  HostPipe& hp = g_host_pipe[dev];
  if (!host_pipe_init(hp)) return MFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* s = static_cast<char*>(scratch);
  const int G = Hq / Hkv;
  const long long units = (long long)B * Hkv;
  // runs of about 12 MiB of input each (at most kHostChunks): every copy has a fixed cost, and
  // the last run's kernel and copy out are not hidden, so a few large runs beat many small ones
  const long long in_bytes = (long long)(L.q_bytes + 2 * L.kv_bytes);
  const int n_chunks = (int)std::max<long long>(
      1, std::min<long long>(units, std::min<long long>(kHostChunks, in_bytes / (12ll << 20))));
  const size_t q_unit = (size_t)G * Nq * D * 2, kv_unit = (size_t)Nk * D * 2;
  const size_t l_unit = (size_t)G * Nq * sizeof(float);
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // earlier work on the caller's stream (which may still use the scratch) precedes the copies in
  if (!ok(cudaEventRecord(hp.entry, st)) || !ok(cudaStreamWaitEvent(hp.in, hp.entry, 0))) return MFA_ERR_CUDA;
  rc = MFA_OK;
  for (int c = 0; c < n_chunks && rc == MFA_OK; ++c) {
    const long long u0 = units * c / n_chunks, u1 = units * (c + 1) / n_chunks;
    const size_t n = (size_t)(u1 - u0);
    const size_t oq = (size_t)u0 * q_unit, okv = (size_t)u0 * kv_unit, ol = (size_t)u0 * l_unit;
    if (!ok(cudaMemcpyAsync(s + oq, static_cast<const char*>(q) + oq, n * q_unit,
                            cudaMemcpyHostToDevice, hp.in)) ||
        (Nk > 0 && !ok(cudaMemcpyAsync(s + L.off_k + okv, static_cast<const char*>(k) + okv,
                                       n * kv_unit, cudaMemcpyHostToDevice, hp.in))) ||
        (Nk > 0 && !ok(cudaMemcpyAsync(s + L.off_v + okv, static_cast<const char*>(v) + okv,
                                       n * kv_unit, cudaMemcpyHostToDevice, hp.in))) ||
        !ok(cudaEventRecord(hp.in_done[c], hp.in)) || !ok(cudaStreamWaitEvent(st, hp.in_done[c], 0))) {
      rc = MFA_ERR_CUDA;
      break;
    }
    rc = mfa_fwd(s + oq, s + L.off_k + okv, s + L.off_v + okv, s + L.off_out + oq,
                 lse ? reinterpret_cast<float*>(s + L.off_lse + ol) : nullptr, (int)n, G, 1, Nq, Nk,
                 D, scale, causal, win_l, win_r, softcap, dtype, stream);
    if (rc != MFA_OK) break;
    if (!ok(cudaEventRecord(hp.comp_done[c], st)) || !ok(cudaStreamWaitEvent(hp.out, hp.comp_done[c], 0)) ||
        !ok(cudaMemcpyAsync(static_cast<char*>(out) + oq, s + L.off_out + oq, n * q_unit,
                            cudaMemcpyDeviceToHost, hp.out)) ||
        (lse && !ok(cudaMemcpyAsync(reinterpret_cast<char*>(lse) + ol, s + L.off_lse + ol, n * l_unit,
                                    cudaMemcpyDeviceToHost, hp.out))))
      rc = MFA_ERR_CUDA;
  }
  // the caller's stream (and so the next call) continues after the last copy out, also on error
  if (!ok(cudaEventRecord(hp.done, hp.out)) || !ok(cudaStreamWaitEvent(st, hp.done, 0))) return MFA_ERR_CUDA;
  return rc;
}
