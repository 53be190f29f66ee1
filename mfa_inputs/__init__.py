"""Seeded synthetic inputs for exact tiled attention (prefill and paged split-KV decode).

This module is shared by the parity tests, the bench and the oracle driver. It holds no
attention arithmetic: it draws numbers (SplitMix64 + Box-Muller, see gen.c), rounds them to
the storage dtype and lays them out in the shapes the workloads use. The 16-bit bit patterns
it returns are the inputs; the CUDA path uploads them unchanged and the oracle widens them
exactly to fp64.

Stream numbering per workload: q=0, k=1, v=2, sequence lengths=3, page permutation=4.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libmfa_inputs.so")
_SRC = os.path.join(_HERE, "gen.c")

FP16, BF16 = 0, 1
DTYPE_NAMES = {FP16: "fp16", BF16: "bf16"}
STREAM_Q, STREAM_K, STREAM_V, STREAM_LENS, STREAM_PERM, STREAM_KEXTRA, STREAM_MASK = 0, 1, 2, 3, 4, 5, 6
SPARSE_BLOCK = 128  # query rows x keys per block-mask entry (the forward kernel's tile)
PAGE_SIZE = 16


def build() -> str:
    """Compile gen.c into libmfa_inputs.so (gcc, OpenMP)."""
    if (not os.path.exists(_SO)) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _SO, _SRC, "-lm"])
    return _SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.mfa_gen_draw.restype = ctypes.c_uint64
        lib.mfa_gen_draw.argtypes = [ctypes.c_uint64] * 3
        lib.mfa_gen_u64.restype = None
        lib.mfa_gen_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                    ctypes.c_int64, ctypes.c_void_p]
        lib.mfa_gen_normal.restype = None
        lib.mfa_gen_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                       ctypes.c_int64, ctypes.c_double, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_void_p]
        lib.mfa_gen_widen.restype = None
        lib.mfa_gen_widen.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
        _lib = lib
    return _lib


def draws_u64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    if n:
        _load().mfa_gen_u64(seed, stream, offset, n, out.ctypes.data)
    return out


def normal_bits(seed: int, stream: int, shape, dtype: int, mul: float = 1.0,
                offset: int = 0) -> np.ndarray:
    """N(0,1)*mul values rounded to fp16/bf16, returned as uint16 bit patterns of `shape`."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load().mfa_gen_normal(seed, stream, offset, n, mul, dtype, out.ctypes.data, None)
    return out.reshape(shape)


def normal_f64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    """The unrounded fp64 normals (used to check the generator's distribution)."""
    out = np.empty(n, dtype=np.float64)
    if n:
        _load().mfa_gen_normal(seed, stream, offset, n, 1.0, 2, None, out.ctypes.data)
    return out


def widen(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Exact fp64 values of fp16/bf16 bit patterns."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    if bits.size:
        _load().mfa_gen_widen(bits.ctypes.data, bits.size, dtype, out.ctypes.data)
    return out


def uniform_ints(seed: int, stream: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers uniform on [lo, hi] inclusive (multiply-high of the top 32 bits)."""
    d = draws_u64(seed, stream, n) >> np.uint64(32)
    span = np.uint64(hi - lo + 1)
    return (np.int64(lo) + ((d * span) >> np.uint64(32)).astype(np.int64)).astype(np.int64)


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    """Fisher-Yates shuffle of [0, n): step k (k = 0..n-2) swaps i = n-1-k with j uniform on [0, i]."""
    perm = np.arange(n, dtype=np.int64)
    if n < 2:
        return perm
    d = draws_u64(seed, stream, n - 1) >> np.uint64(32)
    i_vals = np.arange(n - 1, 0, -1, dtype=np.uint64)
    j_vals = ((d * (i_vals + np.uint64(1))) >> np.uint64(32)).astype(np.int64)
    for k in range(n - 1):
        i = n - 1 - k
        j = j_vals[k]
        perm[i], perm[j] = perm[j], perm[i]
    return perm


NAN_BITS = {FP16: 0x7E00, BF16: 0x7FC0}


@dataclass
class PrefillCase:
    """Shapes and flags of one dense forward workload; q [B,Hq,Nq,D], k/v [B,Hkv,Nk,D]."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    D: int
    dtype: int
    causal: bool
    win_l: int = -1
    win_r: int = -1
    softcap: float = 0.0
    mul: float = 1.0
    seed: int = 1
    scale: float | None = None

    def scale_f32(self) -> float:
        s = self.scale if self.scale is not None else 1.0 / np.sqrt(self.D)
        return float(np.float32(s))

    def dout(self):
        """The output gradient dO for the backward, [B,Hq,Nq,D] bit patterns: N(0,1) from seed + 500
        (stream 0)."""
        return normal_bits(self.seed + 500, STREAM_Q, (self.B, self.Hq, self.Nq, self.D), self.dtype)

    def tensors(self):
        """(q, k, v) as uint16 bit patterns."""
        return self.batch_slice_tensors(0)

    def batch_slice_tensors(self, index: int):
        """(q, k, v) of batch rows [index * B, (index + 1) * B) of the same workload with a batch
        of any larger multiple of B: the draws continue the streams at those rows' offsets, so
        the slices of consecutive indices are pieces of one larger seeded problem (index 0 is
        tensors())."""
        qn = self.B * self.Hq * self.Nq * self.D
        kn = self.B * self.Hkv * self.Nk * self.D
        q = normal_bits(self.seed, STREAM_Q, (self.B, self.Hq, self.Nq, self.D), self.dtype, self.mul,
                        offset=index * qn)
        k = normal_bits(self.seed, STREAM_K, (self.B, self.Hkv, self.Nk, self.D), self.dtype, self.mul,
                        offset=index * kn)
        v = normal_bits(self.seed, STREAM_V, (self.B, self.Hkv, self.Nk, self.D), self.dtype, self.mul,
                        offset=index * kn)
        return q, k, v


@dataclass
class DecodeCase:
    """Paged split-KV decode workload.

    q [B,Hq,Nq,D]; k/v pages [num_pages, 16, Hkv, D]; block_table int32 [B, max_pages];
    seq_lens int32 [B]. Pages are handed out in the order of a seeded permutation of
    [0, num_pages); table entries past a sequence's last page are -1; page slots at or past
    the sequence length are filled with NaN so that any read of them shows up in the output.
    """
    name: str
    B: int
    Nq: int
    Hq: int
    Hkv: int
    D: int
    dtype: int
    len_lo: int
    len_hi: int
    causal: bool = True
    softcap: float = 0.0
    seed: int = 1
    max_pages: int | None = None
    fixed_lens: list | None = None
    scale: float | None = None
    extra_pages: int = 0
    permute: bool = True
    win_l: int = -1
    _cache: dict = field(default_factory=dict, repr=False)

    def scale_f32(self) -> float:
        s = self.scale if self.scale is not None else 1.0 / np.sqrt(self.D)
        return float(np.float32(s))

    def seq_lens(self) -> np.ndarray:
        if self.fixed_lens is not None:
            return np.asarray(self.fixed_lens, dtype=np.int32)
        return uniform_ints(self.seed, STREAM_LENS, self.B, self.len_lo, self.len_hi).astype(np.int32)

    def max_pages_per_seq(self) -> int:
        if self.max_pages is not None:
            return self.max_pages
        return max(1, -(-self.len_hi // PAGE_SIZE))

    def layout(self):
        """(seq_lens, block_table, num_pages)."""
        lens = self.seq_lens()
        npg = [-(-int(L) // PAGE_SIZE) for L in lens]
        num_pages = int(sum(npg)) + self.extra_pages
        if self.permute:
            perm = permutation(self.seed, STREAM_PERM, num_pages)
        else:
            perm = np.arange(num_pages, dtype=np.int64)
        mp = self.max_pages_per_seq()
        table = np.full((self.B, mp), -1, dtype=np.int32)
        off = 0
        for b in range(self.B):
            table[b, :npg[b]] = perm[off:off + npg[b]]
            off += npg[b]
        return lens, table, max(num_pages, 1)

    def tensors(self):
        """(q, k_pages, v_pages, block_table, seq_lens) with q/k/v as uint16 bit patterns."""
        lens, table, num_pages = self.layout()
        q = normal_bits(self.seed, STREAM_Q, (self.B, self.Hq, self.Nq, self.D), self.dtype)
        shape = (num_pages, PAGE_SIZE, self.Hkv, self.D)
        k = normal_bits(self.seed, STREAM_K, shape, self.dtype)
        v = normal_bits(self.seed, STREAM_V, shape, self.dtype)
        nan = np.uint16(NAN_BITS[self.dtype])
        used = np.zeros(num_pages, dtype=bool)
        for b in range(self.B):
            L = int(lens[b])
            n = -(-L // PAGE_SIZE)
            used[table[b, :n]] = True
            if L % PAGE_SIZE:
                last = table[b, n - 1]
                k[last, L % PAGE_SIZE:] = nan
                v[last, L % PAGE_SIZE:] = nan
        k[~used] = nan
        v[~used] = nan
        return q, k, v, table, lens


@dataclass
class VarlenCase:
    """Packed variable-length prefill: B sequences in one tensor.

    q [total_q, Hq, D], k/v [total_k, Hkv, D]; cu_seqlens_q / cu_seqlens_k int32 [B + 1].
    Query lengths are uniform integers on [len_lo, len_hi] (stream 3); each key length is its
    query length plus a uniform integer on [0, k_extra] (stream 5), the shape of a chunked
    prefill that continues a cached prefix. fixed_q / fixed_k give the lengths explicitly.
    """
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: int
    causal: bool
    len_lo: int = 1
    len_hi: int = 1
    k_extra: int = 0
    win_l: int = -1
    win_r: int = -1
    softcap: float = 0.0
    mul: float = 1.0
    seed: int = 1
    fixed_q: list | None = None
    fixed_k: list | None = None
    scale: float | None = None

    def scale_f32(self) -> float:
        s = self.scale if self.scale is not None else 1.0 / np.sqrt(self.D)
        return float(np.float32(s))

    def lens(self):
        """(query lengths, key lengths), int32 [B] each."""
        if self.fixed_q is not None:
            nq = np.asarray(self.fixed_q, dtype=np.int32)
        else:
            nq = uniform_ints(self.seed, STREAM_LENS, self.B, self.len_lo, self.len_hi).astype(np.int32)
        if self.fixed_k is not None:
            nk = np.asarray(self.fixed_k, dtype=np.int32)
        elif self.k_extra > 0:
            nk = nq + uniform_ints(self.seed, STREAM_KEXTRA, self.B, 0, self.k_extra).astype(np.int32)
        else:
            nk = nq.copy()
        return nq, nk

    def cu_seqlens(self):
        """(cu_seqlens_q, cu_seqlens_k), int32 [B + 1] each, starting at 0."""
        nq, nk = self.lens()
        cq = np.zeros(self.B + 1, dtype=np.int32)
        ck = np.zeros(self.B + 1, dtype=np.int32)
        cq[1:] = np.cumsum(nq)
        ck[1:] = np.cumsum(nk)
        return cq, ck

    def tensors(self):
        """(q, k, v) as uint16 bit patterns in the packed layout."""
        cq, ck = self.cu_seqlens()
        q = normal_bits(self.seed, STREAM_Q, (int(cq[-1]), self.Hq, self.D), self.dtype, self.mul)
        k = normal_bits(self.seed, STREAM_K, (int(ck[-1]), self.Hkv, self.D), self.dtype, self.mul)
        v = normal_bits(self.seed, STREAM_V, (int(ck[-1]), self.Hkv, self.D), self.dtype, self.mul)
        return q, k, v


@dataclass
class SparseCase:
    """Block-sparse prefill: dense q [B,Hq,N,D], k/v [B,Hkv,N,D] and a block mask uint8
    [B, Hq, nb, nb] (nb = ceil(N / 128)); a zero entry removes a 128 x 128 block of (query rows,
    keys) from the visible set.

    pattern "spatial2d": the N tokens are grid[0] x grid[1] blocks of 128 on a 2-D grid in
    row-major order, and block (r1, c1) attends block (r2, c2) iff max(|r1 - r2|, |c1 - c2|) <=
    radius (a local neighbourhood, as in the pages' spatial 2-D masks); the same for every head.
    pattern "random": every entry is on with probability density (stream 6, per batch and head),
    and the diagonal blocks are always on.
    """
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    dtype: int
    causal: bool
    pattern: str = "random"
    density: float = 0.3
    grid: tuple = (1, 1)
    radius: int = 1
    win_l: int = -1
    win_r: int = -1
    softcap: float = 0.0
    mul: float = 1.0
    seed: int = 1
    scale: float | None = None

    @property
    def Nq(self):
        return self.N

    @property
    def Nk(self):
        return self.N

    def scale_f32(self) -> float:
        s = self.scale if self.scale is not None else 1.0 / np.sqrt(self.D)
        return float(np.float32(s))

    def block_mask(self) -> np.ndarray:
        nb = -(-self.N // SPARSE_BLOCK)
        if self.pattern == "spatial2d":
            gh, gw = self.grid
            assert gh * gw == nb, "grid must tile the sequence in 128-token blocks"
            r, c = np.divmod(np.arange(nb), gw)
            m = (np.maximum(np.abs(r[:, None] - r[None, :]), np.abs(c[:, None] - c[None, :]))
                 <= self.radius).astype(np.uint8)
            return np.broadcast_to(m, (self.B, self.Hq, nb, nb)).copy()
        u = uniform_ints(self.seed, STREAM_MASK, self.B * self.Hq * nb * nb, 0, 999)
        m = (u.reshape(self.B, self.Hq, nb, nb) < int(round(self.density * 1000))).astype(np.uint8)
        m[:, :, np.arange(nb), np.arange(nb)] = 1
        return m

    def tensors(self):
        """(q, k, v) as uint16 bit patterns and the block mask."""
        q = normal_bits(self.seed, STREAM_Q, (self.B, self.Hq, self.N, self.D), self.dtype, self.mul)
        k = normal_bits(self.seed, STREAM_K, (self.B, self.Hkv, self.N, self.D), self.dtype, self.mul)
        v = normal_bits(self.seed, STREAM_V, (self.B, self.Hkv, self.N, self.D), self.dtype, self.mul)
        return q, k, v, self.block_mask()


@dataclass
class PagedPrefillCase:
    """Chunked prefill over a paged cache: B sequences with seq_lens uniform on [len_lo, len_hi]
    (or fixed_lens) keys in a page pool laid out, permuted and NaN-poisoned exactly as a
    DecodeCase with the same seed; each sequence contributes its last Nq_b positions as packed
    query rows, Nq_b uniform on [1, min(len_b, q_hi)] (stream 5) or fixed_q."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: int
    len_lo: int
    len_hi: int
    q_hi: int = 256
    causal: bool = True
    win_l: int = -1
    win_r: int = -1
    softcap: float = 0.0
    seed: int = 1
    fixed_lens: list | None = None
    fixed_q: list | None = None
    scale: float | None = None

    def scale_f32(self) -> float:
        s = self.scale if self.scale is not None else 1.0 / np.sqrt(self.D)
        return float(np.float32(s))

    def _pool(self) -> "DecodeCase":
        hi = max(self.fixed_lens) if self.fixed_lens is not None else self.len_hi
        return DecodeCase(self.name, self.B, 1, self.Hq, self.Hkv, self.D, self.dtype, self.len_lo,
                          max(int(hi), 1), seed=self.seed, fixed_lens=self.fixed_lens)

    def chunk_lens(self, lens) -> np.ndarray:
        if self.fixed_q is not None:
            return np.asarray(self.fixed_q, dtype=np.int32)
        u = uniform_ints(self.seed, STREAM_KEXTRA, self.B, 0, 1 << 20)
        cap = np.maximum(1, np.minimum(lens.astype(np.int64), self.q_hi))
        return (1 + u % cap).astype(np.int32)

    def tensors(self):
        """(q packed bits, k_pages, v_pages, block_table, seq_lens, cu_seqlens_q)."""
        _, kp, vp, table, lens = self._pool().tensors()
        nq = self.chunk_lens(lens)
        cq = np.zeros(self.B + 1, dtype=np.int32)
        cq[1:] = np.cumsum(nq)
        q = normal_bits(self.seed, STREAM_Q, (int(cq[-1]), self.Hq, self.D), self.dtype)
        return q, kp, vp, table, lens, cq


def workloads():
    """The named full-size workloads (shapes, flags, seeds and value scales)."""
    return {
        "causal_b1_h2_n128_d64_fp16": PrefillCase(
            "causal_b1_h2_n128_d64_fp16", 1, 2, 2, 128, 128, 64, FP16, True, seed=1001),
        "causal_b2_h8_n4096_d128_fp16": PrefillCase(
            "causal_b2_h8_n4096_d128_fp16", 2, 8, 8, 4096, 4096, 128, FP16, True, seed=1002),
        "noncausal_b2_h8_n4096_d128_fp16": PrefillCase(
            "noncausal_b2_h8_n4096_d128_fp16", 2, 8, 8, 4096, 4096, 128, FP16, False, seed=1002),
        # the causal shape of the window workloads (and their inputs), without a window
        "causal_b2_h8_n8192_d128_fp16": PrefillCase(
            "causal_b2_h8_n8192_d128_fp16", 2, 8, 8, 8192, 8192, 128, FP16, True, seed=1003),
        "window512_b2_h8_n8192_d128_fp16": PrefillCase(
            "window512_b2_h8_n8192_d128_fp16", 2, 8, 8, 8192, 8192, 128, FP16, True, 512, 0,
            seed=1003),
        "window256_b2_h8_n8192_d128_fp16": PrefillCase(
            "window256_b2_h8_n8192_d128_fp16", 2, 8, 8, 8192, 8192, 128, FP16, True, 256, 0,
            seed=1003),
        "gqa_causal_b1_hq32_hkv8_n16384_d128_bf16_cap50": PrefillCase(
            "gqa_causal_b1_hq32_hkv8_n16384_d128_bf16_cap50", 1, 32, 8, 16384, 16384, 128, BF16,
            True, softcap=50.0, mul=0.5, seed=1004),
        "varlen_causal_b8_h8_d128_fp16_len512_8k": VarlenCase(
            "varlen_causal_b8_h8_d128_fp16_len512_8k", 8, 8, 8, 128, FP16, True, 512, 8192,
            seed=1006),
        "sparse_spatial2d_b1_h16_n16384_d128_fp16": SparseCase(
            "sparse_spatial2d_b1_h16_n16384_d128_fp16", 1, 16, 16, 16384, 128, FP16, False,
            pattern="spatial2d", grid=(16, 8), radius=2, seed=1007),
        "paged_prefill_b8_hq32_hkv8_d128_bf16_ctx4k_32k": PagedPrefillCase(
            "paged_prefill_b8_hq32_hkv8_d128_bf16_ctx4k_32k", 8, 32, 8, 128, BF16, 4096, 32768,
            q_hi=2048, seed=1008),
        "decode_b8_hq32_hkv8_d128_bf16_len8k_128k": DecodeCase(
            "decode_b8_hq32_hkv8_d128_bf16_len8k_128k", 8, 1, 32, 8, 128, BF16, 8192, 131072,
            seed=1005),
        # speculative-decoding verify: 4 draft tokens per sequence against the same caches
        "decode_verify_nq4_b8_hq32_hkv8_d128_bf16_len8k_128k": DecodeCase(
            "decode_verify_nq4_b8_hq32_hkv8_d128_bf16_len8k_128k", 8, 4, 32, 8, 128, BF16, 8192,
            131072, seed=1005),
        # D = 256 heads (two kv heads per phase-1 CTA)
        "decode_b8_hq16_hkv8_d256_bf16_len4k_32k": DecodeCase(
            "decode_b8_hq16_hkv8_d256_bf16_len4k_32k", 8, 1, 16, 8, 256, BF16, 4096, 32768,
            seed=1009),
        # the same cache lengths under a 4096-token left window (each query sees 4096 keys)
        "decode_window4k_b8_hq32_hkv8_d128_bf16_len8k_128k": DecodeCase(
            "decode_window4k_b8_hq32_hkv8_d128_bf16_len8k_128k", 8, 1, 32, 8, 128, BF16, 8192,
            131072, win_l=4095, seed=1005),
    }
