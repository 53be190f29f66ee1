"""Python binding of libmfa.so: exact tiled attention (prefill + paged split-KV decode) on B200.

Argument marshalling only: every step of the computation runs in the CUDA kernels behind the C
ABI declared in include/mfa.h. PyTorch provides device memory and the stream. There is no CPU
or library fallback: importing this package fails if libmfa.so has not been built, and every
call raises if the library rejects its arguments.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmfa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it first (python tiled_exact_attention_mfa_b200/build.py "
        "or __graft_entry__.build()). There is no fallback implementation.")

lib = ctypes.CDLL(LIB_PATH)

MFA_DTYPE_FP16 = 0
MFA_DTYPE_BF16 = 1
MFA_DEBUG_NO_TILE_SKIP = 1
MFA_DEBUG_COUNT_TILES = 2
MFA_DEBUG_WITHHOLD_MMA = 4

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

lib.mfa_fwd.restype = _i
lib.mfa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _i, _f, _i, _vp]
lib.mfa_fwd_varlen.restype = _i
lib.mfa_fwd_varlen.argtypes = [_vp] * 7 + [_i] * 7 + [_f, _i, _i, _i, _f, _i, _vp]
lib.mfa_fwd_blocksparse.restype = _i
lib.mfa_fwd_blocksparse.argtypes = [_vp] * 6 + [_i] * 6 + [_f, _i, _i, _i, _f, _i, _vp]
lib.mfa_bwd_workspace_size.restype = ctypes.c_size_t
lib.mfa_bwd_workspace_size.argtypes = [_i, _i, _i]
lib.mfa_bwd.restype = _i
lib.mfa_bwd.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _i, _i, _i, _f, _i, _vp, ctypes.c_size_t, _vp]
lib.mfa_fwd_paged.restype = _i
lib.mfa_fwd_paged.argtypes = [_vp] * 8 + [_i] * 9 + [_f, _i, _i, _i, _f, _i, _vp]
lib.mfa_decode_workspace_size.restype = ctypes.c_size_t
lib.mfa_decode_workspace_size.argtypes = [_i] * 7
lib.mfa_decode_plan.restype = _i
lib.mfa_decode_plan.argtypes = [_i] * 8 + [ctypes.POINTER(ctypes.c_int)] * 3
lib.mfa_decode_splitkv.restype = _i
lib.mfa_decode_splitkv.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                   _f, _i, _f, _i, _vp, ctypes.c_size_t, _vp]
lib.mfa_decode_splitkv_window.restype = _i
lib.mfa_decode_splitkv_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                          _i, _i, _f, _i, _i, _f, _i, _vp, ctypes.c_size_t, _vp]
lib.mfa_decode_phase1.restype = _i
lib.mfa_decode_phase1.argtypes = [_vp] * 5 + [_i] * 8 + [_f, _i, _i, _f, _i, _i, _i, _vp, _vp, _i, _vp]
lib.mfa_decode_combine.restype = _i
lib.mfa_decode_combine.argtypes = [_vp] * 3 + [_i] * 9 + [_vp, _vp, _i, _vp]
lib.mfa_fwd_host_scratch_size.restype = ctypes.c_size_t
lib.mfa_fwd_host_scratch_size.argtypes = [_i] * 6
lib.mfa_fwd_host.restype = _i
lib.mfa_fwd_host.argtypes = [_vp] * 5 + [_i] * 6 + [_f, _i, _i, _i, _f, _i, _vp, ctypes.c_size_t, _vp]
lib.mfa_decode_splitkv_noalloc.restype = _i
lib.mfa_decode_splitkv_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                           _i, _i, _f, _i, _f, _i, _vp]
MFA_NOALLOC_SCRATCH_BYTES = 64 << 20
lib.mfa_status_string.restype = ctypes.c_char_p
lib.mfa_status_string.argtypes = [_i]


class LaunchInfo(ctypes.Structure):
    _fields_ = [(n, _i) for n in (
        "kernel", "grid_x", "grid_y", "grid_z", "block_threads", "smem_bytes", "tile_m", "tile_n",
        "q_tiles_per_cta", "pages_per_split", "max_splits", "kv_heads_per_cta")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


lib.mfa_last_launch_info.restype = _i
lib.mfa_last_launch_info.argtypes = [ctypes.POINTER(LaunchInfo)]
lib.mfa_device_status.restype = _i
lib.mfa_device_status.argtypes = [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i)]
lib.mfa_debug_set_flags.restype = _i
lib.mfa_debug_set_flags.argtypes = [_i]
lib.mfa_debug_tiles_visited.restype = _i
lib.mfa_debug_tiles_visited.argtypes = [_vp, ctypes.POINTER(ctypes.c_ulonglong)]
lib.mfa_debug_tmap_stats.restype = _i
lib.mfa_debug_tmap_stats.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)] * 2
lib.mfa_debug_tmap_probe.restype = _i
lib.mfa_debug_tmap_probe.argtypes = [_vp, _i, _i, ctypes.c_longlong, ctypes.c_longlong, _i,
                                     ctypes.POINTER(_i)]
lib.mfa_debug_set_decode_split_pages.restype = _i
lib.mfa_debug_set_decode_split_pages.argtypes = [_i]

EXPORTED = ("mfa_fwd", "mfa_fwd_varlen", "mfa_fwd_blocksparse", "mfa_fwd_paged", "mfa_bwd_workspace_size", "mfa_bwd",
            "mfa_decode_workspace_size", "mfa_decode_plan", "mfa_decode_splitkv_window", "mfa_decode_splitkv", "mfa_status_string",
            "mfa_last_launch_info", "mfa_device_status", "mfa_debug_set_flags",
            "mfa_debug_tiles_visited", "mfa_debug_set_decode_split_pages",
            "mfa_decode_splitkv_noalloc", "mfa_fwd_host_scratch_size", "mfa_fwd_host",
            "mfa_debug_tmap_stats", "mfa_debug_tmap_probe", "mfa_decode_phase1",
            "mfa_decode_combine")


class MFAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {mfa_status_string(code)} (status {code})")


def mfa_status_string(code: int) -> str:
    return lib.mfa_status_string(code).decode()


def _check(rc: int, where: str):
    if rc != 0:
        raise MFAError(rc, where)


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return MFA_DTYPE_FP16
    if t.dtype == torch.bfloat16:
        return MFA_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float16 or bfloat16")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def mfa_fwd(q, k, v, out=None, lse=None, *, scale=None, causal=False, window=(-1, -1),
            softcap=0.0, return_lse=True, stream=None):
    """Attention forward. q [B,Hq,Nq,D], k/v [B,Hkv,Nk,D]; returns (out, lse or None)."""
    torch = _torch()
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k and v must be [B, Hkv, Nk, D] matching q")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    wl, wr = window
    rc = lib.mfa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Nq, Nk, D,
                     float(scale), int(bool(causal)), int(wl), int(wr), float(softcap),
                     _dtype_code(q), _stream(stream))
    _check(rc, "mfa_fwd")
    return out, lse


def _host_ptr(t):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("mfa_fwd_host takes host (CPU) tensors")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def mfa_fwd_host_scratch_size(B, Hq, Hkv, Nq, Nk, D) -> int:
    return int(lib.mfa_fwd_host_scratch_size(B, Hq, Hkv, Nq, Nk, D))


def mfa_fwd_host(q, k, v, out=None, lse=None, *, scale=None, causal=False, window=(-1, -1),
                 softcap=0.0, scratch=None, return_lse=True, stream=None):
    """Attention forward over HOST tensors (pinned memory lets the copies overlap): q
    [B,Hq,Nq,D], k/v [B,Hkv,Nk,D] on the CPU; the copies to and from the device and the kernels
    are queued on `stream` and two internal copy streams. Returns (out, lse or None) as CPU
    tensors, complete once `stream` has reached this point (synchronize before reading them).
    scratch: a CUDA uint8 tensor of mfa_fwd_host_scratch_size(...) bytes (allocated if None)."""
    torch = _torch()
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k and v must be [B, Hkv, Nk, D] matching q")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32).pin_memory()
    if scratch is None:
        n = mfa_fwd_host_scratch_size(B, Hq, Hkv, Nq, Nk, D)
        scratch = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    wl, wr = window
    rc = lib.mfa_fwd_host(_host_ptr(q), _host_ptr(k), _host_ptr(v), _host_ptr(out), _host_ptr(lse),
                          B, Hq, Hkv, Nq, Nk, D, float(scale), int(bool(causal)), int(wl), int(wr),
                          float(softcap), _dtype_code(q), _ptr(scratch),
                          scratch.numel() * scratch.element_size(), _stream(stream))
    _check(rc, "mfa_fwd_host")
    return out, lse


def mfa_decode_workspace_size(B, Nq, Hq, Hkv, D, max_pages_per_seq, page_size=16) -> int:
    return int(lib.mfa_decode_workspace_size(B, Nq, Hq, Hkv, D, max_pages_per_seq, page_size))


def mfa_decode_plan(B, Nq, Hq, Hkv, D, max_pages_per_seq, page_size=16, win_l=-1) -> dict:
    """The decode split plan for this shape (host only, no launch): pages per split, splits per
    sequence and kv heads per phase-1 CTA."""
    s, n, h = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib.mfa_decode_plan(B, Nq, Hq, Hkv, D, max_pages_per_seq, page_size, win_l,
                               ctypes.byref(s), ctypes.byref(n), ctypes.byref(h)), "mfa_decode_plan")
    return {"pages_per_split": s.value, "max_splits": n.value, "kv_heads_per_cta": h.value}


def mfa_decode_splitkv(q, k_pages, v_pages, block_table, seq_lens, out=None, lse=None, *,
                       scale=None, causal=True, softcap=0.0, workspace=None, return_lse=True,
                       win_l=-1, stream=None):
    """Paged split-KV decode. q [B,Hq,Nq,D]; pages [num_pages,16,Hkv,D]; block_table int32
    [B,max_pages]; seq_lens int32 [B]. win_l >= 0 adds a left window
    (mfa_decode_splitkv_window). Returns (out, lse or None)."""
    torch = _torch()
    B, Hq, Nq, D = q.shape
    num_pages, page, Hkv, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_table and seq_lens must be int32")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    need = mfa_decode_workspace_size(B, Nq, Hq, Hkv, D, max_pages, page)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if win_l == -1:
        rc = lib.mfa_decode_splitkv(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                    _ptr(seq_lens), _ptr(out), _ptr(lse), B, Nq, Hq, Hkv, D, page,
                                    max_pages, num_pages, float(scale), int(bool(causal)),
                                    float(softcap), _dtype_code(q), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
        _check(rc, "mfa_decode_splitkv")
    else:
        rc = lib.mfa_decode_splitkv_window(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                           _ptr(seq_lens), _ptr(out), _ptr(lse), B, Nq, Hq, Hkv, D,
                                           page, max_pages, num_pages, float(scale),
                                           int(bool(causal)), int(win_l), float(softcap),
                                           _dtype_code(q), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream))
        _check(rc, "mfa_decode_splitkv_window")
    return out, lse


def mfa_decode_splitkv_noalloc(q, k_pages, v_pages, block_table, seq_lens, out, lse=None, *,
                               scale=None, causal=True, softcap=0.0, stream=None):
    """mfa_decode_splitkv without a caller workspace, for callers that cannot allocate device
    memory when decode runs (an engine that has handed all of HBM to its KV page pool, code inside
    an allocator callback). The workspace is the library's fixed 64 MiB device array; calls that
    overlap on the GPU race on it, so keep them on one stream.

    This wrapper allocates nothing either: the caller passes `out` (like q) and, if it wants the
    log-sum-exp, `lse` (fp32 [B, Hq, Nq]; None skips it). Returns (out, lse)."""
    torch = _torch()
    B, Hq, Nq, D = q.shape
    num_pages, page, Hkv, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_table and seq_lens must be int32")
    if out is None:
        raise ValueError("mfa_decode_splitkv_noalloc allocates nothing: pass `out`")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rc = lib.mfa_decode_splitkv_noalloc(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                        _ptr(seq_lens), _ptr(out), _ptr(lse), B, Nq, Hq, Hkv, D,
                                        page, max_pages, num_pages, float(scale),
                                        int(bool(causal)), float(softcap), _dtype_code(q),
                                        _stream(stream))
    _check(rc, "mfa_decode_splitkv_noalloc")
    return out, lse


def _check_partials(part_o, part_ml, D):
    torch = _torch()
    if part_o.dtype != torch.float32 or part_ml.dtype != torch.float32:
        raise TypeError("partial buffers must be float32")
    if part_o.dim() != 4 or part_ml.dim() != 4 or part_o.shape[3] != D or part_ml.shape[3] != 2 \
            or part_o.shape[:3] != part_ml.shape[:3]:
        raise ValueError("partials must be [splits, B, Hq*Nq, D] and [splits, B, Hq*Nq, 2]")
    return part_o.shape[0]


def mfa_decode_phase1(q, k_pages, v_pages, block_table, seq_lens, part_o, part_ml, split_lo,
                      split_hi, *, scale=None, causal=True, softcap=0.0, win_l=-1, stream=None):
    """Phase 1 of the split-KV decode for splits [split_lo, split_hi) of every sequence, into
    the split-major partial buffers part_o [cap, B, Hq*Nq, D] / part_ml [cap, B, Hq*Nq, 2]."""
    torch = _torch()
    B, Hq, Nq, D = q.shape
    num_pages, page, Hkv, _ = k_pages.shape
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_table and seq_lens must be int32")
    cap = _check_partials(part_o, part_ml, D)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rc = lib.mfa_decode_phase1(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                               _ptr(seq_lens), B, Nq, Hq, Hkv, D, page, block_table.shape[1],
                               num_pages, float(scale), int(bool(causal)), int(win_l),
                               float(softcap), _dtype_code(q), int(split_lo), int(split_hi),
                               _ptr(part_o), _ptr(part_ml), cap, _stream(stream))
    _check(rc, "mfa_decode_phase1")


def mfa_decode_combine(seq_lens, part_o, part_ml, out, lse=None, *, Hkv, max_pages_per_seq,
                       win_l=-1, stream=None):
    """The combine of the split-KV decode over every split's partials, into out [B, Hq, Nq, D]
    (and lse [B, Hq, Nq] fp32 unless None). Hkv and max_pages_per_seq fix the split plan."""
    B, Hq, Nq, D = out.shape
    cap = _check_partials(part_o, part_ml, D)
    rc = lib.mfa_decode_combine(_ptr(seq_lens), _ptr(out), _ptr(lse), B, Nq, Hq, int(Hkv), D, 16,
                                int(max_pages_per_seq), int(win_l), _dtype_code(out),
                                _ptr(part_o), _ptr(part_ml), cap, _stream(stream))
    _check(rc, "mfa_decode_combine")
    return out, lse


def mfa_last_launch_info() -> dict:
    info = LaunchInfo()
    _check(lib.mfa_last_launch_info(ctypes.byref(info)), "mfa_last_launch_info")
    return info.as_dict()


def mfa_device_status(stream=None):
    code, detail = _i(0), _i(0)
    _check(lib.mfa_device_status(_stream(stream), ctypes.byref(code), ctypes.byref(detail)),
           "mfa_device_status")
    return code.value, detail.value


def mfa_debug_set_flags(flags: int) -> int:
    return lib.mfa_debug_set_flags(flags)


def mfa_debug_tiles_visited(stream=None) -> int:
    n = ctypes.c_ulonglong(0)
    _check(lib.mfa_debug_tiles_visited(_stream(stream), ctypes.byref(n)), "mfa_debug_tiles_visited")
    return n.value


def mfa_debug_tmap_stats() -> dict:
    """Tensor-map cache counters: lookups made by launches (and probes) and encodes done."""
    a, b = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    _check(lib.mfa_debug_tmap_stats(ctypes.byref(a), ctypes.byref(b)), "mfa_debug_tmap_stats")
    return {"lookups": a.value, "encodes": b.value}


def mfa_debug_tmap_probe(base: int, kind: int, dtype: int, outer: int, n: int, D: int) -> bool:
    """Host-only lookup in the tensor-map cache (placeholder maps, no driver): True if it encoded."""
    enc = _i(0)
    _check(lib.mfa_debug_tmap_probe(_vp(base), kind, dtype, outer, n, D, ctypes.byref(enc)),
           "mfa_debug_tmap_probe")
    return bool(enc.value)


def mfa_debug_set_decode_split_pages(pages: int) -> int:
    return lib.mfa_debug_set_decode_split_pages(pages)


def mfa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, out=None, lse=None, *,
                   scale=None, causal=False, window=(-1, -1), softcap=0.0, return_lse=True,
                   stream=None):
    """Packed variable-length forward. q [total_q,Hq,D], k/v [total_k,Hkv,D], cu_seqlens_* int32
    [B+1] on the device; returns (out [total_q,Hq,D], lse [Hq,total_q] or None)."""
    torch = _torch()
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    if k.shape != v.shape or k.shape[2] != D:
        raise ValueError("k and v must be [total_k, Hkv, D] matching q")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    for c in (cu_seqlens_q, cu_seqlens_k):
        if c.dtype != torch.int32 or c.dim() != 1:
            raise TypeError("cu_seqlens must be 1-D int32 tensors")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 offsets")
    B = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    wl, wr = window
    rc = lib.mfa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                            _ptr(cu_seqlens_k), B, int(max_seqlen_q), total_q, total_k, Hq, Hkv, D,
                            float(scale), int(bool(causal)), int(wl), int(wr), float(softcap),
                            _dtype_code(q), _stream(stream))
    _check(rc, "mfa_fwd_varlen")
    return out, lse


def mfa_fwd_blocksparse(q, k, v, block_mask, out=None, lse=None, *, scale=None, causal=False,
                        window=(-1, -1), softcap=0.0, return_lse=True, stream=None):
    """Block-sparse forward. q [B,Hq,Nq,D], k/v [B,Hkv,Nk,D], block_mask uint8
    [B,Hq,ceil(Nq/128),ceil(Nk/128)] on the device; returns (out, lse or None)."""
    torch = _torch()
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k and v must be [B, Hkv, Nk, D] matching q")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    want = (B, Hq, -(-Nq // 128), -(-Nk // 128))
    if block_mask.dtype != torch.uint8 or tuple(block_mask.shape) != want:
        raise ValueError(f"block_mask must be uint8 of shape {want}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    wl, wr = window
    rc = lib.mfa_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(block_mask),
                                 B, Hq, Hkv, Nq, Nk, D, float(scale), int(bool(causal)), int(wl),
                                 int(wr), float(softcap), _dtype_code(q), _stream(stream))
    _check(rc, "mfa_fwd_blocksparse")
    return out, lse


def mfa_bwd_workspace_size(B: int, Hq: int, Nq: int) -> int:
    return lib.mfa_bwd_workspace_size(B, Hq, Nq)


def mfa_bwd(q, k, v, out, dout, lse, dq=None, dk=None, dv=None, *, scale=None, causal=False,
            window=(-1, -1), softcap=0.0, workspace=None, stream=None):
    """Backward of mfa_fwd: gradients of sum(out * dout) given the forward's out and lse.
    q/dq/out/dout [B,Hq,Nq,D], k/v/dk/dv [B,Hkv,Nk,D], lse [B,Hq,Nq] fp32; returns (dq, dk, dv)."""
    torch = _torch()
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    for t in (out, dout):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("out and dout must match q")
    if k.shape != v.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must be [B, Hkv, Nk, D] of q's dtype")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be float32 [B, Hq, Nq]")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = mfa_bwd_workspace_size(B, Hq, Nq)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    wl, wr = window
    rc = lib.mfa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq),
                     _ptr(dk), _ptr(dv), B, Hq, Hkv, Nq, Nk, D, float(scale), int(bool(causal)),
                     int(wl), int(wr), float(softcap), _dtype_code(q), _ptr(workspace),
                     workspace.numel(), _stream(stream))
    _check(rc, "mfa_bwd")
    return dq, dk, dv


def mfa_fwd_paged(q, k_pages, v_pages, block_table, seq_lens, cu_seqlens_q, max_seqlen_q,
                  out=None, lse=None, *, scale=None, causal=True, window=(-1, -1), softcap=0.0,
                  return_lse=True, stream=None):
    """Chunked prefill over a paged cache. q [total_q,Hq,D]; pages [num_pages,16,Hkv,D];
    block_table int32 [B,max_pages]; seq_lens int32 [B]; cu_seqlens_q int32 [B+1] (device).
    Returns (out [total_q,Hq,D], lse [Hq,total_q] or None)."""
    torch = _torch()
    total_q, Hq, D = q.shape
    num_pages, page, Hkv, _ = k_pages.shape
    if k_pages.shape != v_pages.shape or k_pages.shape[3] != D:
        raise ValueError("k_pages and v_pages must be [num_pages, 16, Hkv, D] matching q")
    for t in (block_table, seq_lens, cu_seqlens_q):
        if t.dtype != torch.int32:
            raise TypeError("block_table, seq_lens and cu_seqlens_q must be int32")
    B = seq_lens.numel()
    if cu_seqlens_q.numel() != B + 1 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("cu_seqlens_q must hold B + 1 offsets and block_table B rows")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    wl, wr = window
    rc = lib.mfa_fwd_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens),
                           _ptr(cu_seqlens_q), _ptr(out), _ptr(lse), B, int(max_seqlen_q), total_q,
                           Hq, Hkv, D, page, block_table.shape[1], num_pages, float(scale),
                           int(bool(causal)), int(wl), int(wr), float(softcap), _dtype_code(q),
                           _stream(stream))
    _check(rc, "mfa_fwd_paged")
    return out, lse
