"""The C-ABI boundary without a GPU: the library loads, exports every symbol include/mfa.h
declares, and rejects malformed arguments before touching the device.

Pointers passed here are fake (aligned integers) and every call has exactly one thing wrong,
so each returns its status during validation; no call reaches a CUDA API.
"""
import ctypes
import os
import re

import pytest

import tiled_exact_attention_mfa_b200 as mfa
from conftest import gpu_available

# The rejection tests hand fake addresses to the library; they only run where no GPU is
# reachable, so that a mistake in a case can never turn into a launch on bad pointers.
no_device = pytest.mark.skipif(gpu_available(), reason="fake pointers are used only without a GPU")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mfa.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(mfa_\w+)\s*\(", text, flags=re.M)))


def header_defines():
    return dict(re.findall(r"#define\s+(MFA_\w+)\s+(-?\d+)", open(HEADER).read()))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert "mfa_fwd" in names and "mfa_decode_splitkv" in names
    lib = ctypes.CDLL(mfa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(mfa.EXPORTED)


def test_status_strings_cover_codes():
    d = header_defines()
    codes = [int(v) for k, v in d.items() if k.startswith("MFA_ERR_") or k == "MFA_OK"]
    for c in codes:
        assert mfa.mfa_status_string(c) != "unknown status", c
    assert mfa.mfa_status_string(12345) == "unknown status"
    assert int(d["MFA_DTYPE_BF16"]) == mfa.MFA_DTYPE_BF16


A = 0x10000  # fake, 16-byte aligned device addresses (never dereferenced)


def fwd(**kw):
    args = dict(q=A, k=A, v=A, out=A, lse=A, B=2, Hq=8, Hkv=2, Nq=64, Nk=64, D=128, scale=0.125,
                causal=1, win_l=-1, win_r=-1, softcap=0.0, dtype=1, stream=None)
    args.update(kw)
    return mfa.lib.mfa_fwd(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=2), -3), (dict(D=96), -4), (dict(D=256), -4), (dict(B=-1), -5), (dict(Nk=-3), -5),
    (dict(Hkv=3), -6), (dict(Hkv=0), -6), (dict(win_l=-2), -7), (dict(win_r=-5), -7),
    (dict(softcap=-1.0), -8), (dict(softcap=float("inf")), -8), (dict(softcap=float("nan")), -8),
    (dict(scale=0.0), -9), (dict(scale=float("nan")), -9), (dict(scale=-0.1), -9),
    (dict(q=None), -1), (dict(out=None), -1), (dict(k=None), -1),
    (dict(q=A + 8), -2), (dict(v=A + 4), -2), (dict(lse=A + 2), -2),
])
@no_device
def test_fwd_rejects_malformed(kw, code):
    assert fwd(**kw) == code


@no_device
def test_fwd_empty_problem_is_noop():
    # nothing to compute: OK without any launch, even with NULL pointers
    assert fwd(B=0, q=None, k=None, v=None, out=None) == 0
    assert fwd(Nq=0, q=None, k=None, v=None, out=None) == 0


def fwd_varlen(**kw):
    args = dict(q=A, k=A, v=A, out=A, lse=A, cu_q=A, cu_k=A, B=3, max_q=100, total_q=200,
                total_k=300, Hq=8, Hkv=2, D=128, scale=0.125, causal=1, win_l=-1, win_r=-1,
                softcap=0.0, dtype=0, stream=None)
    args.update(kw)
    return mfa.lib.mfa_fwd_varlen(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=2), -3), (dict(D=32), -4), (dict(B=-1), -5), (dict(total_k=-1), -5),
    (dict(max_q=-1), -5), (dict(max_q=201), -5), (dict(Hkv=3), -6), (dict(win_l=-3), -7),
    (dict(softcap=float("nan")), -8), (dict(scale=0.0), -9), (dict(cu_q=None), -1),
    (dict(cu_k=None), -1), (dict(k=None), -1), (dict(cu_q=A + 2), -2), (dict(out=A + 8), -2),
])
@no_device
def test_fwd_varlen_rejects_malformed(kw, code):
    assert fwd_varlen(**kw) == code


@no_device
def test_fwd_varlen_empty_problem_is_noop():
    assert fwd_varlen(B=0, q=None, k=None, v=None, out=None, cu_q=None, cu_k=None) == 0
    assert fwd_varlen(total_q=0, max_q=0, q=None, out=None) == 0


def fwd_sparse(**kw):
    args = dict(q=A, k=A, v=A, out=A, lse=A, mask=A, B=1, Hq=4, Hkv=2, Nq=512, Nk=512, D=128,
                scale=0.1, causal=0, win_l=-1, win_r=-1, softcap=0.0, dtype=1, stream=None)
    args.update(kw)
    return mfa.lib.mfa_fwd_blocksparse(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=9), -3), (dict(D=100), -4), (dict(Nq=-1), -5), (dict(Hkv=3), -6),
    (dict(win_r=-2), -7), (dict(softcap=-3.0), -8), (dict(scale=float("inf")), -9),
    (dict(mask=None), -1), (dict(q=None), -1), (dict(k=A + 4), -2),
    (dict(Nk=2048 * 128 + 1), -13),
])
@no_device
def test_fwd_blocksparse_rejects_malformed(kw, code):
    assert fwd_sparse(**kw) == code


def dec(**kw):
    ws = kw.pop("ws_bytes", 1 << 30)
    args = dict(q=A, k=A, v=A, table=A, lens=A, out=A, lse=A, B=8, Nq=1, Hq=32, Hkv=8, D=128,
                page=16, max_pages=8192, num_pages=40000, scale=0.088, causal=1, softcap=0.0,
                dtype=1, ws=A, ws_bytes=ws, stream=None)
    args.update(kw)
    return mfa.lib.mfa_decode_splitkv(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=5), -3), (dict(D=80), -4), (dict(Nq=5), -10), (dict(Nq=0), -5), (dict(Hkv=5), -6),
    (dict(page=32), -11), (dict(max_pages=0), -5), (dict(num_pages=0), -5),
    (dict(Hq=64, Hkv=2), -13), (dict(Nq=3, Hq=64, Hkv=8), -13), (dict(softcap=-2.0), -8),
    (dict(scale=float("inf")), -9), (dict(table=None), -1), (dict(lens=None), -1),
    (dict(k=A + 2), -2), (dict(table=A + 4), -2), (dict(ws=None), -12), (dict(ws=A + 16), -12),
    (dict(ws_bytes=1024), -12),
])
@no_device
def test_decode_rejects_malformed(kw, code):
    assert dec(**kw) == code


def decw(win_l, **kw):
    ws = kw.pop("ws_bytes", 1 << 30)
    args = dict(q=A, k=A, v=A, table=A, lens=A, out=A, lse=A, B=8, Nq=1, Hq=32, Hkv=8, D=128,
                page=16, max_pages=8192, num_pages=40000, scale=0.088, causal=1, win_l=win_l,
                softcap=0.0, dtype=1, ws=A, ws_bytes=ws, stream=None)
    args.update(kw)
    return mfa.lib.mfa_decode_splitkv_window(*args.values())


@pytest.mark.parametrize("win_l,kw,code", [
    (-2, {}, -7), (-100, {}, -7), (100, dict(D=80), -4), (100, dict(Nq=5), -10),
    (100, dict(ws_bytes=1024), -12), (0, dict(table=None), -1),
])
@no_device
def test_decode_window_rejects_malformed(win_l, kw, code):
    assert decw(win_l, **kw) == code


def test_decode_head_dims():
    """Decode takes D = 64, 128 and 256 (two kv heads per CTA at 256); other sizes are refused
    before anything else is looked at."""
    for D in (64, 128, 256):
        assert mfa.mfa_decode_workspace_size(8, 1, 32, 8, D, 8192) == \
            8 * 256 * 32 * D * 4 + 8 * 256 * 32 * 2 * 4
    for D in (32, 96, 192, 512):
        assert mfa.mfa_decode_workspace_size(8, 1, 32, 8, D, 8192) == 0


def test_decode_workspace_size_is_shape_only():
    n = mfa.mfa_decode_workspace_size(8, 1, 32, 8, 128, 8192)
    # 8 sequences x 256 splits of 32 pages x 32 rows x (128 + 2) floats
    assert n == 8 * 256 * 32 * 128 * 4 + 8 * 256 * 32 * 2 * 4
    assert mfa.mfa_decode_workspace_size(8, 5, 32, 8, 128, 8192) == 0
    assert mfa.mfa_decode_workspace_size(8, 1, 32, 8, 128, 8192, 8) == 0
    # small grids get smaller splits (more CTAs): 1 sequence of 64 pages -> 4-page splits
    assert mfa.mfa_decode_workspace_size(1, 1, 32, 8, 128, 64) == 16 * 32 * 128 * 4 + 16 * 32 * 2 * 4
    old = mfa.mfa_debug_set_decode_split_pages(8)
    try:
        assert mfa.mfa_decode_workspace_size(1, 1, 32, 8, 128, 64) == 8 * 32 * 128 * 4 + 8 * 32 * 2 * 4
    finally:
        mfa.mfa_debug_set_decode_split_pages(old)


def test_decode_plan_without_window():
    """The shape-only split plan: 32-page splits while the phase-1 grid (splits x B x kv-head
    groups) holds at least 296 CTAs, halved down to 4 pages below that; kv heads per CTA the
    most that divide Hkv with a token row (heads x D x 2 bytes) of at most 1 KB."""
    p = mfa.mfa_decode_plan(8, 1, 32, 8, 128, 8192)
    assert p == {"pages_per_split": 32, "max_splits": 256, "kv_heads_per_cta": 4}
    assert mfa.mfa_decode_workspace_size(8, 1, 32, 8, 128, 8192) == 8 * 256 * 32 * (128 + 2) * 4
    assert mfa.mfa_decode_plan(8, 4, 32, 8, 128, 8192)["max_splits"] == 256  # N_q does not move it
    assert mfa.mfa_decode_workspace_size(8, 4, 32, 8, 128, 8192) == 8 * 256 * 128 * (128 + 2) * 4
    assert mfa.mfa_decode_plan(8, 1, 16, 8, 256, 2048)["kv_heads_per_cta"] == 2
    assert mfa.mfa_decode_plan(8, 1, 32, 8, 64, 2048)["kv_heads_per_cta"] == 8
    assert mfa.mfa_decode_plan(8, 1, 21, 7, 128, 2048)["kv_heads_per_cta"] == 1  # 7 x 256 B > 1 KB
    # 1 sequence of 64 pages, 2 groups: 32 -> 16 -> 8 -> 4 pages per split (16 x 1 x 2 CTAs)
    assert mfa.mfa_decode_plan(1, 1, 32, 8, 128, 64) == \
        {"pages_per_split": 4, "max_splits": 16, "kv_heads_per_cta": 4}
    # 2 sequences of 2048 pages: 64 x 2 x 2 = 256 CTAs at 32 pages is below 296, 16 pages is not
    assert mfa.mfa_decode_plan(2, 1, 32, 8, 128, 2048)["pages_per_split"] == 16


def test_decode_plan_with_window():
    """With a left window the splits cover only the window's page span, (win_l + N_q + 15) / 16
    + 1 pages: the split is the smallest halving of 32 whose grid over that span still fits in
    296 CTAs, never with more splits than the plan without the window; the split override still
    applies."""
    # 4096-token window over 128k-token caches: a span of 257 pages; 16-page splits give
    # 17 x 8 x 2 = 272 CTAs, 8-page splits would give 33 x 8 x 2 = 528
    assert mfa.mfa_decode_plan(8, 1, 32, 8, 128, 8192, win_l=4095) == \
        {"pages_per_split": 16, "max_splits": 17, "kv_heads_per_cta": 4}
    assert mfa.mfa_decode_plan(8, 4, 32, 8, 128, 8192, win_l=4095)["max_splits"] == 17  # 258 pages
    # a window wider than the cache is the plan without a window
    assert mfa.mfa_decode_plan(8, 1, 32, 8, 128, 8192, win_l=10 ** 9) == \
        mfa.mfa_decode_plan(8, 1, 32, 8, 128, 8192)
    # a one-token window spans 2 pages: one split of the smallest size
    assert mfa.mfa_decode_plan(8, 1, 32, 8, 128, 8192, win_l=0) == \
        {"pages_per_split": 4, "max_splits": 1, "kv_heads_per_cta": 4}
    old = mfa.mfa_debug_set_decode_split_pages(8)
    try:
        p = mfa.mfa_decode_plan(8, 1, 32, 8, 128, 8192, win_l=4095)
        assert p["pages_per_split"] == 8 and p["max_splits"] == 33
        assert mfa.mfa_decode_plan(8, 1, 32, 8, 128, 8192)["max_splits"] == 1024
    finally:
        mfa.mfa_debug_set_decode_split_pages(old)


def test_decode_plan_rejects_what_decode_rejects():
    codes = header_defines()
    for args, name in [((8, 5, 32, 8, 128, 8192, 16, -1), "MFA_ERR_NQ_TOO_LARGE"),
                       ((8, 1, 32, 8, 96, 8192, 16, -1), "MFA_ERR_BAD_HEAD_DIM"),
                       ((8, 1, 30, 8, 128, 8192, 16, -1), "MFA_ERR_GQA_GEOMETRY"),
                       ((8, 1, 32, 8, 128, 8192, 8, -1), "MFA_ERR_PAGE_SIZE"),
                       ((8, 1, 32, 8, 128, 8192, 16, -2), "MFA_ERR_BAD_WINDOW")]:
        with pytest.raises(mfa.MFAError) as e:
            mfa.mfa_decode_plan(*args[:6], page_size=args[6], win_l=args[7])
        assert e.value.code == int(codes[name]), name


def test_debug_flags_roundtrip():
    old = mfa.mfa_debug_set_flags(3)
    assert mfa.mfa_debug_set_flags(old) == 3


def fwdh(**kw):
    ws = kw.pop("ws_bytes", 1 << 30)
    args = dict(q=A, k=A, v=A, out=A, lse=A, B=2, Hq=8, Hkv=2, Nq=64, Nk=64, D=128, scale=0.125,
                causal=1, win_l=-1, win_r=-1, softcap=0.0, dtype=1, ws=A, ws_bytes=ws, stream=None)
    args.update(kw)
    return mfa.lib.mfa_fwd_host(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), -3), (dict(D=96), -4), (dict(B=-1), -5), (dict(Hkv=3), -6),
    (dict(win_l=-3), -7), (dict(softcap=-1.0), -8), (dict(scale=0.0), -9),
    (dict(q=None), -1), (dict(k=None), -1), (dict(out=None), -1),
    (dict(ws=None), -12), (dict(ws=A + 128), -12), (dict(ws_bytes=4096), -12),
])
@no_device
def test_fwd_host_rejects_malformed(kw, code):
    assert fwdh(**kw) == code


def test_fwd_host_scratch_size():
    """Device copies of q, k, v, out and lse, each region rounded up to 256 bytes."""
    r = lambda x: (x + 255) // 256 * 256
    B, Hq, Hkv, Nq, Nk, D = 2, 8, 2, 100, 300, 64
    q = B * Hq * Nq * D * 2
    kv = B * Hkv * Nk * D * 2
    lse = B * Hq * Nq * 4
    assert mfa.mfa_fwd_host_scratch_size(B, Hq, Hkv, Nq, Nk, D) == 2 * r(q) + 2 * r(kv) + r(lse)
    assert mfa.mfa_fwd_host_scratch_size(B, Hq, 3, Nq, Nk, D) == 0
    assert mfa.mfa_fwd_host_scratch_size(B, Hq, Hkv, Nq, Nk, 96) == 0
    assert mfa.mfa_fwd_host_scratch_size(0, Hq, Hkv, Nq, Nk, D) == 0 + 0 + 0


@no_device
def test_fwd_host_empty_problem_is_a_no_op():
    assert fwdh(B=0, q=None, k=None, v=None, out=None, lse=None, ws=None) == 0


def test_tensor_map_cache_hits_the_second_time():
    """The tensor-map cache, host only (placeholder maps): a key's first lookup encodes, the
    second with the same key encodes nothing, any changed field is a new key, and after more
    than the cache's 256 distinct keys the least recently used one has been replaced."""
    base = 0x7F0000100000
    before = mfa.mfa_debug_tmap_stats()
    assert mfa.mfa_debug_tmap_probe(base, 0, 0, 16, 4096, 128)
    assert not mfa.mfa_debug_tmap_probe(base, 0, 0, 16, 4096, 128)
    after = mfa.mfa_debug_tmap_stats()
    assert after["lookups"] - before["lookups"] == 2
    assert after["encodes"] - before["encodes"] == 1
    for changed in ((base + 256, 0, 0, 16, 4096, 128), (base, 1, 0, 16, 4096, 128),
                    (base, 0, 1, 16, 4096, 128), (base, 0, 0, 8, 4096, 128),
                    (base, 0, 0, 16, 4095, 128), (base, 0, 0, 16, 4096, 64)):
        assert mfa.mfa_debug_tmap_probe(*changed), changed
        assert not mfa.mfa_debug_tmap_probe(*changed), changed
    # keep the first key recently used while 300 other keys pass through: it stays, the oldest go
    for i in range(300):
        mfa.mfa_debug_tmap_probe(base + 4096 * (i + 1), 2, 1, 8, 16 * 1024, 128)
        assert not mfa.mfa_debug_tmap_probe(base, 0, 0, 16, 4096, 128)
    assert mfa.mfa_debug_tmap_probe(base + 4096, 2, 1, 8, 16 * 1024, 128)  # evicted long ago
