"""GPU parity of mfa_fwd (through the C ABI) against the fp64 oracle on seeded inputs."""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu

P = mi.PrefillCase
SMALL = [
    # name, B, Hq, Hkv, Nq, Nk, D, dtype, causal, win_l, win_r, softcap, mul, seed
    P("causal_ragged_d64_fp16", 1, 2, 2, 300, 300, 64, mi.FP16, True, seed=11),
    P("noncausal_gqa_d128_bf16", 2, 4, 2, 515, 515, 128, mi.BF16, False, seed=12),
    P("causal_nq_lt_nk_gqa4_fp16", 1, 4, 1, 200, 700, 128, mi.FP16, True, seed=13),
    P("causal_nq_gt_nk_empty_rows_bf16", 1, 2, 2, 700, 200, 64, mi.BF16, True, seed=14),
    P("window100_causal_fp16", 1, 2, 2, 1000, 1000, 128, mi.FP16, True, 100, 0, seed=15),
    P("window_two_sided_bf16", 1, 2, 2, 777, 777, 64, mi.BF16, False, 50, 30, seed=16),
    P("window_left_only_noncausal_fp16", 2, 2, 1, 390, 390, 128, mi.FP16, False, 130, -1, seed=17),
    P("gqa_softcap50_bf16", 1, 8, 2, 640, 640, 128, mi.BF16, True, softcap=50.0, mul=0.5, seed=18),
    P("softcap2_large_scores_fp16", 1, 2, 2, 257, 257, 64, mi.FP16, True, softcap=2.0, mul=2.0,
      seed=19),
    P("single_key_window00_bf16", 1, 2, 2, 129, 129, 64, mi.BF16, False, 0, 0, seed=20),
    P("tiny_nk1_fp16", 1, 2, 2, 5, 1, 64, mi.FP16, False, seed=21),
    P("d128_fp16_many_heads", 3, 6, 3, 384, 384, 128, mi.FP16, True, seed=22),
    P("single_query_row_bf16", 2, 4, 2, 1, 1000, 128, mi.BF16, True, seed=23),
    # scores of std 16 (through the scale; V stays unit-scale, as the absolute tolerance on O
    # assumes): the running max moves by more than 2^8 (log2) between tiles, so the lazy rescale
    # of O runs often
    P("large_logits_noncausal_fp16", 1, 2, 2, 400, 900, 128, mi.FP16, False, seed=24,
      scale=16.0 / 128 ** 0.5),
    # windows of INT_MAX on both sides (a common "unbounded" sentinel) with Nq > Nk: the same
    # visible set as no window, and no wrap-around in the position arithmetic
    P("window_int_max_nq_gt_nk_fp16", 1, 2, 2, 300, 200, 64, mi.FP16, True, 2 ** 31 - 1,
      2 ** 31 - 1, seed=25),
    P("window_int_max_noncausal_bf16", 1, 2, 1, 200, 333, 128, mi.BF16, False, 2 ** 31 - 1,
      2 ** 31 - 1, seed=26),
    # windowed launches run one Q tile per CTA (two CTAs per SM): bottom-right alignment with
    # Nq < Nk under GQA, and Nq > Nk with rows that see no key
    P("window_nq_lt_nk_gqa2_d64_bf16", 2, 4, 2, 300, 900, 64, mi.BF16, True, 200, 0, seed=27),
    P("window_nq_gt_nk_empty_rows_fp16", 1, 2, 2, 500, 260, 128, mi.FP16, True, 150, 0, seed=28),
]


def run_gpu(case, q, k, v):
    import tiled_exact_attention_mfa_b200 as mfa
    qt, kt, vt = (to_torch(x, case.dtype) for x in (q, k, v))
    out, lse = mfa.mfa_fwd(qt, kt, vt, scale=case.scale_f32(), causal=case.causal,
                           window=(case.win_l, case.win_r), softcap=case.softcap)
    import torch
    torch.cuda.synchronize()
    return from_torch(out), from_torch(lse)


def oracle_full(case, q, k, v):
    w = lambda x: mi.widen(x, case.dtype)
    return oracle.attention(w(q), w(k), w(v), case.scale_f32(), case.causal, case.win_l, case.win_r,
                            case.softcap)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_cases_match_oracle(cuda_device, case):
    q, k, v = case.tensors()
    o, lse = run_gpu(case, q, k, v)
    o_ref, lse_ref = oracle_full(case, q, k, v)
    check_close(o, lse, o_ref, lse_ref, case.dtype, case.name)


def test_causal_b1_h2_n128_d64_full(cuda_device):
    case = mi.workloads()["causal_b1_h2_n128_d64_fp16"]
    q, k, v = case.tensors()
    o, lse = run_gpu(case, q, k, v)
    o_ref, lse_ref = oracle_full(case, q, k, v)
    check_close(o, lse, o_ref, lse_ref, case.dtype, case.name)


FULL = ["causal_b2_h8_n4096_d128_fp16", "noncausal_b2_h8_n4096_d128_fp16",
        "causal_b2_h8_n8192_d128_fp16",
        "window512_b2_h8_n8192_d128_fp16", "window256_b2_h8_n8192_d128_fp16",
        "gqa_causal_b1_hq32_hkv8_n16384_d128_bf16_cap50"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_every_element(cuda_device, name):
    """Every element of O and LSE of a full-size workload against the oracle (computed on all
    host cores, cached by workload, seed and oracle version)."""
    from oracle import cache
    case = mi.workloads()[name]
    q, k, v = case.tensors()
    o, lse = run_gpu(case, q, k, v)
    ref = cache.reference(name, (q, k, v))
    check_close(o, lse, ref["o"], ref["lse"], case.dtype, name)


def test_tile_skip_is_bitwise_neutral(cuda_device):
    """Visiting every key tile with element masks gives bitwise the same O and LSE."""
    import tiled_exact_attention_mfa_b200 as mfa
    for case in (P("w", 1, 4, 2, 1000, 1000, 128, mi.FP16, True, 200, 0, seed=31),
                 P("c", 2, 2, 2, 900, 640, 64, mi.BF16, True, seed=32),
                 P("t", 1, 2, 1, 700, 700, 128, mi.BF16, False, 90, 40, softcap=30.0, seed=33)):
        q, k, v = case.tensors()
        o1, l1 = run_gpu(case, q, k, v)
        old = mfa.mfa_debug_set_flags(mfa.MFA_DEBUG_NO_TILE_SKIP)
        try:
            o2, l2 = run_gpu(case, q, k, v)
        finally:
            mfa.mfa_debug_set_flags(old)
        assert np.array_equal(o1, o2), case.name
        assert np.array_equal(l1, l2), case.name


def q_rows_per_cta():
    """Query rows one CTA of the forward kernel covers (128 per Q tile), from its launch record."""
    import tiled_exact_attention_mfa_b200 as mfa
    info = mfa.mfa_last_launch_info()
    assert info["kernel"] == 1
    return info["tile_m"] * info["q_tiles_per_cta"]


def tiles_closed_form(case, bm, bn=128):
    """Key tiles intersecting each bm-row block's visible set, counted on the mask itself."""
    vis = oracle.visible(case.Nq, case.Nk, case.causal, case.win_l, case.win_r)
    n = 0
    for r0 in range(0, case.Nq, bm):
        cols = vis[r0:r0 + bm].any(axis=0)
        n += len({j // bn for j in np.nonzero(cols)[0]})
    return n * case.B * case.Hq


def test_visited_tile_count_matches_closed_form(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    mfa.mfa_debug_tiles_visited()  # reset
    for case in (P("c", 1, 2, 2, 1000, 1000, 64, mi.FP16, True, seed=41),
                 P("w", 1, 2, 2, 2048, 2048, 64, mi.FP16, True, 300, 0, seed=42),
                 P("n", 2, 1, 1, 300, 900, 64, mi.BF16, True, 64, 64, seed=43)):
        q, k, v = case.tensors()
        old = mfa.mfa_debug_set_flags(mfa.MFA_DEBUG_COUNT_TILES)
        try:
            run_gpu(case, q, k, v)
            got = mfa.mfa_debug_tiles_visited()
        finally:
            mfa.mfa_debug_set_flags(old)
        bm = q_rows_per_cta()
        assert got == tiles_closed_form(case, bm), case.name
        old = mfa.mfa_debug_set_flags(mfa.MFA_DEBUG_COUNT_TILES | mfa.MFA_DEBUG_NO_TILE_SKIP)
        try:
            run_gpu(case, q, k, v)
            got = mfa.mfa_debug_tiles_visited()
        finally:
            mfa.mfa_debug_set_flags(old)
        assert got == -(-case.Nq // bm) * -(-case.Nk // 128) * case.B * case.Hq
    torch.cuda.synchronize()


def test_empty_keys_and_repeatability(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    q = torch.randn(1, 2, 10, 64, device="cuda", dtype=torch.float16)
    k = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    out, lse = mfa.mfa_fwd(q, k, k.clone(), causal=False)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    case = SMALL[1]
    a = run_gpu(case, *case.tensors())
    b = run_gpu(case, *case.tensors())
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    code, detail = mfa.mfa_device_status()
    assert code == 0, (code, detail)


def test_launch_info_reports_the_prefill_kernel(cuda_device):
    import tiled_exact_attention_mfa_b200 as mfa
    case = SMALL[0]
    run_gpu(case, *case.tensors())
    info = mfa.mfa_last_launch_info()
    assert info["kernel"] == 1 and info["tile_m"] == 128 and info["tile_n"] == 128
    rows = 128 * info["q_tiles_per_cta"]
    assert info["q_tiles_per_cta"] in (1, 2)
    assert info["grid_x"] == -(-300 // rows) * 2  # query blocks x 2 heads


def test_second_call_on_the_same_buffers_encodes_no_tensor_map(cuda_device):
    """The library caches TMA tensor maps per (device, base pointer, dtype, layout, extents): a
    repeated forward over the same buffers encodes none, and new buffers encode theirs."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = SMALL[1]
    q, k, v = case.tensors()
    qt, kt, vt = (to_torch(x, case.dtype) for x in (q, k, v))
    kw = dict(scale=case.scale_f32(), causal=case.causal, window=(case.win_l, case.win_r),
              softcap=case.softcap)
    o1, l1 = mfa.mfa_fwd(qt, kt, vt, **kw)
    s1 = mfa.mfa_debug_tmap_stats()
    o2, l2 = mfa.mfa_fwd(qt, kt, vt, o1, l1, **kw)
    s2 = mfa.mfa_debug_tmap_stats()
    # q, k, v and out each have a map; none is encoded again
    assert s2["lookups"] - s1["lookups"] == 4 and s2["encodes"] == s1["encodes"]
    ref = (o2.clone(), l2.clone())
    mfa.mfa_fwd(qt.clone(), kt, vt, o1, l1, **kw)  # only q lives elsewhere now
    s3 = mfa.mfa_debug_tmap_stats()
    assert s3["encodes"] - s2["encodes"] == 1
    torch.cuda.synchronize()
    assert torch.equal(o1, ref[0]) and torch.equal(l1, ref[1])
