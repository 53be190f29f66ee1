"""GPU parity of mfa_fwd_blocksparse (a 128 x 128 block mask on top of causal / window, through
the C ABI) against the fp64 oracle on seeded inputs."""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu

S = mi.SparseCase
SMALL = [
    # name, B, Hq, Hkv, N, D, dtype, causal, pattern options
    S("random_noncausal_fp16", 2, 4, 2, 700, 128, mi.FP16, False, density=0.35, seed=61),
    S("random_causal_bf16", 1, 8, 2, 1000, 128, mi.BF16, True, density=0.5, seed=62),
    S("random_sparse_d64_fp16", 2, 2, 2, 1300, 64, mi.FP16, False, density=0.1, seed=63),
    S("window_softcap_bf16", 1, 4, 4, 900, 128, mi.BF16, True, density=0.6, win_l=200, win_r=0,
      softcap=25.0, seed=64),
    S("spatial2d_radius1_fp16", 1, 2, 1, 12 * 128, 128, mi.FP16, False, pattern="spatial2d",
      grid=(3, 4), radius=1, seed=65),
]


def run_gpu(case, q, k, v, m):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    out, lse = mfa.mfa_fwd_blocksparse(to_torch(q, case.dtype), to_torch(k, case.dtype),
                                       to_torch(v, case.dtype), torch.from_numpy(m).cuda(),
                                       scale=case.scale_f32(), causal=case.causal,
                                       window=(case.win_l, case.win_r), softcap=case.softcap)
    torch.cuda.synchronize()
    return from_torch(out), from_torch(lse)


def oracle_full(case, q, k, v, m):
    w = lambda x: mi.widen(x, case.dtype)
    return oracle.attention_blocksparse(w(q), w(k), w(v), m, case.scale_f32(), case.causal,
                                        case.win_l, case.win_r, case.softcap)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_blocksparse_cases_match_oracle(cuda_device, case):
    q, k, v, m = case.tensors()
    o, lse = run_gpu(case, q, k, v, m)
    o_ref, l_ref = oracle_full(case, q, k, v, m)
    check_close(o, lse, o_ref, l_ref, case.dtype, case.name)


def test_mask_with_empty_rows_and_nq_ne_nk(cuda_device):
    """Nq != Nk (bottom-right causal), ragged tails, and query blocks whose mask row is all
    zero (their rows get out = 0, lse = -inf)."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = mi.PrefillCase("nq_ne_nk", 1, 4, 2, 300, 650, 128, mi.FP16, True, seed=66)
    q, k, v = case.tensors()
    rng = np.random.default_rng(5)
    m = (rng.random((1, 4, 3, 6)) < 0.5).astype(np.uint8)
    m[0, 1, 1, :] = 0          # a whole 128-row block of head 1 sees nothing
    m[0, 2, :, :] = 0          # head 2 sees nothing at all
    out, lse = mfa.mfa_fwd_blocksparse(to_torch(q, case.dtype), to_torch(k, case.dtype),
                                       to_torch(v, case.dtype), torch.from_numpy(m).cuda(),
                                       scale=case.scale_f32(), causal=True)
    torch.cuda.synchronize()
    w = lambda x: mi.widen(x, case.dtype)
    o_ref, l_ref = oracle.attention_blocksparse(w(q), w(k), w(v), m, case.scale_f32(), True)
    check_close(from_torch(out), from_torch(lse), o_ref, l_ref, case.dtype, "nq_ne_nk")
    assert np.all(from_torch(out)[0, 2] == 0) and np.all(np.isneginf(from_torch(lse)[0, 2]))


def test_all_ones_mask_is_bitwise_the_dense_forward(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    for causal, window, cap in ((True, (-1, -1), 0.0), (False, (150, 40), 0.0), (True, (-1, -1), 30.0)):
        case = mi.PrefillCase("ones", 2, 4, 2, 520, 520, 128, mi.BF16, causal, window[0], window[1],
                              softcap=cap, seed=67)
        q, k, v = case.tensors()
        qt, kt, vt = (to_torch(x, case.dtype) for x in (q, k, v))
        ones = torch.ones((2, 4, 5, 5), dtype=torch.uint8, device="cuda")
        o1, l1 = mfa.mfa_fwd_blocksparse(qt, kt, vt, ones, scale=case.scale_f32(), causal=causal,
                                         window=window, softcap=cap)
        o2, l2 = mfa.mfa_fwd(qt, kt, vt, scale=case.scale_f32(), causal=causal, window=window,
                             softcap=cap)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), (causal, window, cap)


def tiles_closed_form(case, m, bm=256, bn=128):
    """Key tiles a 256-row block visits: those that one of its two 128-row Q tiles both has on in
    the mask and can see with some of its rows (causal / window)."""
    vis = oracle.visible(case.Nq, case.Nk, case.causal, case.win_l, case.win_r)
    n = 0
    for b in range(case.B):
        for h in range(case.Hq):
            for r0 in range(0, case.Nq, bm):
                visited = set()
                for t in range(bm // 128):
                    rs = r0 + 128 * t
                    if rs >= case.Nq:
                        continue
                    cols = vis[rs:rs + 128].any(axis=0)
                    visited |= {j // bn for j in np.nonzero(cols)[0] if m[b, h, rs // 128, j // bn]}
                n += len(visited)
    return n


def test_visited_tiles_and_tile_skip_neutrality(cuda_device):
    """The visited-tile counter equals the closed form, and visiting every key tile of the mask
    (no causal / window skip: each Q tile then also takes part in tiles its rows cannot see,
    which contribute exact zeros) gives bitwise the same outputs."""
    import tiled_exact_attention_mfa_b200 as mfa
    case = S("cnt", 1, 2, 2, 1100, 64, mi.FP16, True, density=0.4, win_l=300, win_r=0, seed=68)
    q, k, v, m = case.tensors()
    mfa.mfa_debug_tiles_visited()  # reset
    old = mfa.mfa_debug_set_flags(mfa.MFA_DEBUG_COUNT_TILES)
    try:
        o1, l1 = run_gpu(case, q, k, v, m)
        got = mfa.mfa_debug_tiles_visited()
    finally:
        mfa.mfa_debug_set_flags(old)
    assert got == tiles_closed_form(case, m)
    old = mfa.mfa_debug_set_flags(mfa.MFA_DEBUG_NO_TILE_SKIP)
    try:
        o2, l2 = run_gpu(case, q, k, v, m)
    finally:
        mfa.mfa_debug_set_flags(old)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_full_size_spatial_workload_every_element(cuda_device):
    from oracle import cache
    case = mi.workloads()["sparse_spatial2d_b1_h16_n16384_d128_fp16"]
    q, k, v, m = case.tensors()
    o, lse = run_gpu(case, q, k, v, m)
    ref = cache.reference(case.name, (q, k, v, m))
    check_close(o, lse, ref["o"], ref["lse"], case.dtype, case.name)
