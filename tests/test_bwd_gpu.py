"""GPU parity of mfa_bwd (through the C ABI) against the fp64 oracle backward on seeded inputs.

The GPU backward starts from its own forward (out rounded to the input type, fp32 LSE) and
rounds P and dS to the input type before the dV, dK and dQ products, so its error scales with
the input type's rounding unit and the gradients' magnitude: the bound below is
max |g - g_oracle| <= TOL[dtype] * max |g_oracle| per tensor, TOL = 4 units of rounding
(4 * 2^-11 for fp16, 4 * 2^-8 for bf16); the cases below measured at most 1.1 units.
"""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import from_torch, to_torch

pytestmark = pytest.mark.gpu

TOL = {mi.FP16: 4 * 2.0 ** -11, mi.BF16: 4 * 2.0 ** -8}

P = mi.PrefillCase
CASES = [
    P("causal_ragged_d64_fp16", 1, 2, 2, 300, 300, 64, mi.FP16, True, seed=71),
    P("noncausal_gqa_d128_bf16", 2, 4, 2, 260, 260, 128, mi.BF16, False, seed=72),
    P("causal_nq_lt_nk_gqa4_fp16", 1, 4, 1, 130, 400, 128, mi.FP16, True, seed=73),
    P("causal_nq_gt_nk_empty_rows_bf16", 1, 2, 2, 400, 150, 64, mi.BF16, True, seed=74),
    P("window_two_sided_fp16", 1, 2, 1, 333, 333, 128, mi.FP16, False, 70, 40, seed=75),
    P("window_causal_softcap_bf16", 1, 4, 2, 500, 500, 128, mi.BF16, True, 150, 0, softcap=20.0,
      seed=76),
    P("softcap_large_scores_fp16", 1, 2, 2, 257, 257, 64, mi.FP16, True, softcap=2.0, mul=2.0,
      seed=77),
]


def dout_bits(case):
    return case.dout()


def run(case):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    q, k, v = case.tensors()
    do = dout_bits(case)
    qt, kt, vt, dot = (to_torch(x, case.dtype) for x in (q, k, v, do))
    win = (case.win_l, case.win_r)
    out, lse = mfa.mfa_fwd(qt, kt, vt, scale=case.scale_f32(), causal=case.causal, window=win,
                           softcap=case.softcap)
    dq, dk, dv = mfa.mfa_bwd(qt, kt, vt, out, dot, lse, scale=case.scale_f32(), causal=case.causal,
                             window=win, softcap=case.softcap)
    torch.cuda.synchronize()
    return (q, k, v, do), (from_torch(dq), from_torch(dk), from_torch(dv))


def check(case, inputs, grads):
    q, k, v, do = inputs
    w = lambda x: mi.widen(x, case.dtype)
    ref = oracle.attention_backward(w(q), w(k), w(v), w(do), case.scale_f32(), case.causal,
                                    case.win_l, case.win_r, case.softcap)
    for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
        assert np.all(np.isfinite(g)), f"{case.name}: non-finite {name}"
        err = float(np.max(np.abs(g - r)))
        bound = TOL[case.dtype] * max(float(np.max(np.abs(r))), 1e-6)
        print(f"{case.name} {name}: max err {err:.3e}  max |ref| {np.max(np.abs(r)):.3e}  bound {bound:.3e}")
        assert err <= bound, f"{case.name}: max |{name} - oracle| = {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_backward_matches_oracle(cuda_device, case):
    inputs, grads = run(case)
    check(case, inputs, grads)


@pytest.mark.parametrize("name", ["causal_b2_h8_n4096_d128_fp16",
                                  "noncausal_b2_h8_n4096_d128_fp16"])
def test_full_size_backward_every_element(cuda_device, name):
    """The backward of the B=2 H=8 N=4096 D=128 workloads, every element of dq / dk / dv against
    the oracle's gradients (cached), at the bound above."""
    from oracle import cache
    case = mi.workloads()[name]
    inputs, grads = run(case)
    ref = cache.reference(name + ":backward", inputs[:3])
    for gname, g in zip(("dq", "dk", "dv"), grads):
        r = ref[gname]
        assert np.all(np.isfinite(g)), f"{name}: non-finite {gname}"
        err = float(np.max(np.abs(g - r)))
        bound = TOL[case.dtype] * max(float(np.max(np.abs(r))), 1e-6)
        print(f"{name} {gname}: max err {err:.3e}  max |ref| {np.max(np.abs(r)):.3e}  bound {bound:.3e}")
        assert err <= bound, f"{name}: max |{gname} - oracle| = {err:.3e} > {bound:.3e}"


def test_backward_is_deterministic_and_empty_rows_get_zero_dq(cuda_device):
    case = CASES[3]  # Nq > Nk causal: the first Nq - Nk rows see no key
    _, g1 = run(case)
    _, g2 = run(case)
    for a, b in zip(g1, g2):
        assert np.array_equal(a, b)
    assert np.all(g1[0][:, :, :case.Nq - case.Nk] == 0)


@pytest.mark.parametrize("idx", [0, 5, 6])
def test_backward_repeats_bitwise(cuda_device, idx):
    """Eight backward calls on the same inputs give the same bits: the passes have no atomics, so
    any difference would come from a read that raced a write (an early phase wait, a buffer
    reused before its reader finished). The capped cases take the fastest elementwise path, where
    the dQ epilogue once read its accumulator before the last MMAs completed."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = CASES[idx]
    q, k, v = case.tensors()
    qt, kt, vt, dot = (to_torch(x, case.dtype) for x in (q, k, v, dout_bits(case)))
    win = (case.win_l, case.win_r)
    out, lse = mfa.mfa_fwd(qt, kt, vt, scale=case.scale_f32(), causal=case.causal, window=win,
                           softcap=case.softcap)
    first = None
    for _ in range(8):
        g = mfa.mfa_bwd(qt, kt, vt, out, dot, lse, scale=case.scale_f32(), causal=case.causal,
                        window=win, softcap=case.softcap)
        torch.cuda.synchronize()
        if first is None:
            first = [t.clone() for t in g]
        else:
            for a, b in zip(first, g):
                assert torch.equal(a, b)


def test_backward_empty_sides(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    q = torch.randn(1, 2, 10, 64, device="cuda", dtype=torch.float16)
    k = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    out, lse = mfa.mfa_fwd(q, k, k.clone())
    dq, dk, dv = mfa.mfa_bwd(q, k, k.clone(), out, torch.randn_like(q), lse)
    torch.cuda.synchronize()
    assert torch.all(dq == 0)
