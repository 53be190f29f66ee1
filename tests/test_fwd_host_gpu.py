"""mfa_fwd_host -- the forward over host buffers, its copies pipelined over runs of
(batch, kv-head) units -- against mfa_fwd on the same data: the outputs are bitwise equal
whatever the run boundaries (each run is the same per-row computation), and also within the
oracle's tolerance."""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu

P = mi.PrefillCase
CASES = [
    P("gqa4_causal_fp16_6units", 3, 8, 2, 300, 300, 128, mi.FP16, True, seed=91),
    P("mha_window_bf16_13units", 1, 13, 13, 200, 450, 64, mi.BF16, False, 100, 20, seed=92),
    P("softcap_nq_gt_nk_fp16_5units", 5, 2, 1, 260, 130, 128, mi.FP16, True, softcap=30.0, seed=93),
    P("single_unit_bf16", 1, 4, 1, 700, 700, 128, mi.BF16, True, seed=94),
]


def host(bits, dtype):
    return to_torch(bits, dtype, device="cpu").pin_memory()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_host_forward_equals_device_forward(cuda_device, case):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    q, k, v = case.tensors()
    kw = dict(scale=case.scale_f32(), causal=case.causal, window=(case.win_l, case.win_r),
              softcap=case.softcap)
    od, ld = mfa.mfa_fwd(to_torch(q, case.dtype), to_torch(k, case.dtype), to_torch(v, case.dtype), **kw)
    oh, lh = mfa.mfa_fwd_host(host(q, case.dtype), host(k, case.dtype), host(v, case.dtype), **kw)
    torch.cuda.synchronize()
    assert not oh.is_cuda and not lh.is_cuda
    assert torch.equal(od.cpu(), oh) and torch.equal(ld.cpu(), lh)
    w = lambda x: mi.widen(x, case.dtype)
    o_ref, l_ref = oracle.attention(w(q), w(k), w(v), case.scale_f32(), case.causal, case.win_l,
                                    case.win_r, case.softcap)
    check_close(from_torch(oh), from_torch(lh), o_ref, l_ref, case.dtype, case.name)


def test_back_to_back_calls_share_one_scratch(cuda_device):
    """Two calls queued before any synchronisation, through one scratch buffer: the second call's
    copies in wait for the first call's kernels and copies out."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    a = P("a", 2, 4, 2, 500, 500, 128, mi.FP16, True, seed=95)
    b = P("b", 2, 4, 2, 500, 500, 128, mi.FP16, True, seed=96)
    n = mfa.mfa_fwd_host_scratch_size(2, 4, 2, 500, 500, 128)
    scratch = torch.empty(n, dtype=torch.uint8, device="cuda")
    outs = []
    for c in (a, b, a):
        q, k, v = c.tensors()
        outs.append(mfa.mfa_fwd_host(host(q, c.dtype), host(k, c.dtype), host(v, c.dtype),
                                     scale=c.scale_f32(), causal=True, scratch=scratch))
    torch.cuda.synchronize()
    for c, (oh, lh) in zip((a, b, a), outs):
        q, k, v = c.tensors()
        od, ld = mfa.mfa_fwd(to_torch(q, c.dtype), to_torch(k, c.dtype), to_torch(v, c.dtype),
                             scale=c.scale_f32(), causal=True)
        torch.cuda.synchronize()
        assert torch.equal(od.cpu(), oh) and torch.equal(ld.cpu(), lh)


def test_empty_keys_and_no_lse(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    q = torch.randn(2, 4, 50, 64, dtype=torch.bfloat16).pin_memory()
    k = torch.empty(2, 2, 0, 64, dtype=torch.bfloat16).pin_memory()
    out, lse = mfa.mfa_fwd_host(q, k, k.clone())
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    c = P("nolse", 2, 4, 2, 130, 260, 64, mi.FP16, False, seed=97)
    qb, kb, vb = c.tensors()
    oh, lh = mfa.mfa_fwd_host(host(qb, c.dtype), host(kb, c.dtype), host(vb, c.dtype),
                              scale=c.scale_f32(), return_lse=False)
    od, _ = mfa.mfa_fwd(to_torch(qb, c.dtype), to_torch(kb, c.dtype), to_torch(vb, c.dtype),
                        scale=c.scale_f32())
    torch.cuda.synchronize()
    assert lh is None and torch.equal(od.cpu(), oh)
