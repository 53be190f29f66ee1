"""GPU parity of mfa_fwd_varlen (packed variable-length batches, through the C ABI) against the
fp64 oracle on seeded inputs."""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu

V = mi.VarlenCase
SMALL = [
    # name, B, Hq, Hkv, D, dtype, causal, ..., explicit lengths
    V("causal_ragged_lengths_fp16", 4, 4, 2, 128, mi.FP16, True, fixed_q=[300, 1, 129, 77],
      fixed_k=[300, 1, 129, 77], seed=51),
    V("chunked_prefill_nk_gt_nq_bf16", 3, 8, 2, 128, mi.BF16, True, fixed_q=[64, 200, 17],
      fixed_k=[500, 260, 400], seed=52),
    V("noncausal_nq_gt_nk_d64_fp16", 3, 2, 2, 64, mi.FP16, False, fixed_q=[250, 40, 130],
      fixed_k=[90, 300, 1], seed=53),
    V("empty_sequences_bf16", 5, 4, 4, 64, mi.BF16, True, fixed_q=[0, 33, 140, 0, 20],
      fixed_k=[10, 0, 140, 0, 50], seed=54),
    V("window_softcap_gqa_bf16", 3, 8, 2, 128, mi.BF16, True, win_l=90, win_r=0, softcap=30.0,
      fixed_q=[400, 129, 257], fixed_k=[400, 200, 257], seed=55),
    V("two_sided_window_fp16", 2, 2, 1, 128, mi.FP16, False, win_l=40, win_r=25,
      fixed_q=[333, 128], fixed_k=[333, 128], seed=56),
    V("seeded_lengths_fp16", 6, 4, 4, 128, mi.FP16, True, 1, 700, k_extra=300, seed=57),
]


def upload(case):
    import torch
    q, k, v = case.tensors()
    cq, ck = case.cu_seqlens()
    dev = torch.device("cuda")
    return (q, k, v, cq, ck, to_torch(q, case.dtype), to_torch(k, case.dtype),
            to_torch(v, case.dtype), torch.from_numpy(cq).to(dev), torch.from_numpy(ck).to(dev))


def run_gpu(case, qt, kt, vt, cqt, ckt, max_q):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    out, lse = mfa.mfa_fwd_varlen(qt, kt, vt, cqt, ckt, max_q, scale=case.scale_f32(),
                                  causal=case.causal, window=(case.win_l, case.win_r),
                                  softcap=case.softcap)
    torch.cuda.synchronize()
    return from_torch(out), from_torch(lse)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_varlen_cases_match_oracle(cuda_device, case):
    import tiled_exact_attention_mfa_b200 as mfa
    q, k, v, cq, ck, qt, kt, vt, cqt, ckt = upload(case)
    nq, _ = case.lens()
    o, lse = run_gpu(case, qt, kt, vt, cqt, ckt, int(nq.max()))
    w = lambda x: mi.widen(x, case.dtype)
    o_ref, l_ref = oracle.attention_varlen(w(q), w(k), w(v), cq, ck, case.scale_f32(), case.causal,
                                           case.win_l, case.win_r, case.softcap)
    check_close(o, lse, o_ref, l_ref, case.dtype, case.name)
    assert mfa.mfa_device_status() == (0, 0)


def test_equal_lengths_match_dense_forward_bitwise(cuda_device):
    """With every sequence of length N, the packed forward is the dense forward in another
    layout: the same tiles and the same arithmetic, so bitwise the same O and LSE."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    # (no softcap here: its per-warp choice between two tanh forms looks at every score of a
    # tile, and past a sequence's end the packed layout holds the next sequence's keys where the
    # dense layout holds zeros, so the choice, not the accuracy, may differ)
    for causal, window, cap in ((True, (-1, -1), 0.0), (False, (70, 20), 0.0), (True, (100, 0), 0.0)):
        case = V("eq", 3, 4, 2, 128, mi.BF16, causal, fixed_q=[300] * 3, fixed_k=[300] * 3,
                 win_l=window[0], win_r=window[1], softcap=cap, seed=58)
        q, k, v, cq, ck, qt, kt, vt, cqt, ckt = upload(case)
        o_v, l_v = run_gpu(case, qt, kt, vt, cqt, ckt, 300)
        dense = lambda t: t.view(3, 300, t.shape[1], t.shape[2]).permute(0, 2, 1, 3).contiguous()
        o_d, l_d = mfa.mfa_fwd(dense(qt), dense(kt), dense(vt), scale=case.scale_f32(),
                               causal=causal, window=window, softcap=cap)
        torch.cuda.synchronize()
        o_d = from_torch(o_d.permute(0, 2, 1, 3).reshape(900, 4, 128))
        l_d = from_torch(l_d.permute(1, 0, 2).reshape(4, 900))
        assert np.array_equal(o_v, o_d), (causal, window, cap)
        assert np.array_equal(l_v, l_d), (causal, window, cap)


def test_full_size_varlen_workload_every_element(cuda_device):
    from oracle import cache
    case = mi.workloads()["varlen_causal_b8_h8_d128_fp16_len512_8k"]
    q, k, v, cq, ck, qt, kt, vt, cqt, ckt = upload(case)
    nq, _ = case.lens()
    o, lse = run_gpu(case, qt, kt, vt, cqt, ckt, int(nq.max()))
    ref = cache.reference(case.name, (q, k, v))
    check_close(o, lse, ref["o"], ref["lse"], case.dtype, case.name)


def test_malformed_offsets_are_reported_on_the_device(cuda_device):
    """Offsets live on the device, so the kernel checks them: a decreasing entry, an entry past
    the packed total, or a sequence longer than max_seqlen_q records the device status."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = SMALL[0]
    q, k, v, cq, ck, qt, kt, vt, cqt, ckt = upload(case)
    mfa.mfa_device_status()  # clear
    bad = cqt.clone()
    bad[2] = bad[1] - 5                       # decreasing
    mfa.mfa_fwd_varlen(qt, kt, vt, bad, ckt, 300)
    torch.cuda.synchronize()
    assert mfa.mfa_device_status()[0] == -24
    bad = ckt.clone()
    bad[-1] = kt.shape[0] + 128               # past the packed total of k
    mfa.mfa_fwd_varlen(qt, kt, vt, cqt, bad, 300)
    torch.cuda.synchronize()
    assert mfa.mfa_device_status()[0] == -24
    mfa.mfa_fwd_varlen(qt, kt, vt, cqt, ckt, 200)   # the first sequence holds 300 rows
    torch.cuda.synchronize()
    assert mfa.mfa_device_status()[0] == -24
    # a well-formed call afterwards runs clean
    o, lse = run_gpu(case, qt, kt, vt, cqt, ckt, 300)
    assert mfa.mfa_device_status() == (0, 0)
