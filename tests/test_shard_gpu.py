"""The sharded paths on one GPU, through the C ABI: the ranks' pieces computed one after another
(no kernel waits on another) must give what the unsharded call gives.

  * prefill: every rank's forward over its (sequence, kv-head) units, into one output, is
    bitwise the whole forward;
  * decode: phase 1 over each rank's block of splits -- with a page pool in which every page the
    rank does not own is NaN, so a read outside its pages would show -- into the split-major
    partial buffers, then the combine, is bitwise the one-call split-KV decode, and within the
    tolerances of the oracle.
"""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3, 5])
def test_prefill_shards_are_bitwise_the_whole_forward(cuda_device, world):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    from tiled_exact_attention_mfa_b200 import shard
    case = mi.PrefillCase("shard", 2, 8, 4, 700, 900, 128, mi.BF16, True, 300, -1, softcap=30.0,
                          seed=95)
    qt, kt, vt = (to_torch(x, case.dtype) for x in case.tensors())
    kw = dict(scale=case.scale_f32(), causal=case.causal, window=(case.win_l, case.win_r),
              softcap=case.softcap)
    o_ref, l_ref = mfa.mfa_fwd(qt, kt, vt, **kw)
    out = torch.full_like(o_ref, float("nan"))
    lse = torch.full_like(l_ref, float("nan"))
    for r in range(world):
        shard.fwd_sharded(qt, kt, vt, out, lse, world, r, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)


@pytest.mark.parametrize("world,win_l", [(2, -1), (3, -1), (4, 700)])
def test_decode_splits_over_ranks_are_bitwise_the_one_call_decode(cuda_device, world, win_l):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    from tiled_exact_attention_mfa_b200 import shard
    case = mi.DecodeCase("shard_dec", 4, 2, 16, 4, 128, mi.BF16, 1, 6000, win_l=win_l, seed=96)
    q, kp, vp, table, lens = case.tensors()
    qt = to_torch(q, case.dtype)
    tt, lt = torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda()
    kw = dict(scale=case.scale_f32(), causal=case.causal, softcap=case.softcap, win_l=win_l)
    o_ref, l_ref = mfa.mfa_decode_splitkv(qt, to_torch(kp, case.dtype), to_torch(vp, case.dtype),
                                          tt, lt, **kw)
    plan = mfa.mfa_decode_plan(case.B, case.Nq, case.Hq, case.Hkv, case.D, table.shape[1], 16, win_l)
    assert plan["max_splits"] >= world  # every rank owns some splits
    so, sm = shard.decode_partial_shapes(case.B, case.Nq, case.Hq, case.D, plan["max_splits"], world)
    po = torch.full(so, float("nan"), dtype=torch.float32, device="cuda")
    pm = torch.full(sm, float("nan"), dtype=torch.float32, device="cuda")
    nan = np.uint16(mi.NAN_BITS[case.dtype])
    for r in range(world):
        s0, s1 = shard.split_range(plan["max_splits"], world, r)
        own = np.zeros(kp.shape[0], dtype=bool)
        for b in range(case.B):
            for s in range(s0, s1):
                pages = shard.split_pages(plan, int(lens[b]), s, win_l=win_l, Nq=case.Nq)
                own[table[b, pages.start:pages.stop]] = True
        kr, vr = kp.copy(), vp.copy()
        kr[~own] = nan
        vr[~own] = nan
        mfa.mfa_decode_phase1(qt, to_torch(kr, case.dtype), to_torch(vr, case.dtype), tt, lt, po, pm,
                              s0, s1, **kw)
        torch.cuda.synchronize()  # this rank's pool copies may be freed now
    out = torch.empty_like(o_ref)
    lse = torch.empty_like(l_ref)
    mfa.mfa_decode_combine(lt, po, pm, out, lse, Hkv=case.Hkv, max_pages_per_seq=table.shape[1],
                           win_l=win_l)
    torch.cuda.synchronize()
    assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)
    w = lambda x: mi.widen(x, case.dtype)
    ro, rl = oracle.decode(w(q), w(kp), w(vp), table, lens, case.scale_f32(), case.causal,
                           case.softcap, win_l=win_l)
    check_close(from_torch(out), from_torch(lse), ro, rl, case.dtype, "decode over split ranges")
    assert mfa.mfa_device_status() == (0, 0)


def test_phase1_and_combine_reject_bad_split_ranges_and_capacity(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = mi.DecodeCase("shard_bad", 2, 1, 8, 2, 64, mi.FP16, 100, 900, seed=97)
    q, kp, vp, table, lens = case.tensors()
    qt, kt, vt = (to_torch(x, case.dtype) for x in (q, kp, vp))
    tt, lt = torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda()
    plan = mfa.mfa_decode_plan(case.B, 1, 8, 2, 64, table.shape[1])
    S = plan["max_splits"]
    po = torch.empty(S, 2, 8, 64, device="cuda")
    pm = torch.empty(S, 2, 8, 2, device="cuda")
    for lo, hi in ((-1, 1), (2, 1), (0, S + 1)):
        with pytest.raises(mfa.MFAError) as e:
            mfa.mfa_decode_phase1(qt, kt, vt, tt, lt, po, pm, lo, hi)
        assert e.value.code == -5
    with pytest.raises(mfa.MFAError) as e:
        mfa.mfa_decode_phase1(qt, kt, vt, tt, lt, po[:S - 1], pm[:S - 1], 0, 1)
    assert e.value.code == -12
    with pytest.raises(mfa.MFAError) as e:
        mfa.mfa_decode_combine(lt, po[:S - 1], pm[:S - 1], torch.empty_like(qt), Hkv=2,
                               max_pages_per_seq=table.shape[1])
    assert e.value.code == -12
