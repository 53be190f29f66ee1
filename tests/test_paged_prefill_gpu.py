"""GPU parity of mfa_fwd_paged (chunked prefill of packed query chunks over a paged KV cache,
through the C ABI) against the fp64 oracle on seeded inputs. Page slots past each sequence's
length and unused pages hold NaN, so any read of them that reached the arithmetic would show."""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu

PP = mi.PagedPrefillCase
CASES = [
    PP("causal_chunks_fp16", 4, 4, 2, 128, mi.FP16, 1, 700, q_hi=300, seed=81),
    PP("causal_gqa4_bf16", 3, 8, 2, 128, mi.BF16, 100, 1500, q_hi=600, seed=82),
    PP("noncausal_d64_fp16", 3, 2, 2, 64, mi.FP16, 1, 400, q_hi=400, causal=False, seed=83),
    PP("window_softcap_bf16", 2, 4, 4, 128, mi.BF16, 300, 900, q_hi=400, win_l=200, win_r=0,
       softcap=30.0, seed=84),
    PP("edge_lengths_fp16", 5, 2, 1, 128, mi.FP16, 1, 1, fixed_lens=[1, 16, 17, 128, 129],
       fixed_q=[1, 16, 5, 128, 129], seed=85),
    PP("empty_sequence_bf16", 3, 2, 2, 64, mi.BF16, 1, 1, fixed_lens=[0, 50, 300],
       fixed_q=[0, 50, 100], seed=86),
]


def run_gpu(case, q, kp, vp, table, lens, cq):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    dev = torch.device("cuda")
    out, lse = mfa.mfa_fwd_paged(to_torch(q, case.dtype), to_torch(kp, case.dtype),
                                 to_torch(vp, case.dtype), torch.from_numpy(table).to(dev),
                                 torch.from_numpy(lens).to(dev), torch.from_numpy(cq).to(dev),
                                 int(max(1, np.max(np.diff(cq)))), scale=case.scale_f32(),
                                 causal=case.causal, window=(case.win_l, case.win_r),
                                 softcap=case.softcap)
    torch.cuda.synchronize()
    return from_torch(out), from_torch(lse)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_paged_prefill_matches_oracle(cuda_device, case):
    import tiled_exact_attention_mfa_b200 as mfa
    q, kp, vp, table, lens, cq = case.tensors()
    o, lse = run_gpu(case, q, kp, vp, table, lens, cq)
    w = lambda x: mi.widen(x, case.dtype)
    o_ref, l_ref = oracle.attention_paged_prefill(w(q), w(kp), w(vp), table, lens, cq,
                                                  case.scale_f32(), case.causal, case.win_l,
                                                  case.win_r, case.softcap)
    check_close(o, lse, o_ref, l_ref, case.dtype, case.name)
    assert mfa.mfa_device_status() == (0, 0)


def test_full_size_paged_prefill_every_element(cuda_device):
    """The chunked-prefill workload (8 sequences, 4k-32k cached keys in a permuted page pool,
    chunks of up to 2048 queries) against the oracle, every element (cached)."""
    import tiled_exact_attention_mfa_b200 as mfa
    from oracle import cache
    case = mi.workloads()["paged_prefill_b8_hq32_hkv8_d128_bf16_ctx4k_32k"]
    q, kp, vp, table, lens, cq = case.tensors()
    o, lse = run_gpu(case, q, kp, vp, table, lens, cq)
    ref = cache.reference(case.name, (q, kp, vp, table, lens, cq))
    check_close(o, lse, ref["o"], ref["lse"], case.dtype, case.name)
    assert mfa.mfa_device_status() == (0, 0)


def test_short_chunks_equal_split_kv_decode(cuda_device):
    """With 1-4 queries per sequence, the paged prefill and the split-KV decode compute the same
    definition: both within the tolerance of the oracle and of each other."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = PP("short", 4, 8, 2, 128, mi.BF16, 200, 2000, fixed_q=[3, 3, 3, 3], seed=87)
    q, kp, vp, table, lens, cq = case.tensors()
    o_p, l_p = run_gpu(case, q, kp, vp, table, lens, cq)
    dev = torch.device("cuda")
    qd = to_torch(q, case.dtype).view(4, 3, 8, 128).permute(0, 2, 1, 3).contiguous()
    o_d, l_d = mfa.mfa_decode_splitkv(qd, to_torch(kp, case.dtype), to_torch(vp, case.dtype),
                                      torch.from_numpy(table).to(dev), torch.from_numpy(lens).to(dev),
                                      scale=case.scale_f32(), causal=True)
    torch.cuda.synchronize()
    o_d = from_torch(o_d.permute(0, 2, 1, 3).reshape(12, 8, 128))
    l_d = from_torch(l_d.permute(1, 0, 2).reshape(8, 12))
    check_close(o_p, l_p, o_d, l_d, case.dtype, "paged prefill vs decode")


def test_page_order_is_irrelevant(cuda_device):
    """The same cache in two page orders (the seeded permutation vs the identity) gives bitwise
    the same output."""
    import tiled_exact_attention_mfa_b200 as mfa
    case = PP("perm", 3, 4, 2, 128, mi.FP16, 100, 800, q_hi=300, seed=88)
    q, kp, vp, table, lens, cq = case.tensors()
    o1, l1 = run_gpu(case, q, kp, vp, table, lens, cq)
    num = kp.shape[0]
    order = np.argsort(table[table >= 0])  # a different arrangement of the used pages
    used = table[table >= 0]
    remap = np.arange(num)
    remap[used] = used[order]
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[remap] = kp
    vp2[remap] = vp
    table2 = np.where(table >= 0, remap[np.maximum(table, 0)], -1).astype(np.int32)
    o2, l2 = run_gpu(case, q, kp2, vp2, table2, lens, cq)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    assert mfa.mfa_device_status() == (0, 0)
