"""GPU parity of mfa_decode_splitkv (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu

Dc = mi.DecodeCase
SMALL = [
    Dc("nq1_gqa4_d128_bf16", 3, 1, 32, 8, 128, mi.BF16, 1, 700, seed=51),
    Dc("nq4_gqa4_d128_bf16", 3, 4, 16, 4, 128, mi.BF16, 1, 300, seed=52),
    Dc("nq2_gqa2_d64_fp16", 4, 2, 8, 4, 64, mi.FP16, 1, 2000, seed=53),
    Dc("nq3_mha_d64_fp16", 2, 3, 4, 4, 64, mi.FP16, 1, 90, seed=54),
    Dc("nq1_gqa16_d128_fp16", 2, 1, 32, 2, 128, mi.FP16, 1, 3000, seed=55),
    Dc("edge_lengths_bf16", 6, 1, 8, 2, 128, mi.BF16, 0, 0, fixed_lens=[1, 16, 17, 0, 31, 513],
       max_pages=40, seed=56),
    Dc("nq4_short_lengths_causal_fp16", 4, 4, 8, 8, 64, mi.FP16, 0, 0, fixed_lens=[1, 2, 3, 5],
       seed=57, max_pages=2),
    Dc("noncausal_nq2_bf16", 2, 2, 8, 2, 128, mi.BF16, 1, 500, causal=False, seed=58),
    Dc("softcap30_bf16", 2, 1, 16, 4, 128, mi.BF16, 100, 900, softcap=30.0, seed=59),
    Dc("more_than_8_kv_heads_fp16", 2, 1, 32, 16, 64, mi.FP16, 50, 400, seed=60),
    # left sliding window: spans that begin mid-page and several splits into the sequence
    Dc("window100_nq1_gqa4_bf16", 4, 1, 32, 8, 128, mi.BF16, 1, 2000, win_l=100, seed=65),
    Dc("window30_nq4_fp16", 3, 4, 16, 4, 64, mi.FP16, 40, 900, win_l=30, seed=66),
    Dc("window0_nq3_bf16", 2, 3, 8, 2, 128, mi.BF16, 5, 300, win_l=0, seed=67),
    Dc("window_longer_than_seq_fp16", 3, 2, 8, 4, 128, mi.FP16, 1, 700, win_l=5000, seed=68),
    Dc("window_noncausal_softcap_bf16", 2, 2, 16, 4, 128, mi.BF16, 200, 1500, causal=False,
       softcap=30.0, win_l=250, seed=69),
    Dc("window_edge_lengths_fp16", 6, 1, 8, 2, 64, mi.FP16, 0, 0,
       fixed_lens=[1, 16, 17, 0, 33, 513], max_pages=40, win_l=16, seed=70),
    # a window of INT_MAX (a common "no window" sentinel) over sequences shorter than N_q: the
    # position arithmetic must not wrap around, every row sees its whole causal prefix
    Dc("window_int_max_short_lens_bf16", 5, 4, 8, 2, 128, mi.BF16, 0, 0,
       fixed_lens=[0, 1, 2, 3, 40], max_pages=4, win_l=2 ** 31 - 1, seed=71),
    # D = 256: two kv heads per CTA when Hkv is even, one otherwise
    Dc("d256_nq1_gqa4_bf16", 3, 1, 16, 4, 256, mi.BF16, 1, 1500, seed=72),
    Dc("d256_nq4_gqa4_window_fp16", 2, 4, 8, 2, 256, mi.FP16, 100, 900, win_l=200, seed=73),
    Dc("d256_nq2_softcap_bf16", 2, 2, 8, 4, 256, mi.BF16, 1, 600, softcap=30.0, seed=74),
    Dc("d256_odd_kv_heads_fp16", 2, 1, 6, 3, 256, mi.FP16, 1, 700, seed=75),
    Dc("d256_edge_lengths_noncausal_bf16", 5, 3, 4, 4, 256, mi.BF16, 0, 0, causal=False,
       fixed_lens=[1, 16, 0, 17, 300], max_pages=20, seed=76),
]


def run_gpu(case, q, k, v, table, lens, split_pages=0):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    old = mfa.mfa_debug_set_decode_split_pages(split_pages)
    try:
        out, lse = mfa.mfa_decode_splitkv(
            to_torch(q, case.dtype), to_torch(k, case.dtype), to_torch(v, case.dtype),
            torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda(),
            scale=case.scale_f32(), causal=case.causal, softcap=case.softcap, win_l=case.win_l)
    finally:
        mfa.mfa_debug_set_decode_split_pages(old)
    torch.cuda.synchronize()
    return from_torch(out), from_torch(lse)


def oracle_full(case, q, k, v, table, lens):
    w = lambda x: mi.widen(x, case.dtype)
    return oracle.decode(w(q), w(k), w(v), table, lens, case.scale_f32(), case.causal, case.softcap,
                         win_l=case.win_l)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_cases_match_oracle(cuda_device, case):
    q, k, v, table, lens = case.tensors()
    o, lse = run_gpu(case, q, k, v, table, lens)
    o_ref, lse_ref = oracle_full(case, q, k, v, table, lens)
    check_close(o, lse, o_ref, lse_ref, case.dtype, case.name)
    import tiled_exact_attention_mfa_b200 as mfa
    assert mfa.mfa_device_status() == (0, 0)


@pytest.mark.parametrize("name", sorted(n for n, c in mi.workloads().items()
                                         if isinstance(c, mi.DecodeCase)))
def test_full_size_every_element(cuda_device, name):
    """Every output row of a full-size decode workload against the oracle (cached)."""
    from oracle import cache
    case = mi.workloads()[name]
    q, k, v, table, lens = case.tensors()
    o, lse = run_gpu(case, q, k, v, table, lens)
    ref = cache.reference(name, (q, k, v, table, lens))
    check_close(o, lse, ref["o"], ref["lse"], case.dtype, case.name)
    import tiled_exact_attention_mfa_b200 as mfa
    assert mfa.mfa_device_status() == (0, 0)


def test_page_permutation_is_bitwise_neutral(cuda_device):
    """Same logical K/V, identity page order vs a permuted pool: bitwise equal at a fixed plan."""
    base = Dc("perm", 3, 2, 16, 4, 128, mi.BF16, 200, 1500, seed=61)
    q, k, v, table, lens = base.tensors()
    o1, l1 = run_gpu(base, q, k, v, table, lens)
    ident = np.full_like(table, -1)
    perm_pool_k = np.empty_like(k)
    perm_pool_v = np.empty_like(v)
    nxt = 0
    for b in range(base.B):
        n = -(-int(lens[b]) // 16)
        ident[b, :n] = np.arange(nxt, nxt + n)
        perm_pool_k[nxt:nxt + n] = k[table[b, :n]]
        perm_pool_v[nxt:nxt + n] = v[table[b, :n]]
        nxt += n
    o2, l2 = run_gpu(base, q, perm_pool_k[:nxt], perm_pool_v[:nxt], ident, lens)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_split_size_changes_only_rounding(cuda_device):
    case = Dc("split", 2, 1, 32, 8, 128, mi.BF16, 3000, 5000, seed=62)
    q, k, v, table, lens = case.tensors()
    ref = oracle_full(case, q, k, v, table, lens)
    outs = [run_gpu(case, q, k, v, table, lens, split_pages=s) for s in (1, 4, 32)]
    for o, lse in outs:
        check_close(o, lse, *ref, case.dtype, "split")
    assert np.max(np.abs(outs[0][1] - outs[2][1])) < 1e-4


def test_decode_equals_prefill_on_gathered_cache(cuda_device):
    """Decode of Nq query tokens == the dense forward on the gathered K/V (bottom-right causal)."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = Dc("eq", 2, 4, 16, 4, 128, mi.FP16, 600, 900, seed=63)
    q, k, v, table, lens = case.tensors()
    o, lse = run_gpu(case, q, k, v, table, lens)
    for b in range(case.B):
        L = int(lens[b])
        t = np.arange(L)
        kb = k[table[b, t // 16], t % 16].transpose(1, 0, 2)[None].copy()
        vb = v[table[b, t // 16], t % 16].transpose(1, 0, 2)[None].copy()
        of, lf = mfa.mfa_fwd(to_torch(q[b:b + 1], case.dtype), to_torch(kb, case.dtype),
                             to_torch(vb, case.dtype), scale=case.scale_f32(), causal=True)
        torch.cuda.synchronize()
        assert np.max(np.abs(from_torch(of)[0] - o[b])) <= 4e-3
        assert np.max(np.abs(from_torch(lf)[0] - lse[b])) <= 1e-4


def test_out_of_range_entries_are_reported_not_read(cuda_device):
    """A block_table entry outside the pool and a too-long seq_lens entry set the device
    status; the kernel skips the copy instead of reading outside the pool."""
    import tiled_exact_attention_mfa_b200 as mfa
    mfa.mfa_device_status()  # clear
    case = Dc("bad", 2, 1, 8, 2, 64, mi.FP16, 0, 0, fixed_lens=[40, 20], max_pages=3, seed=64)
    q, k, v, table, lens = case.tensors()
    bad = table.copy()
    bad[0, 1] = 10_000_000
    run_gpu(case, q, k, v, bad, lens)
    code, _ = mfa.mfa_device_status()
    assert code == -22
    lens2 = lens.copy()
    lens2[1] = 3 * 16 + 5
    run_gpu(case, q, k, v, table, lens2)
    code, _ = mfa.mfa_device_status()
    assert code == -22
    assert mfa.mfa_device_status() == (0, 0)


def test_window_split_size_changes_only_rounding(cuda_device):
    """The splits left of the window are skipped whole; the result does not depend on where the
    split boundaries fall relative to the window's first token."""
    case = Dc("wsplit", 2, 2, 32, 8, 128, mi.BF16, 3000, 5000, win_l=700, seed=71)
    q, k, v, table, lens = case.tensors()
    ref = oracle_full(case, q, k, v, table, lens)
    for s in (1, 3, 8, 32):
        o, lse = run_gpu(case, q, k, v, table, lens, split_pages=s)
        check_close(o, lse, *ref, case.dtype, f"wsplit{s}")


def test_window_minus_one_is_the_plain_decode(cuda_device):
    """win_l = -1 through the window entry point is bitwise the plain decode; a window covering
    the whole sequence differs from it only by rounding."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = SMALL[0]
    q, k, v, table, lens = case.tensors()
    args = (to_torch(q, case.dtype), to_torch(k, case.dtype), to_torch(v, case.dtype),
            torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda())
    o1, l1 = mfa.mfa_decode_splitkv(*args, scale=case.scale_f32())
    ws = torch.empty(mfa.mfa_decode_workspace_size(q.shape[0], q.shape[2], q.shape[1], k.shape[2], case.D,
                                              table.shape[1]),
                     dtype=torch.uint8, device="cuda")
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    rc = mfa.lib.mfa_decode_splitkv_window(
        mfa._ptr(args[0]), mfa._ptr(args[1]), mfa._ptr(args[2]), mfa._ptr(args[3]),
        mfa._ptr(args[4]), mfa._ptr(o2), mfa._ptr(l2), q.shape[0], q.shape[2], q.shape[1],
        k.shape[2], case.D, 16, table.shape[1], k.shape[0], case.scale_f32(), 1, -1, 0.0,
        mfa._dtype_code(args[0]), mfa._ptr(ws), ws.numel(), mfa._stream(None))
    assert rc == 0
    o3, l3 = mfa.mfa_decode_splitkv(*args, scale=case.scale_f32(), win_l=100000)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert float((o1.float() - o3.float()).abs().max()) <= 1.6e-2
    assert float((l1 - l3).abs().max()) <= 1e-4
    assert mfa.mfa_device_status() == (0, 0)
