"""Tensors past 2^31 elements: every offset the kernels form must be 64-bit.

Forward and backward run on q / k / v / out / dout / dq / dk / dv of 1 x 1,040 heads x 16,384
rows x 128 = 2.18e9 elements each (4.4 GB) under a causal window (64, 0); head h is the seeded
base head rotated by a head-dependent number of rows, so every head differs and a read from a
wrong head would show. The window makes a 512-row slice self-contained away from its first 64
rows (those rows' keys, and the rows that see its keys, lie inside the slice), so the fp64 oracle
runs on slices at the first and the last head, the last one past element 2^31.

Decode and chunked prefill read a page pool of 131,200 pages x 16 tokens x 8 kv heads x 128 =
2.15e9 elements per pool, with the sequences' pages at the far end of the pool (and one sequence
spread over both ends); unused slots hold NaN. The oracle sees a compact copy of the same pages.
"""
import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch

pytestmark = pytest.mark.gpu

H, N, D = 1040, 16384, 128
WIN = 64
SL = 512
ROT = (37, 53, 71, 89)  # rows of rotation per head for q, k, v, dout


def base(stream, seed=4242):
    return mi.normal_bits(seed, stream, (N, D), mi.FP16)


def head_np(b, rot, h):
    return np.roll(b, rot * h, axis=0)


def full_gpu(b, rot):
    import torch
    t = torch.from_numpy(b.view(np.int16)).view(torch.float16).cuda()
    idx = (torch.arange(N, device="cuda")[None, :] - rot * torch.arange(H, device="cuda")[:, None]) % N
    return t[idx][None]  # [1, H, N, D]: head h row i = base row (i - rot h) mod N


def test_forward_and_backward_past_2_31_elements(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    assert H * N * D > 2 ** 31
    bq, bk, bv, bd = base(mi.STREAM_Q), base(mi.STREAM_K), base(mi.STREAM_V), base(mi.STREAM_KEXTRA)
    q, k, v, do = (full_gpu(b, r) for b, r in zip((bq, bk, bv, bd), ROT))
    scale = float(np.float32(1.0 / np.sqrt(D)))
    win = (WIN, 0)
    out, lse = mfa.mfa_fwd(q, k, v, scale=scale, causal=True, window=win)
    dq, dk, dv = mfa.mfa_bwd(q, k, v, out, do, lse, scale=scale, causal=True, window=win)
    torch.cuda.synchronize()
    assert mfa.mfa_device_status() == (0, 0)
    w = lambda x: mi.widen(x, mi.FP16)
    tol = 4 * 2.0 ** -11
    for h in (0, H - 1):
        for s in (0, N - SL):
            sl = slice(s, s + SL)
            qs, ks, vs, ds = (w(head_np(b, r, h)[sl])[None, None] for b, r in zip((bq, bk, bv, bd), ROT))
            o_ref, l_ref = oracle.attention(qs, ks, vs, scale, True, WIN, 0)
            g_ref = oracle.attention_backward(qs, ks, vs, ds, scale, True, WIN, 0)
            r0 = 0 if s == 0 else WIN          # rows whose keys all lie in the slice
            rows = slice(r0, SL)
            check_close(from_torch(out[0, h, s + r0:s + SL]), from_torch(lse[0, h, s + r0:s + SL]),
                        o_ref[0, 0, rows], l_ref[0, 0, rows], mi.FP16, f"fwd h{h} s{s}")
            err = float(np.max(np.abs(from_torch(dq[0, h, s + r0:s + SL]) - g_ref[0][0, 0, rows])))
            assert err <= tol * float(np.max(np.abs(g_ref[0]))), (h, s, "dq", err)
            k0, k1 = r0, SL - WIN              # keys whose rows all lie in the slice
            for name, g, r in (("dk", dk, g_ref[1]), ("dv", dv, g_ref[2])):
                err = float(np.max(np.abs(from_torch(g[0, h, s + k0:s + k1]) - r[0, 0, k0:k1])))
                assert err <= tol * float(np.max(np.abs(r))), (h, s, name, err)


def test_decode_and_paged_prefill_on_a_pool_past_2_31_elements(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    Hq, Hkv, page = 32, 8, 16
    num_pages = 131200
    assert num_pages * page * Hkv * D > 2 ** 31
    lens = np.array([3000, 16, 1, 2049], dtype=np.int32)
    npg = (lens + page - 1) // page
    max_pages = int(npg.max())
    rng = np.random.default_rng(7)
    # pages from the last 1,000 of the pool in a shuffled order; sequence 3 alternates between
    # the first pages of the pool and the last ones
    high = rng.permutation(np.arange(num_pages - 1000, num_pages))
    table = np.full((4, max_pages), -1, dtype=np.int32)
    used = []
    hi_i = 0
    for b in range(4):
        for p in range(npg[b]):
            if b == 3 and p % 2 == 0:
                pid = p // 2
            else:
                pid = int(high[hi_i])
                hi_i += 1
            table[b, p] = pid
            used.append(pid)
    used = np.array(used)
    # compact pool for the oracle: page i of it is pool page used[i]
    kc = mi.normal_bits(77, mi.STREAM_K, (len(used), page, Hkv, D), mi.BF16)
    vc = mi.normal_bits(77, mi.STREAM_V, (len(used), page, Hkv, D), mi.BF16)
    remap = {int(pid): i for i, pid in enumerate(used)}
    table_c = np.where(table >= 0, np.vectorize(lambda x: remap.get(int(x), 0))(table), -1).astype(np.int32)
    kp = torch.full((num_pages, page, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vp = torch.full_like(kp, float("nan"))
    uidx = torch.from_numpy(used).long().cuda()
    kp[uidx] = torch.from_numpy(kc.view(np.int16)).view(torch.bfloat16).cuda()
    vp[uidx] = torch.from_numpy(vc.view(np.int16)).view(torch.bfloat16).cuda()
    scale = float(np.float32(1.0 / np.sqrt(D)))
    w = lambda x: mi.widen(x, mi.BF16)
    tt, lt = torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda()

    # decode, 2 query tokens per sequence
    qd = mi.normal_bits(78, mi.STREAM_Q, (4, Hq, 2, D), mi.BF16)
    qdt = torch.from_numpy(qd.view(np.int16)).view(torch.bfloat16).cuda()
    o, l = mfa.mfa_decode_splitkv(qdt, kp, vp, tt, lt, scale=scale, causal=True)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.decode(w(qd), w(kc), w(vc), table_c, lens, scale, True)
    check_close(from_torch(o), from_torch(l), o_ref, l_ref, mi.BF16, "decode")

    # chunked prefill: the last 100 / 16 / 1 / 300 positions of each sequence as query chunks
    nq = np.array([100, 16, 1, 300])
    cq = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    qp = mi.normal_bits(79, mi.STREAM_Q, (int(cq[-1]), Hq, D), mi.BF16)
    qpt = torch.from_numpy(qp.view(np.int16)).view(torch.bfloat16).cuda()
    o, l = mfa.mfa_fwd_paged(qpt, kp, vp, tt, lt, torch.from_numpy(cq).cuda(), int(nq.max()),
                             scale=scale, causal=True)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention_paged_prefill(w(qp), w(kc), w(vc), table_c, lens, cq, scale, True)
    check_close(from_torch(o), from_torch(l), o_ref, l_ref, mi.BF16, "paged prefill")
    assert mfa.mfa_device_status() == (0, 0)
