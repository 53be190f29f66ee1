"""Sharding one problem over ranks (tiled_exact_attention_mfa_b200.shard), on CPU with gloo.

No GPU here, so what runs on each rank is the fp64 oracle (prefill) or a NumPy restatement of
the decode's phase-1 partials and combine (decode); what is under test is the host logic the GPU
path uses: which units / splits a rank owns, that the ranks' pieces tile the problem exactly
once, and that the all-gather of the split-major partial blocks in rank order rebuilds the
arrays a single process computing every split holds, whose combine is the oracle's decode.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import mfa_inputs as mi
import oracle
from tiled_exact_attention_mfa_b200 import mfa_decode_plan, shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("n_units", [1, 2, 7, 16, 32, 33])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_unit_ranges_tile_the_units_once_in_order(n_units, world):
    seen = []
    for r in range(world):
        u0, u1 = shard.unit_range(n_units, world, r)
        assert u1 - u0 in (n_units // world, -(-n_units // world))
        seen += list(range(u0, u1))
    assert seen == list(range(n_units))


@pytest.mark.parametrize("max_splits", [1, 5, 16, 256, 257])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_split_ranges_are_equal_blocks_covering_every_split_once(max_splits, world):
    c = shard.split_chunk(max_splits, world)
    seen = []
    for r in range(world):
        s0, s1 = shard.split_range(max_splits, world, r)
        assert s0 == min(r * c, max_splits) and s1 - s0 <= c
        seen += list(range(s0, s1))
    assert seen == list(range(max_splits))
    po, pm = shard.decode_partial_shapes(3, 2, 8, 64, max_splits, world)
    assert po[0] == pm[0] == c * world >= max_splits


def test_split_pages_cover_each_sequence_once():
    plan = mfa_decode_plan(4, 1, 8, 2, 64, 200)
    for L in (0, 1, 16, 17, 3000, 3200):
        for win in (-1, 0, 100, 5000):
            pages = []
            for s in range(plan["max_splits"]):
                pages += list(shard.split_pages(plan, L, s, win_l=win))
            n = -(-L // 16)
            first = 0 if win < 0 else max(0, L - 1 - win) // 16
            assert pages == list(range(first, n)), (L, win)


# ------------------------------------------------------------------ prefill over 2 gloo ranks
PCASE = mi.PrefillCase("shard_gqa", 3, 8, 2, 200, 260, 64, mi.FP16, True, 50, -1, softcap=20.0,
                       seed=91)


def _prefill_rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    c = PCASE
    q, k, v = (mi.widen(x, c.dtype) for x in c.tensors())
    o = np.zeros(q.shape)
    lse = np.full(q.shape[:3], -np.inf)
    qv, kv, vv, ov, lv = shard.prefill_shard_views(q, k, v, o, lse, world, rank)
    so, sl = oracle.attention(qv, kv, vv, c.scale_f32(), c.causal, c.win_l, c.win_r, c.softcap)
    ov[...] = so
    lv[...] = sl
    # every rank contributes its slice; the others' slices of its arrays are still empty
    u0, u1 = shard.prefill_units(c.B, c.Hkv, world, rank)
    G = c.Hq // c.Hkv
    flat_o = torch.from_numpy(o.reshape(c.B * c.Hkv, -1))
    pieces = [torch.zeros_like(flat_o) for _ in range(world)]
    dist.all_gather(pieces, flat_o)
    full = sum(p for p in pieces)  # disjoint slices: the sum is their union
    mine = np.zeros(c.B * c.Hkv, dtype=bool)
    mine[u0:u1] = True
    out.put((rank, full.numpy(), mine, bool(np.all(o.reshape(c.B * c.Hkv, -1)[~mine] == 0)), G))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_prefill_shards_rebuild_the_whole_forward():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_prefill_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    c = PCASE
    qq, kk, vv = (mi.widen(x, c.dtype) for x in c.tensors())
    ref, _ = oracle.attention(qq, kk, vv, c.scale_f32(), c.causal, c.win_l, c.win_r, c.softcap)
    masks = [m for _, _, m, _, _ in res]
    assert not np.any(masks[0] & masks[1]) and np.all(masks[0] | masks[1])
    for _, full, _, untouched, _ in res:
        assert untouched                       # a rank wrote only its own units
        assert np.array_equal(full.reshape(ref.shape), ref)


# ------------------------------------------------------------------ decode over 2 gloo ranks
DCASE = mi.DecodeCase("shard_decode", 3, 2, 8, 2, 64, mi.BF16, 1, 2500, win_l=-1, seed=92,
                      max_pages=160)


def _phase1_partials(case, q, kp, vp, table, lens, plan, splits, cap, win_l=-1):
    """Partials of the given splits, as the phase-1 kernel defines them: per (split, sequence,
    query row) the running max m of the split's visible scores in log2 units, l = sum 2^(s c - m)
    and o = sum 2^(s c - m) v (c = scale log2 e), in the split-major layout."""
    B, Hq, Nq, D = q.shape
    Hkv = kp.shape[2]
    G = Hq // Hkv
    c = case.scale_f32() * np.log2(np.e)
    po = np.zeros((cap, B, Hq * Nq, D))
    pm = np.zeros((cap, B, Hq * Nq, 2))
    for s in splits:
        for b in range(B):
            L = int(lens[b])
            pages = shard.split_pages(plan, L, s, win_l=win_l, Nq=Nq)
            if len(pages) == 0:
                continue
            toks = np.arange(pages.start * 16, min(pages.stop * 16, L))
            pg = table[b][toks // 16]
            for h in range(Hq):
                g = h // G
                kb = kp[pg, toks % 16, g]
                vb = vp[pg, toks % 16, g]
                for t in range(Nq):
                    a = L - Nq + t
                    vis = toks <= a if case.causal else np.ones(len(toks), bool)
                    if win_l >= 0:
                        vis &= toks >= a - win_l
                    x = np.where(vis, (kb @ q[b, h, t]) * c, -np.inf)  # scores in log2 units
                    m = np.max(x) if vis.any() else -np.inf
                    w = np.where(vis, np.exp2(x - (m if np.isfinite(m) else 0.0)), 0.0)
                    row = h * Nq + t
                    po[s, b, row] = w @ vb
                    pm[s, b, row] = (m, w.sum())
    return po, pm


def _combine(po, pm, lens, plan, Nq, win_l=-1):
    """O = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over each sequence's splits."""
    cap, B, R, D = po.shape
    out = np.zeros((B, R, D))
    lse = np.full((B, R), -np.inf)
    for b in range(B):
        L = int(lens[b])
        n_pages = -(-L // 16)
        first = 0 if win_l < 0 else max(0, L - Nq - win_l) // 16
        n_splits = -(-(n_pages - first) // plan["pages_per_split"])
        m = pm[:n_splits, b, :, 0]
        M = np.max(m, axis=0)
        ok = np.isfinite(M)
        wgt = np.where(np.isfinite(m), np.exp2(m - np.where(ok, M, 0.0)), 0.0)
        Lsum = np.sum(wgt * pm[:n_splits, b, :, 1], axis=0)
        out[b] = np.where(ok[:, None], np.einsum("sr,srd->rd", wgt, po[:n_splits, b]) /
                          np.where(ok, Lsum, 1.0)[:, None], 0.0)
        lse[b] = np.where(ok, (M + np.log2(np.where(ok, Lsum, 1.0))) * np.log(2.0), -np.inf)
    return out, lse


def _decode_rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    c = DCASE
    qb, kb, vb, table, lens = c.tensors()
    q, kp, vp = (mi.widen(x, c.dtype) for x in (qb, kb, vb))
    plan = mfa_decode_plan(c.B, c.Nq, c.Hq, c.Hkv, c.D, table.shape[1], 16, c.win_l)
    po_shape, _ = shard.decode_partial_shapes(c.B, c.Nq, c.Hq, c.D, plan["max_splits"], world)
    cap = po_shape[0]
    s0, s1 = shard.split_range(plan["max_splits"], world, rank)
    po, pm = _phase1_partials(c, q, kp, vp, table, lens, plan, range(s0, s1), cap)
    blk = slice(rank * (cap // world), (rank + 1) * (cap // world))
    to, tm = torch.from_numpy(po), torch.from_numpy(pm)
    dist.all_gather_into_tensor(to, to[blk].clone())
    dist.all_gather_into_tensor(tm, tm[blk].clone())
    out.put((rank, to.numpy(), tm.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_decode_gather_rebuilds_single_gpu_partials_and_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decode_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    c = DCASE
    qb, kb, vb, table, lens = c.tensors()
    q, kp, vp = (mi.widen(x, c.dtype) for x in (qb, kb, vb))
    plan = mfa_decode_plan(c.B, c.Nq, c.Hq, c.Hkv, c.D, table.shape[1], 16, c.win_l)
    assert plan["max_splits"] > 2  # the sequences really are split over both ranks
    cap = res[0][1].shape[0]
    po1, pm1 = _phase1_partials(c, q, kp, vp, table, lens, plan, range(plan["max_splits"]), cap)
    for _, po, pm in res:
        # every slot the combine reads is the single-process value, bit for bit
        for b in range(c.B):
            n = -(-(-(-int(lens[b]) // 16)) // plan["pages_per_split"])
            assert np.array_equal(po[:n, b], po1[:n, b]) and np.array_equal(pm[:n, b], pm1[:n, b])
        o, lse = _combine(po, pm, lens, plan, c.Nq)
        ro, rl = oracle.decode(q, kp, vp, table, lens, c.scale_f32(), c.causal, c.softcap)
        assert np.max(np.abs(o.reshape(ro.shape) - ro)) < 1e-12
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(lse.reshape(rl.shape)), fin)
        assert np.max(np.abs(lse.reshape(rl.shape)[fin] - rl[fin])) < 1e-12
