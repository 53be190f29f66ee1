"""Sharding one attention problem over the GPUs of a node (one process per GPU).

Host-side partitioning only; every step of the attention runs in libmfa.so's kernels.

Prefill: a forward problem is a set of independent units (b, g), one per sequence and kv head,
each owning the G = Hq / Hkv query heads that read kv head g ("mlx-bun 0.4.0 -> 1.0.0,
flash-attention.ts", forward shader: kv_head = head / reps). In the [B, H, N, D] layouts the
units are contiguous in b * Hkv + g order, so rank r takes a contiguous range of units, i.e. a
contiguous slice of q / k / v / out / lse, and runs the forward on it as the problem B' = its
unit count, Hq' = G, Hkv' = 1. No data crosses GPUs.

Decode: the splits of every sequence ("mlx-mfa 2.5.2", Features: Flash Decode two-phase
split-KV; "mxflashattn 1.4.0 -> 1.5.0", README: per-split (m, l) slots merged by a combine) are
cut into equal ranges of c = ceil(max_splits / world) splits; rank r holds the pages of splits
[r c, (r + 1) c) of each sequence and computes their partials (phase 1). The partial arrays are
split-major, so rank r's partials are one contiguous block; one all-gather (NCCL over NVLink) in
rank order gives every rank the arrays a single GPU computing all splits would hold, and the
combine runs on them. The exchange is B * Hq * Nq * (D + 2) * 4 bytes per split.
"""
from __future__ import annotations

import math


def unit_range(n_units: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous range [u0, u1) of rank `rank` among `world` ranks; sizes differ by at most 1,
    and the ranges of ranks 0 .. world - 1 tile [0, n_units) in order."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    return n_units * rank // world, n_units * (rank + 1) // world


def prefill_units(B: int, Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """The (b, g) units, numbered b * Hkv + g, of rank `rank`."""
    return unit_range(B * Hkv, world, rank)


def prefill_shard_views(q, k, v, out, lse, world: int, rank: int):
    """Views of rank `rank`'s slice: q / out [B, Hq, Nq, D] -> [u, G, Nq, D], k / v [B, Hkv, Nk, D]
    -> [u, 1, Nk, D], lse [B, Hq, Nq] -> [u, G, Nq] (u = the rank's unit count)."""
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    u0, u1 = prefill_units(B, Hkv, world, rank)
    qv = q.reshape(B * Hkv, G, Nq, D)[u0:u1]
    kv = k.reshape(B * Hkv, 1, Nk, D)[u0:u1]
    vv = v.reshape(B * Hkv, 1, Nk, D)[u0:u1]
    ov = out.reshape(B * Hkv, G, Nq, D)[u0:u1]
    lv = None if lse is None else lse.reshape(B * Hkv, G, Nq)[u0:u1]
    return qv, kv, vv, ov, lv


def fwd_sharded(q, k, v, out, lse, world: int, rank: int, **kw):
    """The forward of rank `rank`'s units, written into its slice of out / lse (the other ranks'
    slices are not touched). kw as mfa_fwd (scale, causal, window, softcap, stream)."""
    from . import mfa_fwd
    qv, kv, vv, ov, lv = prefill_shard_views(q, k, v, out, lse, world, rank)
    if qv.shape[0] == 0:
        return
    mfa_fwd(qv, kv, vv, ov, lv, **kw)


def split_chunk(max_splits: int, world: int) -> int:
    """Splits per rank: the plan's splits cut into `world` equal ranges (the last may be padded)."""
    return max(1, math.ceil(max_splits / world))


def split_range(max_splits: int, world: int, rank: int) -> tuple[int, int]:
    """Rank `rank`'s splits [s0, s1) of a decode plan with max_splits splits."""
    c = split_chunk(max_splits, world)
    return min(rank * c, max_splits), min((rank + 1) * c, max_splits)


def split_pages(plan: dict, seq_len: int, split: int, win_l: int = -1, Nq: int = 1) -> range:
    """Logical pages of a sequence that one split covers (the pages its owner must hold): from
    the sequence's first visible page (a left window moves it), pages_per_split per split."""
    n_pages = -(-int(seq_len) // 16)
    first = 0 if win_l < 0 else max(0, int(seq_len) - Nq - win_l) // 16
    p0 = first + split * plan["pages_per_split"]
    return range(min(p0, n_pages), min(p0 + plan["pages_per_split"], n_pages))


def decode_partial_shapes(B: int, Nq: int, Hq: int, D: int, max_splits: int, world: int):
    """Shapes of (part_o, part_ml) for `world` ranks: split capacity c * world (split-major)."""
    cap = split_chunk(max_splits, world) * world
    return (cap, B, Hq * Nq, D), (cap, B, Hq * Nq, 2)


def decode_sharded(q, k_pages, v_pages, block_table, seq_lens, out, lse, part_o, part_ml,
                   world: int, rank: int, group=None, *, scale=None, causal=True, softcap=0.0,
                   win_l=-1, stream=None):
    """Split-KV decode with the splits spread over the ranks of `group`: phase 1 over this rank's
    splits, an all-gather of the partial blocks, then the combine (every rank gets out / lse).
    part_o / part_ml: float32 device tensors of decode_partial_shapes(...). Everything is queued
    on torch's current stream (enter torch.cuda.stream(s) to use another), where the collective
    runs too; `stream` is accepted for symmetry and must be None or that current stream."""
    import torch
    if stream is not None and stream != torch.cuda.current_stream():
        raise ValueError("decode_sharded runs on the current stream; use torch.cuda.stream(s)")
    import torch.distributed as dist
    from . import mfa_decode_combine, mfa_decode_phase1, mfa_decode_plan
    B, Hq, Nq, D = q.shape
    Hkv = k_pages.shape[2]
    plan = mfa_decode_plan(B, Nq, Hq, Hkv, D, block_table.shape[1], 16, win_l)
    c = split_chunk(plan["max_splits"], world)
    if part_o.shape[0] != c * world or part_ml.shape[0] != c * world:
        raise ValueError("partial buffers must hold ceil(max_splits / world) * world splits")
    s0, s1 = split_range(plan["max_splits"], world, rank)
    mfa_decode_phase1(q, k_pages, v_pages, block_table, seq_lens, part_o, part_ml, s0, s1,
                      scale=scale, causal=causal, softcap=softcap, win_l=win_l, stream=stream)
    if world > 1:
        blk = slice(rank * c, (rank + 1) * c)
        dist.all_gather_into_tensor(part_o, part_o[blk].clone(), group=group)
        dist.all_gather_into_tensor(part_ml, part_ml[blk].clone(), group=group)
    mfa_decode_combine(seq_lens, part_o, part_ml, out, lse, Hkv=Hkv,
                       max_pages_per_seq=block_table.shape[1], win_l=win_l, stream=stream)
    return out, lse
