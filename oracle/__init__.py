"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package: only the tests,
the smoke check and the bench's CPU-baseline / reference arm may call it. It shares no code
with the CUDA library and never reads anything the CUDA path produced.

What it computes is the plain definition that the tiled online-softmax forward reaches exactly
(up to rounding order): for every query row an explicit score vector over all keys, a
visibility mask, a softmax and a weighted sum of value rows, all in fp64.

Sources (web pages, cited by title and section):
  * "mlx-bun 0.4.0 -> 1.0.0, src/model/flash-attention.ts" (diffend): the file header states
    the forward is FlashAttention-2 that never materialises the [.,L,L] score matrix; its
    forward shader defines the score as scale * q.k, the key-to-head map kv_head = head / reps,
    and the saved statistic m + log(l); its manualSdpa helper is a materialised
    matmul -> mask -> softmax -> matmul reference with GQA by grouping.
  * "mlx-mfa 2.5.2" (pypi.org), Features and Usage: sliding window as a (left, right) tuple
    with -1 meaning unbounded, native GQA without repeating K/V, tanh softcap (softcap=50.0),
    paged KV with a block_table, two-phase split-KV decode for N_q <= 4.
  * "mxflashattn 1.4.0 -> 1.5.0" (diffend), README: paged decode reads a paged KV cache with
    page size 16 and GQA 4; public entry points include a varlen forward.
  * "mlx-mfa 2.5.2" Features: variable-length packed sequences with cu_seqlens; "mlx-mfa
    2.61.0" (essential correctness update): varlen causal with N_q < N_k changed toward the
    bottom-right alignment used here per sequence.
  * "mlx-bun 0.4.0 -> 1.0.0, src/model/flash-attention.ts", Backward: three passes that
    recompute the scores — D_i = rowsum(dO_i * O_i); per key row p = exp(s - L_i),
    dp = dO_i . v_j, ds = p (dp - D_i), dV_j += p dO_i, dK_j += ds q_i scale; per query row
    dq_i += ds k_j scale.
  * "mlx-mfa 2.5.2" Features and Usage: block-sparse attention, flash_attention_sparse(q, k, v,
    block_mask, causal=...), a block mask whose zero blocks are never attended; here a block is
    `block` query rows x `block` keys and the mask further restricts the causal / window set.

Readings where the pages are silent or ambiguous (the kernels and tests follow the same ones):
  * window: key j is visible from absolute query position a iff a - win_l <= j <= a + win_r
    (inclusive; -1 = unbounded on that side), ANDed with causality when both are given;
  * causal with Nq != Nk is bottom-right aligned: query i sits at absolute position
    a = i + (Nk - Nq);
  * softcap: s <- cap * tanh(s / cap) applied to the scaled score before masking/softmax,
    disabled when cap <= 0; the LSE uses the capped scores;
  * LSE is the natural log-sum-exp of the final visible scores;
  * a row with no visible key has output 0 and LSE = -inf;
  * GQA groups are contiguous: query head h uses kv head h // (Hq // Hkv).
"""
from __future__ import annotations

import numpy as np

__all__ = ["visible", "attention", "attention_rows", "attention_varlen", "attention_varlen_rows",
           "attention_blocksparse", "attention_blocksparse_rows", "attention_backward",
           "paged_gather", "attention_paged_prefill", "decode", "decode_rows"]


def visible(Nq: int, Nk: int, causal: bool, win_l: int = -1, win_r: int = -1) -> np.ndarray:
    """Boolean [Nq, Nk]: may query row i attend to key j.

    Causal masking (mlx-bun forward shader masks keys after the query; mlx-mfa 2.5.2 Features,
    "Causal tile-skip") is aligned bottom-right; the window tuple follows mlx-mfa 2.5.2 Usage,
    window_size=(left, right) with -1 unbounded.
    """
    i = np.arange(Nq, dtype=np.int64)[:, None]
    j = np.arange(Nk, dtype=np.int64)[None, :]
    a = i + (Nk - Nq)
    vis = np.ones((Nq, Nk), dtype=bool)
    if causal:
        vis &= j <= a
    if win_l >= 0:
        vis &= j >= a - win_l
    if win_r >= 0:
        vis &= j <= a + win_r
    return vis


def _rows_for_head(qh, kh, vh, vis_rows, scale, softcap):
    """Attention for a block of query rows of one head.

    qh [r, D], kh/vh [Nk, D] fp64; vis_rows [r, Nk] bool. Returns (o [r, D], lse [r]).
    """
    s = (qh @ kh.T) * float(scale)                      # scaled scores (mlx-bun forward shader)
    if softcap > 0.0:                                   # mlx-mfa 2.5.2 Features: tanh softcap
        s = float(softcap) * np.tanh(s / float(softcap))
    s = np.where(vis_rows, s, -np.inf)
    has = vis_rows.any(axis=1)
    m = np.where(has, s.max(axis=1, initial=-np.inf), 0.0)
    w = np.exp(s - m[:, None])                          # exp(-inf) = 0 for masked keys
    l = w.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.where(has[:, None], (w @ vh) / np.where(has, l, 1.0)[:, None], 0.0)
        lse = np.where(has, m + np.log(np.where(has, l, 1.0)), -np.inf)
    return o, lse


def attention(q, k, v, scale, causal=False, win_l=-1, win_r=-1, softcap=0.0, row_block=512):
    """Full forward. q [B,Hq,Nq,D], k/v [B,Hkv,Nk,D] (fp64). Returns (o [B,Hq,Nq,D], lse [B,Hq,Nq])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    assert Hq % Hkv == 0, "Hkv must divide Hq"
    G = Hq // Hkv
    vis = visible(Nq, Nk, causal, win_l, win_r)
    o = np.zeros((B, Hq, Nq, D))
    lse = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // G                                   # mlx-bun forward shader: kv_head = head / reps
            for r0 in range(0, Nq, row_block):
                r1 = min(Nq, r0 + row_block)
                o[b, h, r0:r1], lse[b, h, r0:r1] = _rows_for_head(
                    q[b, h, r0:r1], k[b, g], v[b, g], vis[r0:r1], scale, softcap)
    return o, lse


def attention_rows(q, k, v, rows, scale, causal=False, win_l=-1, win_r=-1, softcap=0.0):
    """Selected rows only. rows: int array [n, 3] of (b, h, i). Returns (o [n, D], lse [n])."""
    q = np.asarray(q)
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    G = Hq // Hkv
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o = np.zeros((len(rows), D))
    lse = np.full(len(rows), -np.inf)
    j = np.arange(Nk, dtype=np.int64)
    for n, (b, h, i) in enumerate(rows):
        g = h // G
        a = i + (Nk - Nq)
        vis = np.ones(Nk, dtype=bool)
        if causal:
            vis &= j <= a
        if win_l >= 0:
            vis &= j >= a - win_l
        if win_r >= 0:
            vis &= j <= a + win_r
        qi = np.asarray(q[b, h, i:i + 1], dtype=np.float64)
        oi, li = _rows_for_head(qi, np.asarray(k[b, g], dtype=np.float64),
                                np.asarray(v[b, g], dtype=np.float64), vis[None, :], scale, softcap)
        o[n], lse[n] = oi[0], li[0]
    return o, lse


def _sequence_views(q, k, v, cu_q, cu_k, b):
    """Sequence b of a packed batch as [1, H, N, D] arrays (q [total_q, Hq, D] -> [1, Hq, Nq_b, D])."""
    q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
    k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
    qs = np.asarray(q[q0:q1], dtype=np.float64).transpose(1, 0, 2)[None]
    ks = np.asarray(k[k0:k1], dtype=np.float64).transpose(1, 0, 2)[None]
    vs = np.asarray(v[k0:k1], dtype=np.float64).transpose(1, 0, 2)[None]
    return qs, ks, vs


def attention_varlen(q, k, v, cu_q, cu_k, scale, causal=False, win_l=-1, win_r=-1, softcap=0.0):
    """Packed variable-length forward: sequence b (rows cu_q[b]..cu_q[b+1] of q, cu_k[b]..cu_k[b+1]
    of k / v) is attended on its own with the dense definition, bottom-right aligned per
    sequence. q [total_q, Hq, D], k/v [total_k, Hkv, D]. Returns (o [total_q, Hq, D],
    lse [Hq, total_q])."""
    total_q, Hq, D = np.shape(q)
    o = np.zeros((total_q, Hq, D))
    lse = np.full((Hq, total_q), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        if q1 == q0:
            continue
        qs, ks, vs = _sequence_views(q, k, v, cu_q, cu_k, b)
        ob, lb = attention(qs, ks, vs, scale, causal, win_l, win_r, softcap)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[:, q0:q1] = lb[0]
    return o, lse


def attention_varlen_rows(q, k, v, cu_q, cu_k, rows, scale, causal=False, win_l=-1, win_r=-1,
                          softcap=0.0):
    """Selected rows of the packed forward. rows: int array [n, 2] of (h, packed row r).
    Returns (o [n, D], lse [n])."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
    D = np.shape(q)[2]
    o = np.zeros((len(rows), D))
    lse = np.full(len(rows), -np.inf)
    cu_q = np.asarray(cu_q, dtype=np.int64)
    for n, (h, r) in enumerate(rows):
        b = int(np.searchsorted(cu_q, r, side="right") - 1)   # sequence holding packed row r
        qs, ks, vs = _sequence_views(q, k, v, cu_q, cu_k, b)
        oi, li = attention_rows(qs, ks, vs, [(0, h, r - cu_q[b])], scale, causal, win_l, win_r,
                                softcap)
        o[n], lse[n] = oi[0], li[0]
    return o, lse


def _block_visibility(block_mask, b, h, Nq, Nk, block):
    """[Nq, Nk] boolean: query row i may attend key j as far as the block mask is concerned."""
    m = np.asarray(block_mask[b, h], dtype=bool)
    return np.repeat(np.repeat(m, block, axis=0), block, axis=1)[:Nq, :Nk]


def attention_blocksparse(q, k, v, block_mask, scale, causal=False, win_l=-1, win_r=-1,
                          softcap=0.0, block=128, row_block=512):
    """Block-sparse forward: the dense definition with visibility vis(i, j) AND
    block_mask[b, h, i // block, j // block] != 0. q [B,Hq,Nq,D], k/v [B,Hkv,Nk,D],
    block_mask [B, Hq, ceil(Nq/block), ceil(Nk/block)]. Returns (o [B,Hq,Nq,D], lse [B,Hq,Nq]).
    Rows are independent; they are taken row_block at a time (as in attention) so that the
    score block stays row_block x Nk."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    G = Hq // Hkv
    vis = visible(Nq, Nk, causal, win_l, win_r)
    o = np.zeros((B, Hq, Nq, D))
    lse = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            vb = vis & _block_visibility(block_mask, b, h, Nq, Nk, block)
            for r0 in range(0, Nq, row_block):
                r1 = min(Nq, r0 + row_block)
                o[b, h, r0:r1], lse[b, h, r0:r1] = _rows_for_head(
                    q[b, h, r0:r1], k[b, h // G], v[b, h // G], vb[r0:r1], scale, softcap)
    return o, lse


def attention_blocksparse_rows(q, k, v, block_mask, rows, scale, causal=False, win_l=-1,
                               win_r=-1, softcap=0.0, block=128):
    """Selected rows (b, h, i) of the block-sparse forward. Returns (o [n, D], lse [n])."""
    B, Hq, Nq, D = np.shape(q)
    _, Hkv, Nk, _ = np.shape(k)
    G = Hq // Hkv
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o = np.zeros((len(rows), D))
    lse = np.full(len(rows), -np.inf)
    j = np.arange(Nk, dtype=np.int64)
    for n, (b, h, i) in enumerate(rows):
        a = i + Nk - Nq
        vis = np.ones(Nk, dtype=bool)
        if causal:
            vis &= j <= a
        if win_l >= 0:
            vis &= j >= a - win_l
        if win_r >= 0:
            vis &= j <= a + win_r
        keep = np.repeat(np.asarray(block_mask[b, h, i // block], dtype=bool), block)[:Nk]
        qi = np.asarray(q[b, h, i:i + 1], dtype=np.float64)
        oi, li = _rows_for_head(qi, np.asarray(k[b, h // G], dtype=np.float64),
                                np.asarray(v[b, h // G], dtype=np.float64),
                                (vis & keep)[None, :], scale, softcap)
        o[n], lse[n] = oi[0], li[0]
    return o, lse


def attention_backward(q, k, v, do, scale, causal=False, win_l=-1, win_r=-1, softcap=0.0):
    """Gradients of sum(O * dO) with O the forward above: returns (dq, dk, dv) in fp64 with the
    shapes of q, k, v. Written from the definition: for each (b, h) the probabilities P are
    materialised, dV = P^T dO, dP = dO V^T, D = rowsum(dO * O), dC = P * (dP - D), and with a cap
    dS = dC * (1 - tanh^2(s / cap)) (the derivative of cap * tanh(s / cap)), dQ = scale dS K,
    dK = scale dS^T Q (summed over the query heads of a kv group)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, Hq, Nq, D = q.shape
    _, Hkv, Nk, _ = k.shape
    G = Hq // Hkv
    vis = visible(Nq, Nk, causal, win_l, win_r)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s = scale * (q[b, h] @ k[b, g].T)
            if softcap > 0:
                t = np.tanh(s / softcap)
                c = softcap * t
            else:
                c = s
            c = np.where(vis, c, -np.inf)
            m = np.max(c, axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            w = np.where(vis, np.exp(c - m), 0.0)
            l = w.sum(axis=1, keepdims=True)
            p = np.divide(w, l, out=np.zeros_like(w), where=l > 0)
            o = p @ v[b, g]
            dp = do[b, h] @ v[b, g].T
            dvec = np.sum(do[b, h] * o, axis=1, keepdims=True)
            dc = p * (dp - dvec)
            ds = dc * (1.0 - t * t) if softcap > 0 else dc
            dq[b, h] = scale * (ds @ k[b, g])
            dk[b, g] += scale * (ds.T @ q[b, h])
            dv[b, g] += p.T @ do[b, h]
    return dq, dk, dv


def paged_gather(k_pages, v_pages, block_table, seq_len: int, b: int, page_size: int = 16):
    """Logical K/V of sequence b: token t lives in page block_table[b][t // page_size], slot
    t % page_size (mlx-mfa 2.5.2 Features, "Paged KV ... with block_table"; page size 16 as in
    the mxflashattn 1.5.0 README). Pages are [num_pages, page_size, Hkv, D]. Returns [Hkv, len, D]."""
    t = np.arange(int(seq_len), dtype=np.int64)
    pages = np.asarray(block_table[b], dtype=np.int64)[t // page_size]
    slots = t % page_size
    kb = np.asarray(k_pages[pages, slots], dtype=np.float64)   # [len, Hkv, D]
    vb = np.asarray(v_pages[pages, slots], dtype=np.float64)
    return kb.transpose(1, 0, 2), vb.transpose(1, 0, 2)


def decode(q, k_pages, v_pages, block_table, seq_lens, scale, causal=True, softcap=0.0,
           page_size: int = 16, win_l: int = -1):
    """Decode over a paged cache: each sequence is gathered, then the dense definition applies
    with Nk = len_b (query t of Nq sits at position len_b - Nq + t). Split-KV is a schedule of the
    same sum (mlx-mfa 2.5.2 Features, "Flash Decode -- two-phase split-KV"), so the oracle does
    not split. win_l >= 0 adds a left window (key j visible from a iff j >= a - win_l).
    q [B,Hq,Nq,D]. Returns (o [B,Hq,Nq,D], lse [B,Hq,Nq])."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, Nq, D = q.shape
    o = np.zeros((B, Hq, Nq, D))
    lse = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        kb, vb = paged_gather(k_pages, v_pages, block_table, L, b, page_size)
        ob, lb = attention(q[b:b + 1], kb[None], vb[None], scale, causal=causal, win_l=win_l,
                           softcap=softcap)
        o[b], lse[b] = ob[0], lb[0]
    return o, lse


def attention_paged_prefill(q, k_pages, v_pages, block_table, seq_lens, cu_q, scale, causal=True,
                            win_l=-1, win_r=-1, softcap=0.0, page_size: int = 16):
    """Chunked prefill over a paged cache: sequence b has cu_q[b+1] - cu_q[b] packed query rows
    (rows of q [total_q, Hq, D]) and seq_lens[b] keys gathered through its block_table row; the
    dense definition applies per sequence, the queries being the last Nq_b positions
    (bottom-right). Returns (o [total_q, Hq, D], lse [Hq, total_q])."""
    total_q, Hq, D = np.shape(q)
    o = np.zeros((total_q, Hq, D))
    lse = np.full((Hq, total_q), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        L = int(seq_lens[b])
        if q1 == q0 or L == 0:
            continue
        kb, vb = paged_gather(k_pages, v_pages, block_table, L, b, page_size)
        qs = np.asarray(q[q0:q1], dtype=np.float64).transpose(1, 0, 2)[None]
        ob, lb = attention(qs, kb[None], vb[None], scale, causal, win_l, win_r, softcap)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[:, q0:q1] = lb[0]
    return o, lse


def decode_rows(q, k_pages, v_pages, block_table, seq_lens, rows, scale, causal=True,
                softcap=0.0, page_size: int = 16, to_f64=None, win_l: int = -1):
    """Decode outputs for selected rows only, gathering just the kv head each row needs
    (win_l >= 0: the left window of decode()).

    rows: int array [n, 3] of (b, h, t). to_f64 converts a gathered slice of the pools to fp64
    (default: numpy conversion). Returns (o [n, D], lse [n])."""
    conv = to_f64 if to_f64 is not None else (lambda a: np.asarray(a, dtype=np.float64))
    B, Hq, Nq, D = np.asarray(q).shape
    Hkv = k_pages.shape[2]
    G = Hq // Hkv
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o = np.zeros((len(rows), D))
    lse = np.full(len(rows), -np.inf)
    for n, (b, h, t) in enumerate(rows):
        L = int(seq_lens[b])
        if L == 0:
            continue
        g = h // G
        tok = np.arange(L, dtype=np.int64)
        pages = np.asarray(block_table[b], dtype=np.int64)[tok // page_size]
        slots = tok % page_size
        kb = conv(k_pages[pages, slots, g])           # [L, D]
        vb = conv(v_pages[pages, slots, g])
        a = L - Nq + t                               # position of query token t
        vis = np.ones(L, dtype=bool)
        if causal:
            vis &= tok <= a
        if win_l >= 0:
            vis &= tok >= a - win_l
        qi = conv(np.asarray(q)[b, h, t:t + 1])
        oi, li = _rows_for_head(qi, kb, vb, vis[None, :], scale, softcap)
        o[n], lse[n] = oi[0], li[0]
    return o, lse
