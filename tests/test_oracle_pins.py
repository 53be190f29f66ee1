"""Pins for the fp64 oracle, independent of the oracle's own code.

Each check below uses something other than the oracle's arithmetic: torch's fp64 SDPA with a
mask built from torch's band routines, closed forms (Q = 0 gives LSE = ln(#visible keys)),
hand-computed two-key cases, and the invariants of exact attention (one visible key, identical
value rows, key permutation, GQA == MHA on repeated heads, cap -> infinity). A dropped scale,
a wrong mask index or sign, log2 instead of ln, or h % G instead of h // G fails at least one.
"""
import math

import numpy as np
import pytest
import torch

import oracle

rng = np.random.default_rng(7)


def band_mask_torch(Nq, Nk, causal, win_l, win_r):
    """Visibility built from torch.tril / torch.triu diagonals (bottom-right alignment:
    query i sits at i + Nk - Nq)."""
    off = Nk - Nq
    m = torch.ones(Nq, Nk, dtype=torch.bool)
    if causal:
        m &= torch.tril(torch.ones(Nq, Nk, dtype=torch.bool), diagonal=off)
    if win_r >= 0:
        m &= torch.tril(torch.ones(Nq, Nk, dtype=torch.bool), diagonal=off + win_r)
    if win_l >= 0:
        m &= torch.triu(torch.ones(Nq, Nk, dtype=torch.bool), diagonal=off - win_l)
    return m


def sdpa_ref(q, k, v, scale, mask):
    G = q.shape[1] // k.shape[1]
    kt = torch.from_numpy(k).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), kt, vt, attn_mask=mask, scale=scale).numpy()


CASES = [
    # B, Hq, Hkv, Nq, Nk, D, causal, win_l, win_r
    (2, 4, 2, 37, 53, 16, False, -1, -1),
    (2, 4, 2, 37, 53, 16, True, -1, -1),
    (1, 6, 3, 40, 40, 8, True, 5, -1),
    (1, 4, 4, 33, 33, 8, False, 3, 2),
    (1, 4, 1, 20, 64, 8, True, 11, 0),
    (1, 2, 2, 64, 29, 8, False, 7, 7),
]


@pytest.mark.parametrize("case", CASES)
def test_output_matches_torch_sdpa(case):
    B, Hq, Hkv, Nq, Nk, D, causal, wl, wr = case
    q = rng.standard_normal((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    scale = 0.37
    o, lse = oracle.attention(q, k, v, scale, causal, wl, wr)
    mask = band_mask_torch(Nq, Nk, causal, wl, wr)
    has = mask.any(dim=1).numpy()
    ref = sdpa_ref(q, k, v, scale, mask)
    np.testing.assert_allclose(o[:, :, has], ref[:, :, has], rtol=0, atol=1e-12)
    assert np.all(o[:, :, ~has] == 0.0)
    assert np.all(np.isneginf(lse[:, :, ~has]))
    assert np.all(np.isfinite(lse[:, :, has]))


def closed_form_count(Nq, Nk, causal, wl, wr):
    """Number of visible keys for each row, written as interval arithmetic."""
    out = []
    for i in range(Nq):
        a = i + Nk - Nq
        lo = 0 if wl < 0 else max(0, a - wl)
        hi = Nk - 1
        if causal:
            hi = min(hi, a)
        if wr >= 0:
            hi = min(hi, a + wr)
        out.append(max(0, hi - lo + 1))
    return np.array(out)


@pytest.mark.parametrize("case", CASES + [(1, 2, 2, 300, 300, 4, True, 128, 0)])
def test_zero_query_lse_is_log_count(case):
    """Q = 0: every visible score is 0, so LSE = ln(#visible) and O = mean of visible V rows."""
    B, Hq, Hkv, Nq, Nk, D, causal, wl, wr = case
    q = np.zeros((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    o, lse = oracle.attention(q, k, v, 0.5, causal, wl, wr, softcap=3.0)
    cnt = closed_form_count(Nq, Nk, causal, wl, wr)
    G = Hq // Hkv
    csum = np.concatenate([np.zeros((B, Hkv, 1, D)), np.cumsum(v, axis=2)], axis=2)
    for i in range(Nq):
        if cnt[i] == 0:
            assert np.all(np.isneginf(lse[:, :, i]))
            continue
        np.testing.assert_allclose(lse[:, :, i], math.log(cnt[i]), rtol=0, atol=1e-13)
        a = i + Nk - Nq
        lo = 0 if wl < 0 else max(0, a - wl)
        mean = (csum[:, :, lo + cnt[i]] - csum[:, :, lo]) / cnt[i]
        for h in range(Hq):
            np.testing.assert_allclose(o[:, h, i], mean[:, h // G], rtol=0, atol=1e-12)


def test_sliding_window_512_closed_form():
    """Causal + window (512, 0): LSE_i = ln(min(i + 1, 513)) when Q = 0."""
    N = 1100
    q = np.zeros((1, 1, N, 2))
    k = rng.standard_normal((1, 1, N, 2))
    v = rng.standard_normal((1, 1, N, 2))
    _, lse = oracle.attention(q, k, v, 0.1, True, 512, 0)
    want = np.log(np.minimum(np.arange(N) + 1, 513))
    np.testing.assert_allclose(lse[0, 0], want, rtol=0, atol=1e-13)


def test_one_visible_key_gives_its_value_row_and_score():
    """Window (0, 0), non-causal, Nq = Nk: row i sees key i only."""
    N, D = 9, 4
    q = rng.integers(-3, 4, (1, 2, N, D)).astype(float)
    k = rng.integers(-3, 4, (1, 2, N, D)).astype(float)
    v = rng.standard_normal((1, 2, N, D))
    for cap in (0.0, 2.5):
        o, lse = oracle.attention(q, k, v, 0.5, False, 0, 0, softcap=cap)
        np.testing.assert_array_equal(o, v)
        for h in range(2):
            for i in range(N):
                s = 0.5 * sum(q[0, h, i, d] * k[0, h, i, d] for d in range(D))
                if cap > 0:
                    s = cap * math.tanh(s / cap)
                assert lse[0, h, i] == pytest.approx(s, abs=1e-14)


def test_causal_row_zero_equals_first_value_row():
    q = rng.standard_normal((1, 3, 16, 8))
    k = rng.standard_normal((1, 3, 16, 8))
    v = rng.standard_normal((1, 3, 16, 8))
    o, lse = oracle.attention(q, k, v, 0.3, True)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=0, atol=1e-15)
    for h in range(3):
        assert lse[0, h, 0] == pytest.approx(0.3 * float(q[0, h, 0] @ k[0, h, 0]), abs=1e-13)


def test_identical_value_rows():
    v = np.tile(rng.standard_normal((1, 2, 1, 8)), (1, 1, 30, 1))
    q = rng.standard_normal((1, 4, 30, 8)) * 3
    k = rng.standard_normal((1, 2, 30, 8)) * 3
    o, _ = oracle.attention(q, k, v, 0.7, True, 6, -1, softcap=5.0)
    for h in range(4):
        np.testing.assert_allclose(o[0, h], np.broadcast_to(v[0, h // 2, 0], (30, 8)), rtol=0, atol=1e-12)


def test_two_key_hand_case():
    """q = (1, 0), k0 = (2, 0), k1 = (0, 1), scale 1: weights e^2/(e^2+1) and 1/(e^2+1)."""
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[2.0, 0.0], [0.0, 1.0]]]])
    v = np.array([[[[1.0, -1.0], [3.0, 5.0]]]])
    o, lse = oracle.attention(q, k, v, 1.0)
    w0 = math.exp(2) / (math.exp(2) + 1)
    w1 = 1 / (math.exp(2) + 1)
    assert o[0, 0, 0, 0] == pytest.approx(w0 * 1 + w1 * 3, abs=1e-15)
    assert o[0, 0, 0, 1] == pytest.approx(-w0 + 5 * w1, abs=1e-15)
    assert lse[0, 0, 0] == pytest.approx(math.log(math.exp(2) + 1), abs=1e-15)
    # with softcap 1: scores become tanh(2) and tanh(0) = 0
    o, lse = oracle.attention(q, k, v, 1.0, softcap=1.0)
    t = math.tanh(2.0)
    assert lse[0, 0, 0] == pytest.approx(math.log(math.exp(t) + 1), abs=1e-15)
    assert o[0, 0, 0, 0] == pytest.approx((math.exp(t) * 1 + 3) / (math.exp(t) + 1), abs=1e-15)


def test_key_permutation_invariance_unmasked():
    q = rng.standard_normal((1, 2, 11, 8))
    k = rng.standard_normal((1, 2, 23, 8))
    v = rng.standard_normal((1, 2, 23, 8))
    p = rng.permutation(23)
    o1, l1 = oracle.attention(q, k, v, 0.4)
    o2, l2 = oracle.attention(q, k[:, :, p], v[:, :, p], 0.4)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_gqa_equals_mha_on_repeated_heads():
    q = rng.standard_normal((2, 8, 19, 8))
    k = rng.standard_normal((2, 2, 19, 8))
    v = rng.standard_normal((2, 2, 19, 8))
    o1, l1 = oracle.attention(q, k, v, 0.3, True, 4, -1, softcap=2.0)
    o2, l2 = oracle.attention(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), 0.3, True, 4, -1,
                              softcap=2.0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_softcap_limits():
    q = rng.standard_normal((1, 2, 17, 8)) * 4
    k = rng.standard_normal((1, 2, 17, 8)) * 4
    v = rng.standard_normal((1, 2, 17, 8))
    o0, l0 = oracle.attention(q, k, v, 0.5, True)
    o1, l1 = oracle.attention(q, k, v, 0.5, True, softcap=1e9)  # s - cap*tanh(s/cap) ~ s^3/(3 cap^2)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-9)
    np.testing.assert_allclose(l1, l0, rtol=0, atol=1e-9)
    # with a tiny cap every score is squeezed into (-cap, cap): LSE <= cap + ln(#visible)
    _, l2 = oracle.attention(q, k, v, 0.5, True, softcap=0.25)
    n = np.arange(1, 18)
    assert np.all(l2[0] <= 0.25 + np.log(n)[None, :] + 1e-12)
    assert np.all(l2[0] >= -0.25 + np.log(n)[None, :] - 1e-12)


def test_window_special_cases():
    q = rng.standard_normal((1, 2, 25, 8))
    k = rng.standard_normal((1, 2, 25, 8))
    v = rng.standard_normal((1, 2, 25, 8))
    full = oracle.attention(q, k, v, 0.3, False)
    unb = oracle.attention(q, k, v, 0.3, False, -1, -1)
    np.testing.assert_array_equal(full[0], unb[0])
    causal = oracle.attention(q, k, v, 0.3, True)
    wide = oracle.attention(q, k, v, 0.3, False, 25, 0)
    np.testing.assert_array_equal(causal[0], wide[0])
    np.testing.assert_array_equal(causal[1], wide[1])


def test_empty_rows_when_queries_precede_all_keys():
    """Bottom-right causal with Nq > Nk: the first Nq - Nk rows see no key."""
    q = rng.standard_normal((1, 1, 6, 4))
    k = rng.standard_normal((1, 1, 4, 4))
    v = rng.standard_normal((1, 1, 4, 4))
    o, lse = oracle.attention(q, k, v, 1.0, True)
    assert np.all(o[0, 0, :2] == 0) and np.all(np.isneginf(lse[0, 0, :2]))
    np.testing.assert_allclose(o[0, 0, 2], v[0, 0, 0], atol=1e-15)


def test_rows_helper_matches_full():
    q = rng.standard_normal((2, 4, 30, 8))
    k = rng.standard_normal((2, 2, 41, 8))
    v = rng.standard_normal((2, 2, 41, 8))
    o, lse = oracle.attention(q, k, v, 0.2, True, 9, 3, softcap=4.0)
    rows = np.array([[0, 0, 0], [1, 3, 29], [0, 2, 17], [1, 1, 5]])
    o2, l2 = oracle.attention_rows(q, k, v, rows, 0.2, True, 9, 3, softcap=4.0)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(o2[n], o[b, h, i], rtol=0, atol=1e-14)
        assert l2[n] == pytest.approx(lse[b, h, i], abs=1e-14)


def _paged_from_contiguous(kc, vc, lens, page=16, perm_seed=3):
    """Scatter contiguous [B, Hkv, N, D] caches into a permuted page pool."""
    B, Hkv, N, D = kc.shape
    npg = [-(-L // page) for L in lens]
    total = sum(npg)
    perm = np.random.default_rng(perm_seed).permutation(total)
    kp = np.full((total, page, Hkv, D), np.nan)
    vp = np.full((total, page, Hkv, D), np.nan)
    table = np.full((B, max(npg) + 2), -1, dtype=np.int64)
    off = 0
    for b in range(B):
        for p in range(npg[b]):
            pid = perm[off + p]
            table[b, p] = pid
            for s in range(page):
                t = p * page + s
                if t < lens[b]:
                    kp[pid, s] = kc[b, :, t]
                    vp[pid, s] = vc[b, :, t]
        off += npg[b]
    return kp, vp, table


@pytest.mark.parametrize("Nq", [1, 3, 4])
def test_decode_gather_matches_sdpa_on_contiguous_cache(Nq):
    B, Hq, Hkv, D = 3, 8, 2, 8
    lens = [37, 16, 70]
    N = max(lens)
    kc = rng.standard_normal((B, Hkv, N, D))
    vc = rng.standard_normal((B, Hkv, N, D))
    q = rng.standard_normal((B, Hq, Nq, D))
    kp, vp, table = _paged_from_contiguous(kc, vc, lens)
    o, lse = oracle.decode(q, kp, vp, table, lens, 0.3, causal=True)
    for b in range(B):
        L = lens[b]
        mask = band_mask_torch(Nq, L, True, -1, -1)
        ref = sdpa_ref(q[b:b + 1], kc[b:b + 1, :, :L], vc[b:b + 1, :, :L], 0.3, mask)
        np.testing.assert_allclose(o[b], ref[0], rtol=0, atol=1e-12)
    assert np.all(np.isfinite(o))


@pytest.mark.parametrize("Nq", [1, 2, 4])
def test_decode_window_matches_sdpa_band(Nq):
    """A left window on the paged decode keeps, for query row t, the keys within win_l of its
    bottom-right position L - Nq + t: the gathered-cache SDPA under the band mask."""
    B, Hq, Hkv, D, win = 3, 4, 2, 8, 20
    lens = [37, 16, 70]
    kc = rng.standard_normal((B, Hkv, 70, D))
    vc = rng.standard_normal((B, Hkv, 70, D))
    q = rng.standard_normal((B, Hq, Nq, D))
    kp, vp, table = _paged_from_contiguous(kc, vc, lens)
    o, lse = oracle.decode(q, kp, vp, table, lens, 0.3, causal=True, win_l=win)
    for b in range(B):
        L = lens[b]
        mask = band_mask_torch(Nq, L, True, win, -1)
        ref = sdpa_ref(q[b:b + 1], kc[b:b + 1, :, :L], vc[b:b + 1, :, :L], 0.3, mask)
        np.testing.assert_allclose(o[b], ref[0], rtol=0, atol=1e-12)


def test_decode_window_equals_decode_of_the_cache_tail():
    """One query with a left window of w sees exactly the last w + 1 cached tokens, so it equals
    the unwindowed decode of a cache holding only those tokens; a window at least as long as the
    sequence changes nothing."""
    B, Hq, Hkv, D, w = 2, 4, 1, 8, 25
    lens = [90, 26]
    kc = rng.standard_normal((B, Hkv, 90, D))
    vc = rng.standard_normal((B, Hkv, 90, D))
    q = rng.standard_normal((B, Hq, 1, D))
    o, lse = oracle.decode(q, *_paged_from_contiguous(kc, vc, lens), lens, 0.3, win_l=w)
    for b in range(B):
        L = lens[b]
        kt = kc[b:b + 1, :, L - w - 1:L].copy()
        vt = vc[b:b + 1, :, L - w - 1:L].copy()
        o2, l2 = oracle.decode(q[b:b + 1], *_paged_from_contiguous(kt, vt, [w + 1]), [w + 1], 0.3)
        np.testing.assert_allclose(o[b], o2[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], l2[0], rtol=0, atol=1e-12)
    paged = _paged_from_contiguous(kc, vc, lens)
    a = oracle.decode(q, *paged, lens, 0.3, win_l=90)
    c = oracle.decode(q, *paged, lens, 0.3)
    np.testing.assert_allclose(a[0], c[0], rtol=0, atol=1e-14)


def test_decode_page_permutation_and_empty_sequence():
    B, Hq, Hkv, D = 2, 4, 2, 8
    lens = [50, 0]
    kc = rng.standard_normal((B, Hkv, 50, D))
    vc = rng.standard_normal((B, Hkv, 50, D))
    q = rng.standard_normal((B, Hq, 1, D))
    a = oracle.decode(q, *_paged_from_contiguous(kc, vc, [50, 1], perm_seed=1), [50, 0], 0.3)
    b = oracle.decode(q, *_paged_from_contiguous(kc, vc, [50, 1], perm_seed=2), [50, 0], 0.3)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    assert np.all(a[0][1] == 0) and np.all(np.isneginf(a[1][1]))


def test_decode_rows_helper_matches_pinned_decode():
    B, Hq, Hkv, D, Nq = 3, 8, 2, 8, 2
    lens = [37, 16, 70]
    kc = rng.standard_normal((B, Hkv, 70, D))
    vc = rng.standard_normal((B, Hkv, 70, D))
    q = rng.standard_normal((B, Hq, Nq, D))
    kp, vp, table = _paged_from_contiguous(kc, vc, lens)
    o, lse = oracle.decode(q, kp, vp, table, lens, 0.3, causal=True, softcap=4.0)
    rows = np.array([[0, 0, 0], [1, 7, 1], [2, 3, 0], [2, 4, 1]])
    o2, l2 = oracle.decode_rows(q, kp, vp, table, lens, rows, 0.3, True, 4.0)
    for n, (b, h, t) in enumerate(rows):
        np.testing.assert_allclose(o2[n], o[b, h, t], rtol=0, atol=1e-14)
        assert l2[n] == pytest.approx(lse[b, h, t], abs=1e-14)
    o, lse = oracle.decode(q, kp, vp, table, lens, 0.3, causal=False, win_l=9)
    o2, l2 = oracle.decode_rows(q, kp, vp, table, lens, rows, 0.3, False, win_l=9)
    for n, (b, h, t) in enumerate(rows):
        np.testing.assert_allclose(o2[n], o[b, h, t], rtol=0, atol=1e-14)
        assert l2[n] == pytest.approx(lse[b, h, t], abs=1e-14)


# ---------------------------------------------------------------- packed variable-length batches
VARLEN = [
    # Hq, Hkv, D, query lengths, key lengths, causal, win_l, win_r
    (4, 2, 8, [5, 0, 17, 9], [5, 3, 30, 9], True, -1, -1),
    (2, 2, 8, [12, 7, 1], [20, 7, 4], False, 3, 2),
    (6, 3, 4, [8, 8], [2, 0], True, 4, 0),
]


def _packed(lens, H, D):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return cu, rng.standard_normal((int(cu[-1]), H, D))


@pytest.mark.parametrize("case", VARLEN)
def test_varlen_matches_torch_sdpa_per_sequence(case):
    """Each sequence of the packed batch against torch's SDPA on that sequence alone, with the
    bottom-right band mask built from torch.tril / torch.triu at its own Nq, Nk."""
    Hq, Hkv, D, nq, nk, causal, wl, wr = case
    cq, q = _packed(nq, Hq, D)
    ck, k = _packed(nk, Hkv, D)
    v = rng.standard_normal(k.shape)
    o, lse = oracle.attention_varlen(q, k, v, cq, ck, 0.41, causal, wl, wr)
    assert o.shape == q.shape and lse.shape == (Hq, cq[-1])
    for b in range(len(nq)):
        if nq[b] == 0:
            continue
        qs = q[cq[b]:cq[b + 1]].transpose(1, 0, 2)[None]
        ks = k[ck[b]:ck[b + 1]].transpose(1, 0, 2)[None]
        vs = v[ck[b]:ck[b + 1]].transpose(1, 0, 2)[None]
        ob = o[cq[b]:cq[b + 1]].transpose(1, 0, 2)[None]
        lb = lse[:, cq[b]:cq[b + 1]][None]
        if nk[b] == 0:
            assert np.all(ob == 0) and np.all(np.isneginf(lb))
            continue
        mask = band_mask_torch(nq[b], nk[b], causal, wl, wr)
        has = mask.any(dim=1).numpy()
        ref = sdpa_ref(qs, ks, vs, 0.41, mask)
        np.testing.assert_allclose(ob[:, :, has], ref[:, :, has], rtol=0, atol=1e-12)
        assert np.all(ob[:, :, ~has] == 0) and np.all(np.isneginf(lb[:, :, ~has]))


def test_varlen_zero_query_lse_is_log_count_per_sequence():
    """Q = 0 in every sequence: LSE of packed row r of sequence b = ln(#keys visible at its own
    bottom-right offset) — pins the per-sequence offsets and lengths."""
    nq, nk = [7, 30, 1, 0, 12], [9, 30, 40, 5, 3]
    cq, _ = _packed(nq, 2, 4)
    ck, k = _packed(nk, 2, 4)
    q = np.zeros((int(cq[-1]), 2, 4))
    v = rng.standard_normal(k.shape)
    for causal, wl, wr in ((True, -1, -1), (True, 5, 0), (False, 2, 6)):
        _, lse = oracle.attention_varlen(q, k, v, cq, ck, 0.7, causal, wl, wr)
        for b in range(len(nq)):
            cnt = closed_form_count(nq[b], nk[b], causal, wl, wr)
            for i in range(nq[b]):
                got = lse[:, cq[b] + i]
                if cnt[i] == 0:
                    assert np.all(np.isneginf(got))
                else:
                    np.testing.assert_allclose(got, math.log(cnt[i]), rtol=0, atol=1e-13)


def test_varlen_sequences_do_not_see_each_other():
    """Changing one sequence's K / V leaves every other sequence's output bitwise unchanged."""
    nq, nk = [6, 9, 4], [6, 11, 4]
    cq, q = _packed(nq, 2, 8)
    ck, k = _packed(nk, 2, 8)
    v = rng.standard_normal(k.shape)
    o1, l1 = oracle.attention_varlen(q, k, v, cq, ck, 0.3, True)
    k2, v2 = k.copy(), v.copy()
    k2[ck[1]:ck[2]] += 5.0
    v2[ck[1]:ck[2]] *= -3.0
    o2, l2 = oracle.attention_varlen(q, k2, v2, cq, ck, 0.3, True)
    for b in (0, 2):
        assert np.array_equal(o1[cq[b]:cq[b + 1]], o2[cq[b]:cq[b + 1]])
        assert np.array_equal(l1[:, cq[b]:cq[b + 1]], l2[:, cq[b]:cq[b + 1]])
    assert not np.allclose(o1[cq[1]:cq[2]], o2[cq[1]:cq[2]])


def test_varlen_rows_helper_matches_full():
    nq, nk = [5, 13, 2], [8, 13, 20]
    cq, q = _packed(nq, 4, 8)
    ck, k = _packed(nk, 2, 8)
    v = rng.standard_normal(k.shape)
    o, lse = oracle.attention_varlen(q, k, v, cq, ck, 0.5, True, 6, -1, softcap=2.0)
    rows = np.array([(h, r) for h in range(4) for r in range(int(cq[-1]))])
    orow, lrow = oracle.attention_varlen_rows(q, k, v, cq, ck, rows, 0.5, True, 6, -1, softcap=2.0)
    np.testing.assert_allclose(orow, o[rows[:, 1], rows[:, 0]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lrow, lse[rows[:, 0], rows[:, 1]], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- block-sparse masks
def _torch_block_mask(bm, Nq, Nk, block):
    """[Nq, Nk] boolean from a block mask, expanded with torch.repeat_interleave."""
    t = torch.from_numpy(np.asarray(bm, dtype=bool))
    return t.repeat_interleave(block, 0).repeat_interleave(block, 1)[:Nq, :Nk]


@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1), (True, 9, 0), (False, 4, 6)])
def test_blocksparse_matches_torch_sdpa(causal, wl, wr):
    """Against torch's SDPA with the band mask AND the block mask (expanded by torch)."""
    B, Hq, Hkv, Nq, Nk, D, blk = 2, 4, 2, 37, 45, 8, 8
    q = rng.standard_normal((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    bm = (rng.random((B, Hq, -(-Nq // blk), -(-Nk // blk))) < 0.5).astype(np.uint8)
    o, lse = oracle.attention_blocksparse(q, k, v, bm, 0.3, causal, wl, wr, block=blk)
    band = band_mask_torch(Nq, Nk, causal, wl, wr)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            m = band & _torch_block_mask(bm[b, h], Nq, Nk, blk)
            has = m.any(dim=1).numpy()
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, h][None, None]), torch.from_numpy(k[b, h // G][None, None]),
                torch.from_numpy(v[b, h // G][None, None]), attn_mask=m, scale=0.3).numpy()[0, 0]
            np.testing.assert_allclose(o[b, h, has], ref[has], rtol=0, atol=1e-12)
            assert np.all(o[b, h, ~has] == 0) and np.all(np.isneginf(lse[b, h, ~has]))


def test_blocksparse_all_ones_is_dense_and_all_zeros_is_empty():
    B, Hq, Hkv, Nq, Nk, D, blk = 1, 2, 1, 40, 40, 8, 16
    q = rng.standard_normal((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    ones = np.ones((B, Hq, 3, 3), dtype=np.uint8)
    o1, l1 = oracle.attention_blocksparse(q, k, v, ones, 0.4, True, block=blk)
    o2, l2 = oracle.attention(q, k, v, 0.4, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    o3, l3 = oracle.attention_blocksparse(q, k, v, 0 * ones, 0.4, True, block=blk)
    assert np.all(o3 == 0) and np.all(np.isneginf(l3))


def test_blocksparse_zero_query_lse_counts_active_keys():
    """Q = 0: LSE of row i = ln(#keys that are band-visible AND in an active block), counted by
    interval arithmetic per active key block."""
    Nq, Nk, blk = 50, 70, 16
    bm = (rng.random((1, 1, 4, 5)) < 0.6).astype(np.uint8)
    bm[0, 0, :, 0] = 1
    q = np.zeros((1, 1, Nq, 4))
    k = rng.standard_normal((1, 1, Nk, 4))
    v = rng.standard_normal((1, 1, Nk, 4))
    for causal, wl, wr in ((True, -1, -1), (True, 20, 0), (False, 7, 3)):
        _, lse = oracle.attention_blocksparse(q, k, v, bm, 1.0, causal, wl, wr, block=blk)
        for i in range(Nq):
            a = i + Nk - Nq
            lo = 0 if wl < 0 else max(0, a - wl)
            hi = Nk - 1
            if causal:
                hi = min(hi, a)
            if wr >= 0:
                hi = min(hi, a + wr)
            cnt = 0
            for jb in range(5):
                if bm[0, 0, i // blk, jb]:
                    cnt += max(0, min(hi, jb * blk + blk - 1, Nk - 1) - max(lo, jb * blk) + 1)
            if cnt == 0:
                assert np.isneginf(lse[0, 0, i])
            else:
                assert abs(lse[0, 0, i] - math.log(cnt)) < 1e-13


def test_blocksparse_rows_helper_matches_full():
    B, Hq, Hkv, Nq, Nk, D, blk = 2, 4, 2, 30, 44, 8, 8
    q = rng.standard_normal((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    bm = (rng.random((B, Hq, 4, 6)) < 0.5).astype(np.uint8)
    o, lse = oracle.attention_blocksparse(q, k, v, bm, 0.5, True, 12, -1, softcap=3.0, block=blk)
    rows = np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in range(Nq)])
    orow, lrow = oracle.attention_blocksparse_rows(q, k, v, bm, rows, 0.5, True, 12, -1,
                                                   softcap=3.0, block=blk)
    np.testing.assert_allclose(orow, o[rows[:, 0], rows[:, 1], rows[:, 2]], rtol=0, atol=1e-13)
    np.testing.assert_array_equal(np.isneginf(lrow), np.isneginf(lse[rows[:, 0], rows[:, 1], rows[:, 2]]))


# ---------------------------------------------------------------- backward
def _torch_grads(q, k, v, do, scale, mask):
    G = q.shape[1] // k.shape[1]
    qt, kt, vt = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(G, dim=1), vt.repeat_interleave(G, dim=1), attn_mask=mask,
        scale=scale)
    (o * torch.from_numpy(do)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("case", [
    (1, 4, 2, 23, 31, 8, False, -1, -1),
    (2, 2, 2, 30, 30, 8, True, -1, -1),
    (1, 6, 3, 25, 40, 4, True, 7, 0),
    (1, 2, 1, 33, 33, 8, False, 5, 3),
])
def test_backward_matches_torch_autograd(case):
    """Against torch autograd through fp64 SDPA (rows with at least one visible key)."""
    B, Hq, Hkv, Nq, Nk, D, causal, wl, wr = case
    q = rng.standard_normal((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    do = rng.standard_normal((B, Hq, Nq, D))
    mask = band_mask_torch(Nq, Nk, causal, wl, wr)
    assert bool(mask.any(dim=1).all()), "every row needs a visible key for the torch reference"
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.35, causal, wl, wr)
    tq, tk, tv = _torch_grads(q, k, v, do, 0.35, mask)
    np.testing.assert_allclose(dq, tq, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, tk, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, tv, rtol=0, atol=1e-11)


def test_backward_softcap_matches_finite_differences():
    """With a cap (no library reference): central differences of sum(O * dO) through the forward
    oracle, on every coordinate of a small case."""
    B, Hq, Hkv, Nq, Nk, D = 1, 2, 1, 5, 7, 3
    q = rng.standard_normal((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    do = rng.standard_normal((B, Hq, Nq, D))
    cap, scale, eps = 1.7, 0.9, 1e-6
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, True, 3, -1, softcap=cap)

    def loss(q_, k_, v_):
        o, _ = oracle.attention(q_, k_, v_, scale, True, 3, -1, softcap=cap)
        return float(np.sum(o * do))

    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            x[idx] += eps
            up = loss(q, k, v)
            x[idx] -= 2 * eps
            dn = loss(q, k, v)
            x[idx] += eps
            num[idx] = (up - dn) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=0, atol=2e-8)


def test_backward_gqa_is_mha_on_repeated_heads_and_empty_rows_give_zero():
    B, Hq, Hkv, Nq, Nk, D = 1, 4, 2, 12, 9, 4
    q = rng.standard_normal((B, Hq, Nq, D))
    k = rng.standard_normal((B, Hkv, Nk, D))
    v = rng.standard_normal((B, Hkv, Nk, D))
    do = rng.standard_normal((B, Hq, Nq, D))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, True)
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    dq2, dk2, dv2 = oracle.attention_backward(q, kr, vr, do, 0.5, True)
    np.testing.assert_allclose(dq, dq2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, 2, Nk, D).sum(axis=2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, 2, Nk, D).sum(axis=2), rtol=0, atol=1e-13)
    # Nq > Nk causal: the first Nq - Nk rows see no key, so their dq is zero
    assert np.all(dq[:, :, :Nq - Nk] == 0)


# ---------------------------------------------------------------- paged (chunked) prefill
def test_paged_prefill_equals_varlen_on_contiguous_and_decode_for_short_chunks():
    """Pages in identity order hold exactly the contiguous K / V, so the paged prefill equals
    the packed varlen forward; with 1-4 queries per sequence it equals the decode oracle."""
    Hq, Hkv, D, page = 4, 2, 8, 16
    lens = np.array([37, 16, 70], dtype=np.int64)
    nq = np.array([5, 16, 3], dtype=np.int64)
    npg = -(-lens // page)
    kc = [rng.standard_normal((int(L), Hkv, D)) for L in lens]
    vc = [rng.standard_normal((int(L), Hkv, D)) for L in lens]
    num = int(npg.sum())
    kp = np.full((num, page, Hkv, D), np.nan)
    vp = np.full((num, page, Hkv, D), np.nan)
    table = np.full((3, int(npg.max())), -1, dtype=np.int64)
    perm = rng.permutation(num)
    off = 0
    for b in range(3):
        for t in range(int(lens[b])):
            pg = perm[off + t // page]
            kp[pg, t % page] = kc[b][t]
            vp[pg, t % page] = vc[b][t]
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    cu_q = np.concatenate([[0], np.cumsum(nq)])
    cu_k = np.concatenate([[0], np.cumsum(lens)])
    q = rng.standard_normal((int(cu_q[-1]), Hq, D))
    for causal, wl, wr in ((True, -1, -1), (True, 9, 0), (False, 4, 2)):
        o, lse = oracle.attention_paged_prefill(q, kp, vp, table, lens, cu_q, 0.3, causal, wl, wr)
        ov, lv = oracle.attention_varlen(q, np.concatenate(kc), np.concatenate(vc), cu_q, cu_k,
                                         0.3, causal, wl, wr)
        np.testing.assert_allclose(o, ov, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, lv, rtol=0, atol=1e-13)
    # short chunks: 3 queries of sequence 2 through the decode oracle
    qd = q[cu_q[2]:cu_q[3]].transpose(1, 0, 2)[None]
    od, ld = oracle.decode(qd, kp, vp, table[2:3], lens[2:3], 0.3, causal=True)
    o, lse = oracle.attention_paged_prefill(q, kp, vp, table, lens, cu_q, 0.3, True)
    np.testing.assert_allclose(o[cu_q[2]:cu_q[3]], od[0].transpose(1, 0, 2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, cu_q[2]:cu_q[3]], ld[0], rtol=0, atol=1e-13)
