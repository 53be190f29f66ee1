"""The seeded generator: deterministic, sliceable, N(0,1), correctly rounded, valid layouts."""
import numpy as np
import torch

import mfa_inputs as mi


def test_deterministic_and_sliceable():
    a = mi.normal_bits(11, 2, (1000,), mi.BF16)
    b = mi.normal_bits(11, 2, (1000,), mi.BF16)
    np.testing.assert_array_equal(a, b)
    c = mi.normal_bits(11, 2, (600,), mi.BF16, offset=400)
    np.testing.assert_array_equal(a[400:], c)
    d = mi.normal_bits(11, 3, (1000,), mi.BF16)
    assert np.mean(a == d) < 0.1


def test_normal_moments():
    z = mi.normal_f64(5, 0, 400_000)
    assert abs(z.mean()) < 0.01
    assert abs(z.var() - 1.0) < 0.01
    assert abs(np.mean(np.abs(z) < 1.0) - 0.6827) < 0.005


def test_rounding_fp16_and_bf16():
    z = mi.normal_f64(9, 1, 50_000) * 0.5
    h = mi.widen(mi.normal_bits(9, 1, (50_000,), mi.FP16, mul=0.5), mi.FP16)
    np.testing.assert_array_equal(h, z.astype(np.float16).astype(np.float64))
    bf = mi.widen(mi.normal_bits(9, 1, (50_000,), mi.BF16, mul=0.5), mi.BF16)
    ref = torch.from_numpy(z.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(bf, ref)


def test_permutation_and_uniform_ints():
    p = mi.permutation(4, 4, 1000)
    assert sorted(p.tolist()) == list(range(1000))
    assert not np.array_equal(p, np.arange(1000))
    u = mi.uniform_ints(4, 3, 20000, 8192, 131072)
    assert u.min() >= 8192 and u.max() <= 131072
    assert abs(u.mean() - (8192 + 131072) / 2) < 2000


def test_decode_layout_valid():
    case = mi.DecodeCase("t", B=3, Nq=1, Hq=4, Hkv=2, D=8, dtype=mi.BF16, len_lo=1, len_hi=100,
                         seed=3)
    q, k, v, table, lens = case.tensors()
    npg = [-(-int(L) // 16) for L in lens]
    ids = np.concatenate([table[b, :npg[b]] for b in range(3)])
    assert sorted(ids.tolist()) == list(range(k.shape[0]))
    for b in range(3):
        assert np.all(table[b, npg[b]:] == -1)
        kv = mi.widen(k, mi.BF16)
        L = int(lens[b])
        last = table[b, npg[b] - 1]
        assert np.all(np.isfinite(kv[last, : (L - 1) % 16 + 1]))
        assert np.all(np.isnan(kv[last, (L - 1) % 16 + 1:]))
