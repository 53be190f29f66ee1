"""The FMA-pipe exp2 of the softmax (exp2_fma2 in csrc/sm100.cuh) against its error bound.

The kernel's coefficients must be the ones csrc/fit_exp2_poly.py produces, and an fp32
emulation of the kernel's steps (clamp at -127, range reduction by adding 1.5 * 2^23, Horner
polynomial with fused multiply-adds, 2^n built as (bits(t) << 23) + (127 - bits(1.5 * 2^23)) << 23) must stay within 4e-6 relative error of 2^x on the range the softmax
uses, and give exactly 0 at or below -127.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_exact_attention_mfa_b200", "csrc")


def kernel_coefficients():
    """(c4, c3, c2, c1) as written in sm100.cuh (constants kExp2C4 .. kExp2C1)."""
    text = open(os.path.join(CSRC, "sm100.cuh")).read()
    val = {k: float(v) for k, v in re.findall(r"constexpr float kExp2(C\d) = (-?\d\.\d+e[-+]\d+)f;", text)}
    return [val["C4"], val["C3"], val["C2"], val["C1"]]


def test_coefficients_come_from_the_fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c32 = fit.fit().astype(np.float32)            # c0 .. c4, c0 = 1
    got = kernel_coefficients()                   # c4, c3 (first fmaf), c2, c1
    want = [c32[4], c32[3], c32[2], c32[1]]
    np.testing.assert_allclose(np.float32(got), want, rtol=2e-7, atol=0)


def emulate(x):
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-127.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    f = (x - n).astype(f32)
    c4, c3, c2, c1 = (f32(v) for v in kernel_coefficients())
    p = (c4 * f + c3).astype(f32)
    p = (p * f + c2).astype(f32)
    p = (p * f + c1).astype(f32)
    p = (p * f + f32(1.0)).astype(f32)
    k = np.uint32(((127 - 0x4B400000) << 23) & 0xFFFFFFFF)
    e = ((t.view(np.uint32) << np.uint32(23)) + k).astype(np.uint32)
    return (p * e.view(np.float32)).astype(f32)


def test_relative_error_and_underflow():
    x = np.linspace(-126.0, 8.0, 2_000_001).astype(np.float32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 4e-6
    z = emulate(np.array([-127.0, -200.0, -np.inf], dtype=np.float32))
    assert np.all(z == 0.0)
    assert emulate(np.array([0.0], dtype=np.float32))[0] == 1.0
