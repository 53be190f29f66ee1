"""The small-argument softcap polynomial (kTanhQ*, tanh_q / tanh_q2 in csrc/sm100.cuh) against
its error bound: coefficients equal to csrc/fit_tanh_poly.py's fit, and an fp32 emulation of
y * q(y^2) within 1.5e-7 absolute (3e-7 relative) of tanh on |y| <= 0.625."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_exact_attention_mfa_b200", "csrc")


def kernel_constants():
    text = open(os.path.join(CSRC, "sm100.cuh")).read()
    val = {k: float(v) for k, v in re.findall(r"constexpr float kTanh(Q\d|PolyMax) = (-?\d\.\d+(?:e[-+]\d+)?)f;", text)}
    return val


def test_coefficients_come_from_the_fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "fit_tanh_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c32 = fit.fit().astype(np.float32)
    k = kernel_constants()
    assert k["PolyMax"] == fit.Y0
    np.testing.assert_allclose(np.float32([k["Q1"], k["Q2"], k["Q3"], k["Q4"]]), c32[1:], rtol=2e-7, atol=0)


def test_error_bound():
    k = kernel_constants()
    f32 = np.float32
    y = np.linspace(-k["PolyMax"], k["PolyMax"], 1_000_001).astype(f32)
    u = (y * y).astype(f32)
    q = f32(k["Q4"])
    for c in (k["Q3"], k["Q2"], k["Q1"], 1.0):
        q = (q * u + f32(c)).astype(f32)
    t = (y * q).astype(f32).astype(np.float64)
    ref = np.tanh(y.astype(np.float64))
    assert np.max(np.abs(t - ref)) < 1.5e-7
    nz = ref != 0
    assert np.max(np.abs(t[nz] / ref[nz] - 1)) < 3e-7

