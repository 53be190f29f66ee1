"""Fits the odd polynomial behind the small-argument softcap path and prints its coefficients.

The softcap s -> cap * tanh(s / cap) needs tanh(y) for every score. When every |y| of a warp's
row block is at most Y0 the kernel uses tanh(y) ~ y * q(y^2) with q a degree-4 polynomial in
u = y^2 (q(0) = 1, the Taylor leading term), evaluated with fused multiply-adds; otherwise it
uses tanh(|y|) = 1 - 2 / (exp(2|y|) + 1). The polynomial is a near-minimax fit of the RELATIVE
error on [0, Y0] by Lawson's iteratively reweighted least squares on a dense grid; coefficients
are rounded to fp32 and the error is re-measured with fp32 Horner evaluation.

Run: python tiled_exact_attention_mfa_b200/csrc/fit_tanh_poly.py
"""
import numpy as np

Y0 = 0.625
DEGREE = 4


def fit(y0=Y0, degree=DEGREE, iters=60, n=20001):
    y = np.linspace(1e-6, y0, n)
    u = y * y
    target = np.tanh(y) / y                      # q(u) target
    # q(u) = 1 + sum_{k>=1} c_k u^k ; minimise max |q(u)/target - 1|
    A = np.stack([u ** k for k in range(1, degree + 1)], axis=1) / target[:, None]
    b = (target - 1.0) / target
    w = np.ones(n) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return np.concatenate([[1.0], c])


def tanh_poly_f32(coef, y):
    y = y.astype(np.float32)
    u = (y * y).astype(np.float32)
    acc = np.float32(coef[-1])
    for ck in coef[-2::-1]:
        acc = (acc * u + np.float32(ck)).astype(np.float32)
    return (acc * y).astype(np.float32)


def main():
    c32 = fit().astype(np.float32)
    y = np.linspace(-Y0, Y0, 400001)
    got = tanh_poly_f32(c32, y).astype(np.float64)
    ref = np.tanh(y.astype(np.float32).astype(np.float64))
    nz = np.abs(ref) > 0
    rel = np.abs(got[nz] / ref[nz] - 1.0).max()
    print(f"|y| <= {Y0}, degree {DEGREE} in y^2: max relative error (fp32) = {rel:.3e}, "
          f"max abs error = {np.abs(got - ref).max():.3e}")
    for k, ck in enumerate(c32):
        print(f"  q{k} = {float(ck):.9e}f")
    return c32, rel


if __name__ == "__main__":
    main()
