"""Fits the polynomial behind exp2_fma() in sm100.cuh and prints its coefficients.

exp2_fma(x) splits x = n + f with n = round(x) (Cody and Waite style range reduction: adding
1.5 * 2^23 rounds to an integer in the low mantissa bits) and f in [-1/2, 1/2], evaluates
p(f) ~ 2^f with a degree-4 polynomial in Horner form, and multiplies by 2^n built directly in the
exponent field. The polynomial is a near-minimax fit of the RELATIVE error on [-1/2, 1/2],
obtained here by Lawson's iteratively reweighted least squares (Lawson, 1961) on a dense grid,
with the constant term pinned to 1 so that p(0) = 1 exactly. Coefficients are rounded to fp32 and
the error is re-measured with fp32 Horner evaluation.

Run: python tiled_exact_attention_mfa_b200/csrc/fit_exp2_poly.py
"""
import numpy as np

DEGREE = 4


def fit(degree=DEGREE, iters=60, n=20001):
    f = np.linspace(-0.5, 0.5, n)
    target = np.exp2(f)
    # p(f) = 1 + sum_{k>=1} c_k f^k ; minimise max |p/2^f - 1|
    A = np.stack([f ** k for k in range(1, degree + 1)], axis=1) / target[:, None]
    b = (target - 1.0) / target
    w = np.ones(n) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return np.concatenate([[1.0], c])


def horner_f32(coef, f):
    f = f.astype(np.float32)
    acc = np.float32(coef[-1])
    for ck in coef[-2::-1]:
        acc = (acc * f + np.float32(ck)).astype(np.float32)
    return acc


def main():
    coef = fit()
    c32 = coef.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(horner_f32(c32, f).astype(np.float64) / np.exp2(f) - 1.0)
    print(f"degree {DEGREE}, max relative error (fp32 Horner) = {rel.max():.3e}")
    for k, ck in enumerate(c32):
        print(f"  c{k} = {float(ck):.9e}f  (0x{np.float32(ck).view(np.uint32):08x})")
    return c32, rel.max()


if __name__ == "__main__":
    main()
