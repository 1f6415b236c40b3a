"""Coefficients of the FMA-pipe 2^f polynomial used by the tensor-core L-step
kernels (``ex2_fma2`` in tc_common.cuh).

2^x is evaluated as 2^n * p(f) with n = rint(x) and f = x - n in [-1/2, 1/2].
p is a degree-5 polynomial with p(0) = 1 whose maximum relative error against
2^f on [-1/2, 1/2] is made (nearly) equal-ripple by Lawson's iteratively
reweighted least squares (C. L. Lawson, "Contributions to the theory of linear
least maximum approximation", 1961), started from Chebyshev nodes.

Run ``python gen_exp2_poly.py`` to print the float32 coefficients and the
relative error of the float32 Horner evaluation; the kernel header holds the
printed values.
"""
import numpy as np

DEGREE = 5


def fit(n=DEGREE, iters=60, m=4000):
    f = 0.5 * np.cos(np.pi * (np.arange(m) + 0.5) / m)
    target = 2.0 ** f
    w = np.ones(m)
    for _ in range(iters):
        a = np.stack([f ** k for k in range(1, n + 1)], 1) / target[:, None]
        b = (target - 1.0) / target
        c, *_ = np.linalg.lstsq(a * w[:, None], b * w, rcond=None)
        p = 1.0 + sum(c[k - 1] * f ** k for k in range(1, n + 1))
        e = np.abs(p / target - 1.0)
        w = w * (1.0 + 50.0 * e / e.max())
    return np.concatenate([[1.0], c])


def horner_f32(coef, f):
    """float32 Horner with fused multiply-adds (product exact in float64)."""
    c = np.asarray(coef, np.float32)
    f = np.asarray(f, np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c[k])).astype(np.float32)
    return p


if __name__ == "__main__":
    coef = fit().astype(np.float32)
    ff = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    rel = np.abs(horner_f32(coef, ff).astype(np.float64) / 2.0 ** ff.astype(np.float64) - 1.0).max()
    for k, c in enumerate(coef):
        print(f"c{k} = {float(c):.9e}f")
    print(f"max relative error (float32 Horner) = {rel:.3e}")
