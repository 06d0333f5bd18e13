"""Fit the polynomials for 2^f, f in [-1/2, 1/2], used by ex2_poly2 in
tc_ptx.cuh (degrees 3, 4 and 5; run: python gen_exp2_poly.py).

Iteratively reweighted least squares on 4000 Chebyshev nodes, minimising the
relative error; prints the float32 coefficients (constant term first) and the
maximum relative error of their float32 Horner evaluation.
"""
import numpy as np


def fit(deg=5, lo=-0.5, hi=0.5, nodes=4000, iters=30):
    k = np.arange(nodes)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * (k + 0.5) / nodes)
    y = np.exp2(x)
    A = np.vander(x, deg + 1, increasing=True)
    w = 1.0 / y
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(A * w[:, None], y * w, rcond=None)
        err = (A @ c - y) / y
        w = w * (1.0 + 50.0 * np.abs(err) / np.abs(err).max())
    return c.astype(np.float32)


def max_rel_err_f32(c):
    x = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.float32(c[-1])
    for cc in c[-2::-1]:
        p = (p * x + cc).astype(np.float32)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    for deg in (3, 4, 5):
        c = fit(deg)
        print(f"degree {deg} coefficients (c0..c{deg}):", [f"{v:.7e}" for v in c])
        print("  max relative error (float32 Horner):", max_rel_err_f32(c))
