"""Fit the degree-5 polynomial for 2^f, f in [-1/2, 1/2], that exp2_fma2 in
tc_common.cuh evaluates on the FMA pipe.

Method: least squares on the relative error at Chebyshev nodes, reweighted
(Lawson's iteration) toward the minimax solution; the coefficients are then
rounded to fp32 and the relative error of fp32 Horner evaluation is reported.
Run with `python fit_exp2_poly.py`; tests/test_numerics.py checks the
constants in tc_common.cuh against the error bound this prints.
"""

import numpy as np


def fit(deg=5, lo=-0.5, hi=0.5, n=20001, iters=30):
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (np.arange(n) + 0.5) / n)
    y = np.exp2(x)
    V = np.vander(x, deg + 1, increasing=True)
    w = np.ones(n)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * (w / y)[:, None], w, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * (err / err.max()) ** 0.3 + 1e-12
        w /= w.max()
    return c.astype(np.float32)


def horner_fp32(c, f):
    acc = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):  # fma: exact product, one rounding of the sum
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(c[k])).astype(np.float32)
    return acc


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    rel = np.abs(horner_fp32(c, f).astype(np.float64) - np.exp2(f.astype(np.float64)))
    rel /= np.exp2(f.astype(np.float64))
    print("coefficients c0..c5:", [float(v) for v in c])
    print(f"max relative error of fp32 Horner evaluation: {rel.max():.3e}")
