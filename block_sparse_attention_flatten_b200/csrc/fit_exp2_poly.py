"""Fits the degree-3 polynomial of 2^f on [-1/2, 1/2] that exp2_poly_f2
(common.cuh) uses: the minimax fit of the RELATIVE error, by Lawson's
iteratively reweighted least squares on a dense grid, then checked with the
fp32 Horner evaluation the kernel performs.  Prints the coefficients (c0 ..
c3) and the maximum relative error."""
import numpy as np


def fit(degree: int = 3, iters: int = 200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    A = np.vstack([f ** k for k in range(degree + 1)]).T
    w = np.ones_like(f)
    for _ in range(iters):
        W = np.sqrt(w) / y
        c, *_ = np.linalg.lstsq(A * W[:, None], y * W, rcond=None)
        err = np.abs(A @ c - y) / y
        w = w * err
        w /= w.sum()
    return c


def horner_fp32_rel_err(c):
    f = np.linspace(-0.5, 0.5, 20001).astype(np.float32)
    c32 = np.asarray(c, dtype=np.float32)
    p = np.float32(c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)
    y = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - y) / y))


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3:", ", ".join(f"{x:.8f}" for x in c))
    print("max relative error (fp32 Horner):", horner_fp32_rel_err(c))
