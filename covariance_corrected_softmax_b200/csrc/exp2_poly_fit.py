"""Coefficients of the degree-4 polynomial for 2^f, f in [-1/2, 1/2], used by
exp2_poly2() in plx_device.cuh (Cody-Waite style range reduction there:
2^x = 2^n * 2^f with n = round(x)).

The fit minimises the maximum relative error by iteratively reweighted least
squares on Chebyshev-spaced points (a discrete stand-in for the Remez exchange).
Run: python exp2_poly_fit.py  -> prints the fp32 coefficients and the fp32
Horner-evaluated maximum relative error on a fine grid.
"""
import numpy as np


def fit(deg: int, iters: int = 60):
    f = np.cos(np.linspace(0.0, np.pi, 4000)) * 0.5
    y = np.exp2(f)
    w = np.ones_like(f)
    for _ in range(iters):
        a = np.vander(f, deg + 1, increasing=True) / y[:, None]
        c, *_ = np.linalg.lstsq(a * w[:, None], w, rcond=None)
        err = np.polyval(c[::-1], f) / y - 1.0
        w = w * (np.abs(err) / np.abs(err).max()) ** 0.1 + 1e-12
    return c.astype(np.float32)


def max_rel_err_fp32(c: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    r = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        r = (r * f + c[k]).astype(np.float32)
    return float(np.abs(r.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0).max())


if __name__ == "__main__":
    c = fit(4)
    for k, v in enumerate(c):
        print(f"c{k} = {float(v):.9e}f")
    print(f"max relative error (fp32 Horner): {max_rel_err_fp32(c):.3e}")
