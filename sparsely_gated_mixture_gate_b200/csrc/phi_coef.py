"""Coefficients of the routing kernels' standard normal CDF (phi.cuh).

For x >= 0, Phi(-x) = exp(-x^2/2) * Q(x) with Q(x) = erfcx(x / sqrt 2) / 2,
a smooth function falling like 1 / (x sqrt(2 pi)).  Q is approximated by a
degree-8 polynomial in t = 1 / (1 + 0.4 x) on [0, 13.5], fitted by least
squares on the relative error with iteratively raised weights where the error
is largest (a Lawson-style approach to the minimax fit).  Run to print the
coefficients (t^0 first) and the fp32 maximum relative error of Phi on
[-12.5, 8] against scipy.special.ndtr.
"""
import numpy as np
from scipy.special import erfcx, ndtr

P = 0.4      # t = 1 / (1 + P x)
DEG = 8
XMAX = 13.5  # beyond it Phi(-x) < 2^-126 (0 in the kernels)


def fit():
    x = np.linspace(0.0, XMAX, 40001)
    t = 1.0 / (1.0 + P * x)
    y = 0.5 * erfcx(x / np.sqrt(2.0))
    A = np.vander(t, DEG + 1, increasing=True)
    wt = np.ones_like(x)
    for _ in range(200):
        c, *_ = np.linalg.lstsq(A * (wt / y)[:, None], wt, rcond=None)
        err = np.abs(A @ c - y) / y
        wt = wt * (1.0 + 2.0 * err / err.max())
        wt /= wt.mean()
    return c.astype(np.float32)


def phi_fp32(z, c):
    """The kernels' evaluation order, each fp32 operation rounded once."""
    f32, f64 = np.float32, np.float64
    z = np.asarray(z, dtype=f32)
    x = np.abs(z)
    t = (f32(1) / (f32(P) * x + f32(1))).astype(f32)
    q = np.full_like(t, c[-1])
    for ck in c[-2::-1]:
        q = (q.astype(f64) * t + ck).astype(f32)                  # fmaf
    hi = (x * x).astype(f32)
    lo = (x.astype(f64) ** 2 - hi).astype(f32)                    # fmaf(x, x, -hi)
    e = np.exp(-0.5 * hi.astype(f64)).astype(f32)                 # expf
    e = (e.astype(f64) * (1.0 - 0.5 * lo.astype(f64))).astype(f32)  # e * fmaf(-0.5, lo, 1)
    v = np.where(x < f32(XMAX), (e * q).astype(f32), f32(0))
    return np.where(z > 0, (f32(1) - v).astype(f32), v)


if __name__ == "__main__":
    c = fit()
    print("coefficients (t^0 .. t^8):", ", ".join(f"{v:.9e}f" for v in c))
    z = np.linspace(-12.5, 8.0, 2000001).astype(np.float32)
    rel = np.abs(phi_fp32(z, c) - ndtr(z.astype(np.float64))) / ndtr(z.astype(np.float64))
    print(f"max relative error of Phi on [-12.5, 8]: {rel.max():.3e}")
