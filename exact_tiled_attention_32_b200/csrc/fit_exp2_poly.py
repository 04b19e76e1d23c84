"""Derives the polynomial the kernel uses for part of its exp2 evaluations.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-0.5, 0.5]
(Cody-Waite style range reduction; for base 2 it is exact).  2^f is then a
degree-3 polynomial whose coefficients minimise the maximum relative error
on [-0.5, 0.5], found here by a Remez exchange in fp64 and rounded to fp32.

    python fit_exp2_poly.py
    degree 3: c0..c3 = 0.99992806 0.69326097 0.24261113 0.05517167, max rel err 7.5e-05

The error is far below the bf16 rounding (2^-9) that P undergoes before the
P V product, and it enters the row sum l only as a relative error <= 7.5e-5.
"""
import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    g = np.linspace(a, b, 200001)
    err = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2 ** x[i]
        c = np.linalg.solve(A, 2 ** x)[:deg + 1]
        err = (np.polyval(c[::-1], g) - 2 ** g) / 2 ** g
        zc = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = [0] + list(zc + 1) + [len(g)]
        ext = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n:
            break
        x = g[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez(3)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 1000001)
    e32 = float(np.max(np.abs(np.polyval(c32.astype(np.float64)[::-1], g) / 2 ** g - 1)))
    print("degree 3: c0..c3 =", " ".join(f"{v:.8f}" for v in c32), f"max rel err {e32:.1e}")
    print("fp32 hex:", " ".join(f"0x{np.float32(v).view(np.uint32):08x}" for v in c32))
