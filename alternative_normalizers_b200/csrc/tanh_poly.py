"""Coefficients of the odd polynomial behind tanh_odd_poly2 (common.cuh).

    python alternative_normalizers_b200/csrc/tanh_poly.py

tanh(x) ~ x * (c0 + c1 x^2 + c2 x^4 + c3 x^6 + c4 x^8) on [-1, 1], fitted for
the smallest maximum absolute error by Lawson's algorithm (iteratively
reweighted least squares: the weight of each grid point grows with its
error until the error levels out).  Prints the coefficients rounded to
float32 and the maximum absolute error of the float32 Horner evaluation.
"""

import numpy as np

NCOEF = 5


def lawson_odd(nc, x, iters=400):
    A = np.stack([x ** (2 * k + 1) for k in range(nc)], axis=1)
    y = np.tanh(x)
    w = np.full(x.shape, 1.0 / x.size)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], y * sw, rcond=None)
        e = np.abs(A @ c - y)
        w = w * (e + 1e-300)
        w /= w.sum()
    return c


def horner_f32(c, x):
    x = x.astype(np.float32)
    t = (x * x).astype(np.float32)
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * t + np.float32(c[k])).astype(np.float32)
    return (x * p).astype(np.float32)


def coefficients():
    grid = np.unique(np.concatenate([np.linspace(0.0, 1.0, 20001),
                                     np.sin(np.linspace(0.0, np.pi / 2, 20001))]))
    return lawson_odd(NCOEF, grid).astype(np.float32)


if __name__ == "__main__":
    c = coefficients()
    g = np.linspace(-1.0, 1.0, 400001)
    err = np.abs(horner_f32(c, g).astype(np.float64) - np.tanh(g.astype(np.float32).astype(np.float64)))
    print("c0..c4 =", ", ".join(f"{v:.9g}f" for v in c.tolist()))
    print("max abs error (float32 Horner) on [-1, 1]:", err.max())
