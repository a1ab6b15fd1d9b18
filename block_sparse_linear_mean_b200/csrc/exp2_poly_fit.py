"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on
f in [-1/2, 1/2] used by the attention softmax for part of its exponentials.

Near-minimax in relative error: weighted least squares on Chebyshev nodes,
refined by Lawson's iteration (reweighting by the current error), in
float64.  Run: python exp2_poly_fit.py  (prints the coefficients and the
maximum relative error on a dense grid)."""

import numpy as np


def fit(degree=3, nodes=400, iters=200):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)          # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative error rows
    b = np.ones_like(f)
    w = np.full(nodes, 1.0 / nodes)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        e = np.abs(A @ c - b)
        w = w * e
        w /= w.sum()
    return c


if __name__ == "__main__":
    c = fit()
    g = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(np.polyval(c[::-1], g) / np.exp2(g) - 1)
    c32 = c.astype(np.float32)
    rel32 = np.abs(np.polyval(c32[::-1].astype(np.float64), g) / np.exp2(g) - 1)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r}  ({v.view(np.uint32):#010x})")
    print(f"max rel err {rel.max():.3e} (float32 coefficients {rel32.max():.3e})")
