"""Fit the polynomial used for exp2 on the FMA pipe (fb_attn_sm100.cu).

2^x = 2^n * 2^f with n = floor(x), f in [0, 1); 2^f is replaced by a cubic
c0 + c1 f + c2 f^2 + c3 f^3 whose maximum relative error on [0, 1) is
minimised (Lawson's iteratively reweighted least squares for the minimax
fit, C. L. Lawson 1961). The softmax rounds P to bf16 (8 significant bits),
so a relative error near 1e-4 is far below what the result keeps.

    python fit_exp2_poly.py      # prints the coefficients and the error
"""
import numpy as np


def fit(degree: int = 3, samples: int = 20001, iters: int = 400):
    f = np.linspace(0.0, 1.0, samples)
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative error rows
    w = np.ones_like(f) / samples
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], np.ones_like(f) * sw, rcond=None)
        err = np.abs(A @ c - 1.0)
        w = w * err
        w /= w.sum()
    rel = np.abs(np.polyval(c[::-1], f) / y - 1.0)
    return c, rel.max()


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v)!r}  ({v:.17g})")
    print(f"max relative error on [0, 1): {e:.3e}")
