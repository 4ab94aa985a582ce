"""Coefficients of the polynomial p(f) ~ 2^f, |f| <= 1/2, that the prefill kernel
uses for the exponentials it computes on the FMA pipe (prefill.cu, exp2_poly2).

The fit minimises the maximum relative error |p(f) / 2^f - 1| on [-1/2, 1/2]:
an iteratively reweighted least-squares fit on Chebyshev points (each pass
raises the weight of the points where the error is largest, which drives the
error towards the equal-ripple minimax shape), then the coefficients are
rounded to float32 and the error is measured on a dense grid with the float32
coefficients, in Horner form.

    python exp2_poly_fit.py      # prints the coefficients and their errors
"""
from __future__ import annotations

import numpy as np


def fit(degree: int, passes: int = 60) -> tuple[np.ndarray, float]:
    """float32 coefficients c_0 .. c_degree of p(f) = sum c_k f^k and the
    largest relative error of p on [-1/2, 1/2] (Horner in float64 with the
    float32 coefficients)."""
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    y = np.exp2(f)
    w = np.ones_like(f)
    c = None
    for _ in range(passes):
        # rows scaled by 1 / 2^f: the residual is the relative error
        a = np.vander(f, degree + 1, increasing=True) / y[:, None]
        c, *_ = np.linalg.lstsq(a * np.sqrt(w)[:, None], np.sqrt(w), rcond=None)
        err = np.abs(np.polyval(c[::-1], f) / y - 1.0)
        w *= err / err.max() + 1e-3
        w /= w.mean()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001)
    p = np.zeros_like(grid)
    for ck in c32[::-1].astype(np.float64):
        p = p * grid + ck
    return c32, float(np.abs(p / np.exp2(grid) - 1.0).max())


if __name__ == "__main__":
    for d in (3, 4):
        c, e = fit(d)
        print(f"degree {d}: {{{', '.join(f'{float(x)!r}f' for x in c)}}}  "
              f"max relative error {e:.3e} = 2^{np.log2(e):.1f}")
