"""Fit of the verification cost C_v(n; l) = a + b l + c n + e n^2 from latency samples.

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
summary), "Method: CaDDTree". The verification cost is profiled offline as a
convex function of the tree size that grows with it, and with the context
length. With the quadratic model in n and a linear term in l, that is a, b, c,
e >= 0: c, e >= 0 make it convex and non-decreasing in n, b >= 0
non-decreasing in l, and a >= 0 keeps it a cost. The fit is the non-negative
least-squares problem
  min || X beta - t ||^2  subject to beta >= 0,  X = [1, l, n, n^2],
solved by the Lawson-Hanson active-set method, written here for four unknowns.
Columns are scaled to unit norm before solving, and the result is scaled back.
"""
from __future__ import annotations

from typing import Sequence

import numpy as np

__all__ = ["fit_cost", "nnls"]


def nnls(A: np.ndarray, y: np.ndarray, max_iter: int = 200) -> np.ndarray:
    """Non-negative least squares, min ||A x - y|| with x >= 0 (Lawson-Hanson)."""
    A = np.asarray(A, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    m, k = A.shape
    x = np.zeros(k)
    passive = np.zeros(k, dtype=bool)
    w = A.T @ (y - A @ x)
    tol = 10.0 * np.finfo(np.float64).eps * np.linalg.norm(A, 1) * max(m, k)
    it = 0
    while (~passive).any() and (w[~passive] > tol).any() and it < max_iter:
        it += 1
        j = np.argmax(np.where(passive, -np.inf, w))
        passive[j] = True
        while True:
            z = np.zeros(k)
            z[passive] = np.linalg.lstsq(A[:, passive], y, rcond=None)[0]
            if (z[passive] > 0).all():
                x = z
                break
            # step back towards x until the first passive variable reaches zero
            neg = passive & (z <= 0)
            den = x[neg] - z[neg]
            ok = den > 0
            alpha = float(np.min(x[neg][ok] / den[ok])) if ok.any() else 0.0
            x = x + alpha * (z - x)
            passive &= x > tol
            x[~passive] = 0.0
        w = A.T @ (y - A @ x)
    return x


def fit_cost(n: Sequence[float], ell: Sequence[float], t: Sequence[float]) -> dict:
    """(a, b, c, e) >= 0 of C_v(n; l) = a + b l + c n + e n^2 fitted to samples (n_i, l_i, t_i).

    Returns the coefficients and the root-mean-square residual."""
    n = np.asarray(n, dtype=np.float64)
    ell = np.asarray(ell, dtype=np.float64)
    t = np.asarray(t, dtype=np.float64)
    X = np.stack([np.ones_like(n), ell, n, n * n], axis=1)
    scale = np.linalg.norm(X, axis=0)
    scale[scale == 0] = 1.0
    beta = nnls(X / scale, t) / scale
    resid = X @ beta - t
    return {"a": float(beta[0]), "b": float(beta[1]), "c": float(beta[2]), "e": float(beta[3]),
            "rms": float(np.sqrt(np.mean(resid * resid)))}
