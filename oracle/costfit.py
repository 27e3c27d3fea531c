"""Cost-model fit oracle: the non-negative least-squares fit of C_v (test infrastructure only).

Source: "Cost-Aware Diffusion Draft Trees for Speculative Decoding"
(gist.science summary), "Method: CaDDTree": the verification cost is profiled
offline as a convex function of the tree size that does not decrease as it
grows, and it grows with the context length. With the configurations' model
C_v(n; l) = a + b l + c n + e n^2 that reads a, b, c, e >= 0, and the fit to
latency samples (n_i, l_i, t_i) is

    min_beta || X beta - t ||^2   subject to   beta >= 0,   X = [1, l, n, n^2].

The oracle takes that definition literally, for its four unknowns: every one
of the 16 subsets F of free coefficients gets the unconstrained least-squares
solution on the columns in F (zeros elsewhere); the candidates with every
coefficient >= 0 are feasible points, the problem's optimum is one of them (its
free set), so the feasible candidate with the smallest residual is the
optimum. Columns are scaled to unit norm for the solves (numpy lstsq) and the
coefficients scaled back. Pinned in tests to SciPy's NNLS, to the KKT
conditions and to exact recovery on noiseless samples.
"""
from __future__ import annotations

import itertools

import numpy as np

__all__ = ["cost_fit"]


def cost_fit(n, ell, t):
    """(a, b, c, e, rms) of the non-negative fit of t ~ a + b l + c n + e n^2 (float64)."""
    n = np.asarray(n, dtype=np.float64)
    ell = np.asarray(ell, dtype=np.float64)
    t = np.asarray(t, dtype=np.float64)
    X = np.stack([np.ones_like(n), ell, n, n * n], axis=1)
    scale = np.linalg.norm(X, axis=0)
    scale[scale == 0] = 1.0
    Xs = X / scale
    best, best_r = np.zeros(4), float(np.sum(t * t))   # the empty free set: beta = 0
    for size in range(1, 5):
        for F in itertools.combinations(range(4), size):
            cols = list(F)
            sol = np.linalg.lstsq(Xs[:, cols], t, rcond=None)[0]
            if (sol < 0).any():
                continue
            x = np.zeros(4)
            x[cols] = sol
            r = float(np.sum((Xs @ x - t) ** 2))
            if r < best_r:
                best, best_r = x, r
    beta = best / scale
    resid = X @ beta - t
    return (float(beta[0]), float(beta[1]), float(beta[2]), float(beta[3]),
            float(np.sqrt(np.mean(resid * resid))))
