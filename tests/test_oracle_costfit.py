"""Pins of the cost-model fit oracle (oracle.cost_fit).

CaDDTree summary (gist.science), "Method: CaDDTree": C_v is profiled offline as
a convex function of the tree size that does not decrease as it grows, i.e. the
non-negative least-squares fit of C_v(n; l) = a + b l + c n + e n^2. The oracle
enumerates the 16 free sets; here it is checked against SciPy's NNLS (a library
routine for the same problem), against the KKT conditions of the problem, and
against exact recovery of noiseless samples of a convex cost.
"""
import numpy as np
import pytest
from scipy.optimize import nnls as scipy_nnls

import oracle


def _design(n, ell):
    n = np.asarray(n, np.float64)
    ell = np.asarray(ell, np.float64)
    return np.stack([np.ones_like(n), ell, n, n * n], axis=1)


def _samples(seed, m=64):
    rng = np.random.default_rng(seed)
    n = rng.integers(1, 512, m).astype(np.float64)
    ell = rng.choice([512.0, 4096.0, 32768.0], m)
    coef = rng.uniform(0, 1, 4) * np.array([2.0, 1e-4, 5e-3, 1e-5])
    coef[rng.random(4) < 0.3] = 0.0
    t = _design(n, ell) @ coef + rng.normal(0, 0.02, m)
    return n, ell, t


@pytest.mark.parametrize("seed", range(25))
def test_matches_scipy_nnls(seed):
    n, ell, t = _samples(900 + seed)
    a, b, c, e, rms = oracle.cost_fit(n, ell, t)
    X = _design(n, ell)
    s = np.linalg.norm(X, axis=0)
    ref = scipy_nnls(X / s, t)[0] / s
    np.testing.assert_allclose([a, b, c, e], ref, rtol=1e-7, atol=1e-12)
    beta = np.array([a, b, c, e])
    assert (beta >= 0).all()
    np.testing.assert_allclose(rms, np.sqrt(np.mean((X @ beta - t) ** 2)), rtol=1e-12)


@pytest.mark.parametrize("seed", range(10))
def test_kkt_conditions(seed):
    n, ell, t = _samples(1200 + seed, m=40)
    beta = np.array(oracle.cost_fit(n, ell, t)[:4])
    X = _design(n, ell)
    s = np.linalg.norm(X, axis=0)
    xs = beta * s
    w = (X / s).T @ (t - X @ beta)      # negative gradient in the scaled variables
    assert (xs >= 0).all()
    assert (w[xs == 0] <= 1e-8).all()
    np.testing.assert_allclose(w[xs > 0], 0.0, atol=1e-8)


def test_recovers_noiseless_convex_cost():
    n = np.repeat(np.arange(1, 513, 17), 3).astype(np.float64)
    ell = np.tile([512.0, 4096.0, 32768.0], len(n) // 3)
    coef = np.array([2.0, 1e-4, 5e-3, 1e-5])        # the configurations' cost
    t = _design(n, ell) @ coef
    a, b, c, e, rms = oracle.cost_fit(n, ell, t)
    np.testing.assert_allclose([a, b, c, e], coef, rtol=1e-9)
    assert rms < 1e-10


def test_concave_data_keeps_e_at_zero():
    n = np.arange(1, 200, dtype=np.float64)
    ell = np.full_like(n, 4096.0)
    t = 3.0 + 0.02 * n - 4e-5 * n * n                # concave in n: the fit cannot follow
    a, b, c, e, _ = oracle.cost_fit(n, ell, t)
    assert e == 0.0 and c > 0.0


def test_planted_mistake_is_caught():
    """A fit that keeps a negative coefficient (the unconstrained least squares)
    differs from the oracle on concave data."""
    n = np.arange(1, 200, dtype=np.float64)
    ell = np.full_like(n, 4096.0)
    t = 3.0 + 0.02 * n - 4e-5 * n * n
    X = _design(n, ell)
    free = np.linalg.lstsq(X, t, rcond=None)[0]
    assert free[3] < 0
    assert not np.allclose(free, oracle.cost_fit(n, ell, t)[:4])
