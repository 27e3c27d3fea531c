"""The non-negative fit of C_v(n; l) = a + b l + c n + e n^2 (host side).

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science),
"Method: CaDDTree": the verification cost is profiled offline as a convex,
non-decreasing function of the tree size (and of the context length), i.e.
a, b, c, e >= 0. The solver is pinned to SciPy's NNLS (an independent
implementation of the same problem) and to coefficient recovery on noiseless
samples; the KKT conditions are checked directly.
"""
import numpy as np
import pytest
from scipy.optimize import nnls as scipy_nnls

from speculative_decoding_draft_07_b200 import costfit


@pytest.mark.parametrize("seed", range(30))
def test_nnls_matches_scipy(seed):
    rng = np.random.default_rng(1400 + seed)
    m, k = int(rng.integers(4, 40)), int(rng.integers(1, 6))
    A = rng.normal(size=(m, k))
    y = rng.normal(size=m) * 2
    ours = costfit.nnls(A, y)
    ref, _ = scipy_nnls(A, y)
    np.testing.assert_allclose(ours, ref, atol=1e-9, rtol=1e-7)
    # KKT: x >= 0, gradient w = A^T (y - A x) <= 0 where x = 0 and == 0 where x > 0
    w = A.T @ (y - A @ ours)
    assert (ours >= 0).all()
    assert (w[ours == 0] <= 1e-8).all()
    np.testing.assert_allclose(w[ours > 0], 0.0, atol=1e-8)


def test_recovers_coefficients_from_exact_samples():
    rng = np.random.default_rng(7)
    n = rng.integers(1, 512, 300).astype(float)
    ell = rng.choice([512, 4096, 32768], 300).astype(float)
    a, b, c, e = 2.0, 1e-4, 5e-3, 1e-5
    t = a + b * ell + c * n + e * n * n
    r = costfit.fit_cost(n, ell, t)
    assert r["a"] == pytest.approx(a, rel=1e-6)
    assert r["b"] == pytest.approx(b, rel=1e-6)
    assert r["c"] == pytest.approx(c, rel=1e-6)
    assert r["e"] == pytest.approx(e, rel=1e-6)
    assert r["rms"] < 1e-9


def test_concave_data_gets_a_convex_fit():
    """Latencies that flatten with n (concave) would want e < 0; the fit keeps e = 0
    and matches SciPy on the same scaled design."""
    n = np.arange(1, 200, dtype=float)
    ell = np.full_like(n, 1000.0)
    t = 3.0 + 0.05 * n - 1e-4 * n * n
    r = costfit.fit_cost(n, ell, t)
    assert r["e"] == 0.0 and r["c"] > 0
    X = np.stack([np.ones_like(n), ell, n, n * n], axis=1)
    s = np.linalg.norm(X, axis=0)
    ref, _ = scipy_nnls(X / s, t)
    np.testing.assert_allclose([r["a"], r["b"], r["c"], r["e"]], ref / s, rtol=1e-7, atol=1e-12)
