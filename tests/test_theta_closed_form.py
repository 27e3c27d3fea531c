"""The closed form of theta that the CaDDTree row-pass filter uses.

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
summary), "Method: CaDDTree": a node can only be added while its prefix
probability exceeds (1 + Phi) dC(n) / C(n), so no token whose marginal is at
most theta = min over n in [1, n_max - 1] of dC(n) / C(n) can enter the tree
(dC(n) = C(n + 1) - C(n), C(n) = C_d + a + b l + c n + e n^2, c, e >= 0).

The row-pass kernel evaluates theta as min(f(1), f(n_max - 1)), f = dC / C,
when C(1) > 0, and uses no filter (theta = 0) when c = e = 0 or C(1) <= 0.
The reason is that with c, e >= 0 the derivative of f has the sign of
-2e^2 n^2 - 2e(c + e) n + (2eA - c^2 - ce), A = C_d + a + b l. That is a
parabola opening downwards, so for n > 0 f only falls, or rises then falls,
and its minimum over an interval is at an end. This test checks the claim
against the definition (brute force over every n) on random costs, including
ones where C(n) <= 0 for the first few n, where the kernel keeps no filter.
"""
import numpy as np
import pytest


def _theta_brute(A, c, e, n_max):
    n = np.arange(1, n_max, dtype=np.float64)
    C = A + c * n + e * n * n
    dC = c + e * (2 * n + 1)
    if (dC <= 0).any():
        return 0.0
    ok = C > 0
    return float((dC[ok] / C[ok]).min()) if ok.any() else 0.0


def _theta_closed(A, c, e, n_max):
    """The kernel's rule, in float64."""
    if n_max < 2 or not (c > 0 or e > 0):
        return 0.0
    C1 = A + c + e
    if not C1 > 0:
        return 0.0
    f = lambda k: (c + e * (2 * k + 1)) / (A + c * k + e * k * k)
    return min(f(1.0), f(float(n_max - 1)))


@pytest.mark.parametrize("seed", range(4))
def test_closed_form_equals_minimum_over_n(seed):
    rng = np.random.default_rng(seed)
    checked = 0
    for _ in range(5000):
        n_max = int(rng.integers(2, 1025))
        A = float(rng.uniform(0.01, 5.0)) + float(rng.uniform(0, 1e-3)) * float(rng.uniform(0, 1e5))
        c = 0.0 if rng.random() < 0.1 else float(rng.uniform(0, 0.05) * 10 ** rng.uniform(-6, 0))
        e = 0.0 if rng.random() < 0.1 else float(rng.uniform(0, 1e-3) * 10 ** rng.uniform(-6, 0))
        want = _theta_brute(A, c, e, n_max)
        got = _theta_closed(A, c, e, n_max)
        assert got == pytest.approx(want, rel=1e-12, abs=0.0), (A, c, e, n_max)
        checked += 1
    assert checked == 5000


def test_interior_maximum_case():
    """A cost whose ratio rises and then falls over the range (2eA > c^2 + ce):
    the minimum is still at an end, here at n = 1."""
    A, c, e, n_max = 50.0, 1e-3, 1e-3, 1024
    n = np.arange(1, n_max, dtype=np.float64)
    f = (c + e * (2 * n + 1)) / (A + c * n + e * n * n)
    assert f.argmax() not in (0, len(f) - 1)          # a real interior maximum
    assert _theta_closed(A, c, e, n_max) == pytest.approx(f.min(), rel=1e-12)
    assert f.argmin() == 0


def test_nonpositive_leading_costs_keep_everything():
    """C(1) <= 0: the growth reports the cost as bad and the filter keeps every
    token. The kernel's value is then no threshold at all, which is safe (a
    superset) whatever the minimum over the n with C(n) > 0 is."""
    A, c, e, n_max = -0.5, 0.01, 1e-4, 512
    assert A + c + e <= 0
    assert _theta_closed(A, c, e, n_max) == 0.0
    assert _theta_brute(A, c, e, n_max) > 0.0
