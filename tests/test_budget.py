"""The fixed-versus-adaptive budget sweep (host side) against the CaDDTree oracle.

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science),
"Method: CaDDTree": the tree of size n is the best-first tree of the n - 1 most
probable nodes whatever the cost, and CaDDTree stops at the first size whose
successor does not raise (1 + Phi_n) / C(n). So the Phi curve of one tree grown
with the stop disabled must reproduce the oracle's adaptive size, Phi and
objective values for every cost.
"""
import numpy as np
import pytest

import oracle
from speculative_decoding_draft_07_b200 import budget


def _fixed_trees(L, anchor, n):
    """The oracle's tree grown with the stop disabled (c = e = 0)."""
    return oracle.cadd_tree_grow(L, anchor, np.zeros(len(anchor)), n, C_d=1.0, a=0.0, b=0.0,
                                 c=0.0, e=0.0)


@pytest.mark.parametrize("seed", range(5))
def test_adaptive_size_and_phi_match_the_oracle(seed):
    rng = np.random.default_rng(1200 + seed)
    batch, D, V, n_max = 8, 5, 30, 64
    L = rng.normal(0, 1.5, size=(batch, D, V))
    L[np.arange(batch)[:, None], np.arange(D)[None, :], rng.integers(0, V, (batch, D))] += \
        rng.uniform(0, 6, size=(batch, D))
    anchor = rng.integers(0, V, batch)
    ctx = rng.integers(0, 40000, batch)
    fixed = _fixed_trees(L, anchor, n_max)
    assert (fixed.count == n_max).all()
    for trial in range(4):
        cost = dict(C_d=float(rng.uniform(0.2, 2)), a=float(rng.uniform(0, 3)),
                    b=float(rng.uniform(0, 1e-3)), c=float(rng.uniform(0, 0.05)),
                    e=float(rng.uniform(0, 1e-3)))
        ref = oracle.cadd_tree_grow(L, anchor, ctx, n_max, **cost)
        for q in range(batch):
            if ref.excluded[q]:
                continue
            phi = budget.phi_curve(fixed.score[q], int(fixed.count[q]))
            n = budget.adaptive_size(phi, float(ctx[q]), *cost.values(), n_max=n_max)
            assert n == ref.count[q], (seed, trial, q)
            assert phi[n - 1] == pytest.approx(ref.phi[q], rel=1e-12, abs=1e-15)
            f = budget.objective_curve(phi, float(ctx[q]), *cost.values())[:n]
            np.testing.assert_allclose(f, ref.f_values[q], rtol=1e-12)


def test_exhausted_tree_ends_the_curve():
    """A vocabulary of 2 and D = 2 has 6 non-root nodes: the curve ends at n = 7."""
    L = np.array([[[0.0, 1.0], [2.0, 0.0]]])
    fixed = _fixed_trees(L, [0], 20)
    assert fixed.count[0] == 7
    phi = budget.phi_curve(fixed.score[0], 7)
    assert len(phi) == 7 and phi[-1] == pytest.approx(fixed.phi[0], rel=1e-12)
    assert budget.adaptive_size(phi, 0.0, 1.0, 0.0, 0.0, 0.0, 0.0) == 7


def test_sweep_by_hand():
    """Two rounds with Phi = [0, .9, 1.5, 1.8] and [0, .5, .7, .8], C(n) = 1 + 0.2 n.

    Fixed n: tokens 2 + (Phi1 + Phi2)(n), cost 2 (1 + 0.2 n):
      n=1: 2 / 2.4 = 0.8333; n=2: 3.4 / 2.8 = 1.2143; n=3: 4.2 / 3.2 = 1.3125;
      n=4: 4.6 / 3.6 = 1.2778 -> best fixed n = 3.
    Adaptive, round 1: f = 1/1.2, 1.9/1.4, 2.5/1.6, 2.8/1.8 = .833, 1.357, 1.5625,
      1.556 -> n* = 3; round 2: 1/1.2, 1.5/1.4, 1.7/1.6, 1.8/1.8 = .833, 1.071,
      1.0625 -> n* = 2. Rate (2.5 + 1.5) / (1.6 + 1.4) = 4 / 3.
    """
    phis = [np.array([0.0, 0.9, 1.5, 1.8]), np.array([0.0, 0.5, 0.7, 0.8])]
    cost = (1.0, 0.0, 0.0, 0.2, 0.0)
    r = budget.budget_sweep(phis, [0.0, 0.0], cost)
    assert r["best_fixed_n"] == 3
    assert r["fixed"][1] == pytest.approx(2 / 2.4)
    assert r["fixed"][3] == pytest.approx(4.2 / 3.2)
    assert r["fixed"][4] == pytest.approx(4.6 / 3.6)
    assert list(r["adaptive_sizes"]) == [3, 2]
    assert r["adaptive_rate"] == pytest.approx(4 / 3)
    assert r["gain"] == pytest.approx((4 / 3) / (4.2 / 3.2))
    assert r["adaptive_size_std"] == pytest.approx(0.5)


def test_sweep_with_misestimated_cost():
    """A planner that believes verification is free (c = e = 0) grows every round to
    its end; the rate is still measured under the true cost."""
    phis = [np.array([0.0, 0.9, 1.5, 1.8]), np.array([0.0, 0.5, 0.7, 0.8])]
    r = budget.budget_sweep(phis, [0.0, 0.0], (1.0, 0.0, 0.0, 0.2, 0.0),
                            plan_cost=(1.0, 0.0, 0.0, 0.0, 0.0))
    assert list(r["adaptive_sizes"]) == [4, 4]
    assert r["adaptive_rate"] == pytest.approx(r["fixed"][4])
