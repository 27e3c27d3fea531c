"""Pins of the CaDDTree oracle (CPU only).

Cost-Aware Diffusion Draft Trees (gist.science summary), "Method: CaDDTree":
best-first growth by prefix probability, throughput (1 + Phi) / (C_d + C_v),
unimodal under a convex C_v, greedy stop at the first non-positive gain.
"""
import math

import numpy as np
import pytest

import brute
import oracle


def _sharp(rng, D, V, scale=1.0):
    return rng.normal(0, scale, size=(D, V))


@pytest.mark.parametrize("seed,V,D", [(0, 3, 4), (1, 4, 3), (2, 5, 3), (3, 2, 6), (4, 6, 2)])
def test_best_first_is_top_prefix_probability_for_every_n(seed, V, D):
    """Stop disabled (c = e = 0, constant cost): T_n = root + the n-1 best paths."""
    rng = np.random.default_rng(seed)
    L = _sharp(rng, D, V, 1.5)
    scores = brute.marginal_path_scores(L.tolist())
    order = brute.ranked(scores)
    for n in range(1, min(40, len(order) + 1) + 1):
        r = oracle.cadd_tree_grow(L[None], [1], [0], n_max=n, C_d=1.0, a=0.0, b=0.0, c=0.0, e=0.0)
        tok, par, dep, sc = brute.canonical_table(1, order[: n - 1], scores)
        assert r.count[0] == n
        assert list(r.tok[0, :n]) == tok and list(r.parent[0, :n]) == par
        assert list(r.depth[0, :n]) == dep
        np.testing.assert_allclose(r.score[0, :n], sc, atol=1e-12)
        phi = sum(math.exp(scores[p]) for p in order[: n - 1])
        assert abs(r.phi[0] - phi) < 1e-12


def _convex_cost(rng):
    return dict(C_d=float(rng.uniform(0.2, 2)), a=float(rng.uniform(0, 2)), b=float(rng.uniform(0, 1e-3)),
                c=float(rng.uniform(0, 0.05)), e=float(rng.uniform(0, 2e-3)))


@pytest.mark.parametrize("seed", range(12))
def test_greedy_stop_is_exhaustive_argmax(seed):
    """n* equals the smallest argmax of f(n) = (1 + Phi_n) / C(n) over n in [1, n_max]."""
    rng = np.random.default_rng(50 + seed)
    V, D = int(rng.integers(2, 6)), int(rng.integers(2, 5))
    L = _sharp(rng, D, V, float(rng.uniform(0.5, 3.0)))
    cost = _convex_cost(rng)
    ell = float(rng.integers(0, 40000))
    scores = brute.marginal_path_scores(L.tolist())
    order = brute.ranked(scores)
    n_max = len(order) + 1
    f, phi = [], 0.0
    for n in range(1, n_max + 1):
        if n > 1:
            phi += math.exp(scores[order[n - 2]])
        C = cost["C_d"] + cost["a"] + cost["b"] * ell + cost["c"] * n + cost["e"] * n * n
        f.append((1 + phi) / C)
    best = max(range(len(f)), key=lambda i: (f[i], -i)) + 1
    r = oracle.cadd_tree_grow(L[None], [0], [ell], n_max=n_max, **cost)
    assert r.count[0] == best
    np.testing.assert_allclose(r.f_values[0][-1], f[best - 1], rtol=1e-12)


@pytest.mark.parametrize("seed", range(20))
def test_objective_is_unimodal_under_convex_cost(seed):
    rng = np.random.default_rng(200 + seed)
    V, D = int(rng.integers(2, 5)), int(rng.integers(2, 5))
    L = _sharp(rng, D, V, float(rng.uniform(0.3, 3.0)))
    cost = _convex_cost(rng)
    scores = brute.marginal_path_scores(L.tolist())
    order = brute.ranked(scores)
    phi, f = 0.0, []
    for n in range(1, len(order) + 2):
        if n > 1:
            phi += math.exp(scores[order[n - 2]])
        f.append((1 + phi) / (cost["C_d"] + cost["a"] + cost["c"] * n + cost["e"] * n * n))
    g = np.diff(f)
    # once the gain turns non-positive it never becomes positive again
    first = next((i for i, x in enumerate(g) if x <= 0), len(g))
    assert (g[first:] <= 1e-15).all()


def test_nonconvex_cost_can_break_unimodality():
    """With e < 0 (concave C_v) some objectives rise again after falling."""
    rng = np.random.default_rng(9)
    found = False
    for _ in range(400):
        V, D = 3, 3
        L = _sharp(rng, D, V, float(rng.uniform(0.3, 3.0)))
        scores = brute.marginal_path_scores(L.tolist())
        order = brute.ranked(scores)
        c, e = float(rng.uniform(0.05, 0.5)), -float(rng.uniform(0.001, 0.02))
        phi, f = 0.0, []
        for n in range(1, len(order) + 2):
            if n > 1:
                phi += math.exp(scores[order[n - 2]])
            C = 1.0 + c * n + e * n * n
            if C <= 0:
                break
            f.append((1 + phi) / C)
        g = np.diff(f)
        first = next((i for i, x in enumerate(g) if x <= 0), len(g))
        if (g[first:] > 1e-9).any():
            found = True
            break
    assert found


def test_uniform_marginals_closed_form():
    """Equal logits, V = 4, D = 2, C(n) = 1 + 0.1 n.

    Every depth-1 node has P = 1/4, every depth-2 node 1/16. f(n) for n = 1..5
    is 1/1.1, 1.25/1.2, 1.5/1.3, 1.75/1.4, 2/1.5 (rising); adding a depth-2 node
    gives 2.0625/1.6 < 2/1.5, so n* = 5, Phi = 1, and the tree is the root with
    its four children in token order.
    """
    L = np.zeros((1, 2, 4)) + 0.37
    r = oracle.cadd_tree_grow(L, [2], [0], n_max=64, C_d=1.0, a=0.0, b=0.0, c=0.1, e=0.0)
    assert r.count[0] == 5 and abs(r.phi[0] - 1.0) < 1e-12 and r.stop_reason[0] == "gain"
    assert list(r.tok[0, :5]) == [2, 0, 1, 2, 3] and list(r.parent[0, :5]) == [-1, 0, 0, 0, 0]
    np.testing.assert_allclose(r.score[0, 1:5], math.log(0.25), atol=1e-12)


def test_context_length_raises_budget():
    """A longer context raises the fixed verification cost, which favours larger trees."""
    rng = np.random.default_rng(3)
    L = rng.normal(0, 2.0, size=(3, 6, 400))
    n = []
    for ell in (512, 4096, 32768):
        r = oracle.cadd_tree_grow(L, [0, 1, 2], [ell] * 3, n_max=512, C_d=1.0, a=2.0, b=1e-4,
                                  c=5e-3, e=1e-5)
        n.append(r.count)
    assert (n[0] <= n[1]).all() and (n[1] <= n[2]).all() and (n[2] > n[0]).any()


def test_monte_carlo_acceptance_equals_phi():
    """Phi(T) is the expected number of accepted drafts when target tokens are drawn from q_d."""
    rng = np.random.default_rng(11)
    V, D = 5, 4
    L = rng.normal(0, 1.5, size=(D, V))
    r = oracle.cadd_tree_grow(L[None], [0], [0], n_max=25, C_d=1.0, a=0.0, b=0.0, c=0.0, e=0.0)
    n = r.count[0]
    tok, par = r.tok[0, :n], r.parent[0, :n]
    q = np.exp(L - L.max(1, keepdims=True))
    q /= q.sum(1, keepdims=True)
    trials = 100_000
    draws = np.stack([rng.choice(V, size=trials, p=q[d]) for d in range(D)], 1)
    child = {}
    for i in range(1, n):
        child[(int(par[i]), int(tok[i]))] = i
    acc = np.zeros(trials)
    for t in range(trials):
        u, a = 0, 0
        for d in range(D):
            u = child.get((u, int(draws[t, d])))
            if u is None:
                break
            a += 1
        acc[t] = a
    sigma = acc.std() / math.sqrt(trials)
    assert abs(acc.mean() - r.phi[0]) < 4 * sigma + 1e-12


def test_exhausted_and_cap():
    L = np.zeros((1, 1, 3))
    r = oracle.cadd_tree_grow(L, [0], [0], n_max=10, C_d=1.0, a=0.0, b=0.0, c=0.0, e=0.0)
    assert r.count[0] == 4 and r.stop_reason[0] == "exhausted"
    r = oracle.cadd_tree_grow(L, [0], [0], n_max=2, C_d=1.0, a=0.0, b=0.0, c=0.0, e=0.0)
    assert r.count[0] == 2 and r.stop_reason[0] == "n_max" and list(r.tok[0]) == [0, 0]
