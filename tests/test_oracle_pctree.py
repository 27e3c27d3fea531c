"""Pins of the PCTree oracle (CPU only).

PCTree article (qiita), section on the chain draft's weakness and the tree that
replaces it: per-parent scores z_d(p) = L_d + Markov(p), local top-k, path score
sum log pi(v|u), per-depth pruning, global top-N. Each test pins the oracle to
something other than itself.
"""
import math

import numpy as np
import pytest

import brute
import oracle
import workloads


def _random_problem(rng, V, D, r, sharp=False):
    L = rng.normal(0, 1.0 if sharp else 2.0, size=(D, V))
    E = rng.normal(0, 0.7, size=(V, r))
    W = rng.normal(0, 0.7, size=(r, V))
    anchor = int(rng.integers(0, V))
    return L, anchor, E, W


@pytest.mark.parametrize("seed,V,D,r,N", [(0, 3, 3, 2, 8), (1, 4, 3, 3, 20), (2, 5, 2, 2, 31),
                                          (3, 3, 4, 1, 40), (4, 6, 2, 4, 12), (5, 2, 5, 2, 63)])
def test_bruteforce_when_nothing_is_pruned(seed, V, D, r, N):
    """k = V and a beam wider than V^D: PCTree equals the top-(N-1) of all paths."""
    rng = np.random.default_rng(seed)
    L, anchor, E, W = _random_problem(rng, V, D, r)
    res = oracle.pct_tree_build(L[None], [anchor], E, W, k=V, beam=V ** D, n_nodes=N)
    scores = brute.conditioned_path_scores(L.tolist(), anchor, E.tolist(), W.tolist())
    sel = brute.ranked(scores)[: N - 1]
    tok, par, dep, sc = brute.canonical_table(anchor, sel, scores)
    n = len(tok)
    assert res.count[0] == n
    np.testing.assert_array_equal(res.tok[0, :n], tok)
    np.testing.assert_array_equal(res.parent[0, :n], par)
    np.testing.assert_array_equal(res.depth[0, :n], dep)
    np.testing.assert_allclose(res.score[0, :n], sc, atol=1e-12)
    assert (res.tok[0, n:] == -1).all() and np.isneginf(res.score[0, n:]).all()


@pytest.mark.parametrize("seed", range(6))
def test_k1_reduces_to_dspark_greedy_chain(seed):
    """k = 1 and N = B: the tree is DSpark's chain y_d = argmax(L_d + Markov(y_{d-1}))."""
    rng = np.random.default_rng(100 + seed)
    V, D, r = 50, 6, 4
    L, anchor, E, W = _random_problem(rng, V, D, r)
    if seed == 0:
        L[2, 7] = L[2, 3] = 40.0       # exact tie in z: both Markov columns are zero
        W[:, 7] = 0.0
        W[:, 3] = 0.0
    res = oracle.pct_tree_build(L[None], [anchor], E, W, k=1, beam=4, n_nodes=D + 1)
    chain, prev = [], anchor
    for d in range(D):
        z = [L[d][v] + sum(E[prev][i] * W[i][v] for i in range(r)) for v in range(V)]
        best = max(range(V), key=lambda v: (z[v], -v))
        chain.append(best)
        prev = best
    assert res.count[0] == D + 1
    assert list(res.tok[0]) == [anchor] + chain
    assert list(res.parent[0]) == [-1] + list(range(D))
    assert list(res.depth[0]) == list(range(D + 1))
    if seed == 0:
        assert chain[2] == 3


def test_hand_derived_finite_beam():
    """V=3, D=2, rank 1, k=2; every number below follows from the definitions by hand.

    E = [1, -1, 0]^T, W = [[1, -1, 0]] so Markov(0) = [1, -1, 0],
    Markov(1) = [-1, 1, 0], Markov(2) = 0. L_1 = [2, 1, 0], L_2 = [0, 0, 0.5],
    anchor 2.
      depth 1: z = [2, 1, 0], lse1 = log(e^2 + e + 1); top-2 children 0, 1.
      depth 2, parent 0: z = [1, -1, 0.5] -> top-2 tokens 0, 2;
               parent 1: z = [-1, 1, 0.5] -> top-2 tokens 1, 2; both rows share
               lse2 = log(e + 1/e + e^0.5).
      scores: (0) 2-lse1, (1) 1-lse1, (0,0) 3-A, (0,2) 2.5-A, (1,1) 2-A,
              (1,2) 1.5-A with A = lse1 + lse2.
      beam 2 keeps (0,0), (0,2); beam 3 also keeps (1,1).
    """
    L = np.array([[2.0, 1.0, 0.0], [0.0, 0.0, 0.5]])
    E = np.array([[1.0], [-1.0], [0.0]])
    W = np.array([[1.0, -1.0, 0.0]])
    e = math.e
    lse1 = math.log(e ** 2 + e + 1)
    A = lse1 + math.log(e + 1 / e + math.exp(0.5))
    s = {(0,): 2 - lse1, (1,): 1 - lse1, (0, 0): 3 - A, (0, 2): 2.5 - A, (1, 1): 2 - A}

    r = oracle.pct_tree_build(L[None], [2], E, W, k=2, beam=2, n_nodes=6)
    assert r.count[0] == 5 and r.frontier_sizes[0] == [2, 2]
    assert list(r.tok[0, :5]) == [2, 0, 1, 0, 2]
    assert list(r.parent[0, :5]) == [-1, 0, 0, 1, 1]
    np.testing.assert_allclose(r.score[0, 1:5], [s[(0,)], s[(1,)], s[(0, 0)], s[(0, 2)]], atol=1e-12)

    r = oracle.pct_tree_build(L[None], [2], E, W, k=2, beam=3, n_nodes=6)
    assert r.count[0] == 6 and r.frontier_sizes[0] == [2, 3]
    assert list(r.tok[0]) == [2, 0, 1, 0, 2, 1]
    assert list(r.parent[0]) == [-1, 0, 0, 1, 1, 2]
    np.testing.assert_allclose(r.score[0, 5], s[(1, 1)], atol=1e-12)

    # global top-N: N = 4 keeps (0), (0,0), (1) -- scores -0.41, -0.96, -1.41
    r = oracle.pct_tree_build(L[None], [2], E, W, k=2, beam=3, n_nodes=4)
    assert list(r.tok[0]) == [2, 0, 1, 0] and list(r.parent[0]) == [-1, 0, 0, 1]


@pytest.mark.parametrize("seed", range(40))
def test_bruteforce_with_finite_k_and_beam(seed):
    """Finite k and beam: the oracle equals the pruned tree defined by predicates over
    every path (eligible = child of a kept path and among its parent's k best by z;
    kept = the beam best eligible paths of the depth; tree = the N-1 best kept)."""
    rng = np.random.default_rng(500 + seed)
    V = int(rng.integers(2, 6))
    D = int(rng.integers(2, 5 if V <= 3 else 4))
    r = int(rng.integers(1, 4))
    k = int(rng.integers(1, V + 1))
    beam = int(rng.integers(1, min(V ** D, 3 * V) + 1))
    N = int(rng.integers(2, 2 + D * beam + 2))
    L, anchor, E, W = _random_problem(rng, V, D, r)
    res = oracle.pct_tree_build(L[None], [anchor], E, W, k=k, beam=beam, n_nodes=N)
    scores = brute.conditioned_path_scores(L.tolist(), anchor, E.tolist(), W.tolist())
    z_of = brute.conditioned_z(L.tolist(), anchor, E.tolist(), W.tolist())
    sel, sizes = brute.pruned_selection(scores, z_of, V, D, k, beam, N)
    assert res.frontier_sizes[0] == sizes
    tok, par, dep, sc = brute.canonical_table(anchor, sel, scores)
    n = len(tok)
    assert res.count[0] == n
    np.testing.assert_array_equal(res.tok[0, :n], tok)
    np.testing.assert_array_equal(res.parent[0, :n], par)
    np.testing.assert_array_equal(res.depth[0, :n], dep)
    np.testing.assert_allclose(res.score[0, :n], sc, atol=1e-12)


def test_zero_markov_matches_best_first_tree():
    """W = 0 and k, beam >= N-1: PCTree's tree is the best-first prefix-probability tree."""
    rng = np.random.default_rng(7)
    V, D, N = 12, 5, 30
    L = rng.normal(0, 1.0, size=(2, D, V))
    L[1, :, 3] += 3.0
    E = rng.normal(0, 1, size=(V, 3))
    W = np.zeros((3, V))
    anchor = [4, 9]
    p = oracle.pct_tree_build(L, anchor, E, W, k=N - 1, beam=N - 1, n_nodes=N)
    c = oracle.cadd_tree_grow(L, anchor, [0, 0], n_max=N, C_d=1.0, a=0.0, b=0.0, c=0.0, e=0.0)
    np.testing.assert_array_equal(p.count, c.count)
    np.testing.assert_array_equal(p.tok, c.tok)
    np.testing.assert_array_equal(p.parent, c.parent)
    np.testing.assert_array_equal(p.depth, c.depth)
    np.testing.assert_allclose(p.score, c.score, atol=1e-12)


@pytest.mark.parametrize("seed,V,D,k,beam,N", [(0, 40, 6, 4, 4, 32), (1, 64, 8, 3, 7, 20),
                                               (2, 30, 5, 8, 16, 64), (3, 16, 10, 2, 5, 100)])
def test_structural_invariants(seed, V, D, k, beam, N):
    rng = np.random.default_rng(seed)
    L, anchor, E, W = _random_problem(rng, V, D, 4)
    r = oracle.pct_tree_build(L[None], [anchor], E, W, k=k, beam=beam, n_nodes=N)
    f, prev = r.frontier_sizes[0], 1
    for size in f:                       # |F_d| = min(beam, |F_{d-1}| * k)
        assert size == min(beam, prev * min(k, V))
        prev = size
    n = r.count[0]
    assert n == min(N, 1 + sum(f))
    tok, par, dep, sc = r.tok[0], r.parent[0], r.depth[0], r.score[0]
    assert tok[0] == anchor and par[0] == -1 and dep[0] == 0 and sc[0] == 0
    for i in range(1, n):
        assert 0 <= par[i] < i and dep[i] == dep[par[i]] + 1
        assert sc[i] <= sc[par[i]] + 1e-15      # log pi <= 0
    keys = [(dep[i], par[i], tok[i]) for i in range(1, n)]
    assert keys == sorted(keys) and len(set(keys)) == len(keys)
    # the selected nodes are the best N-1 of the kept union
    union = sorted((-x.s for x in r.kept[0]))
    if len(union) > N - 1:
        assert max(-sc[1:n]) <= union[N - 2] + 1e-15


def test_tiny_workload_runs_and_is_not_excluded():
    w = workloads.WORKLOADS["tiny"]
    d = workloads.drafter_inputs(w)
    r = oracle.pct_tree_build(oracle.to_f64(d["L"]), d["anchor"].numpy(), oracle.to_f64(d["E"]),
                              oracle.to_f64(d["W"]), w.k, w.beam, w.n_nodes)
    # 4 + 5 * 4 nodes kept, fewer than N - 1 = 31: everything kept
    assert r.count[0] == 25 and r.frontier_sizes[0] == [4, 4, 4, 4, 4, 4]


def test_near_tie_is_reported():
    """Two children of the root whose scores differ by 1e-6: a near tie at the beam cut."""
    V = 5
    L = np.array([[3.0, 1.0, 1.0 + 1e-6, 0.0, -1.0], [0.0] * V])
    E = np.zeros((V, 1))
    W = np.zeros((1, V))
    r = oracle.pct_tree_build(L[None], [0], E, W, k=5, beam=2, n_nodes=10)
    assert r.excluded[0]
    # identical inputs tie exactly: resolved by the lower token id, not excluded
    L[0, 2] = 1.0
    r = oracle.pct_tree_build(L[None], [0], E, W, k=5, beam=2, n_nodes=10)
    assert not r.excluded[0]
    assert sorted(r.tok[0, 1:3]) == [0, 1]
