"""Pins of the oracles' near-tie resolution (``prefer``).

When two candidates at a cut differ by less than the tolerance, either one may
be kept. With ``prefer`` the oracle keeps the preferred one; otherwise nothing
changes. These cases fix what that means on inputs small enough to work out by
hand, and check that a tree whose only differences come from near ties is
reproduced exactly.

PCTree article (qiita), the tree section (local top-k, path score, per-depth
pruning, global top-N); CaDDTree summary (gist.science), "Method: CaDDTree"
(best-first growth, greedy stop).
"""
import math

import numpy as np

import oracle


def _paths(res, b=0):
    """Token paths below the root of request b's tree."""
    tok, par, n = res.tok[b], res.parent[b], int(res.count[b])
    out, paths = set(), {0: ()}
    for i in range(1, n):
        paths[i] = paths[int(par[i])] + (int(tok[i]),)
        out.add(paths[i])
    return out


def _pct(L, E, W, k, beam, N, prefer=None):
    L = np.asarray(L, float)[None]
    return oracle.pct_tree_build(L, np.array([0]), E, W, k, beam, N,
                                 prefer=None if prefer is None else [prefer])


def _zero_markov(V, r=2):
    return np.zeros((V, r)), np.zeros((r, V))


def test_global_cut_follows_preference_only_inside_tolerance():
    # one depth, k = V, one node besides the root: the two best tokens differ by 5e-5
    V = 4
    E, W = _zero_markov(V)
    L = [[1.0, 1.0 - 5e-5, 0.0, -1.0]]
    assert _paths(_pct(L, E, W, V, V, 2)) == {(0,)}
    assert _paths(_pct(L, E, W, V, V, 2, prefer={(1,)})) == {(1,)}
    # 5e-4 apart: the preference cannot override the order
    L = [[1.0, 1.0 - 5e-4, 0.0, -1.0]]
    assert _paths(_pct(L, E, W, V, V, 2, prefer={(1,)})) == {(0,)}


def test_local_top_k_follows_preference():
    # k = 1 child per parent, unlimited beam and budget: depth 1 keeps one token
    V = 5
    E, W = _zero_markov(V)
    L = [[0.0, 2.0, 2.0 - 3e-5, 0.5, 0.1]]
    assert _paths(_pct(L, E, W, 1, 8, 10)) == {(1,)}
    assert _paths(_pct(L, E, W, 1, 8, 10, prefer={(2,)})) == {(2,)}


def test_beam_cut_follows_preference_and_changes_descendants():
    # depth 1 keeps both tokens 0 and 1 (k = 2); the beam of 1 at depth 2 picks
    # between (0, 3) and (1, 3), whose scores differ by 2e-5 (from depth 1)
    V = 4
    E, W = _zero_markov(V)
    L = [[1.0, 1.0 - 2e-5, -9.0, -9.0],
         [-9.0, -9.0, -9.0, 3.0]]
    base = _paths(_pct(L, E, W, 2, 1, 3))
    assert base == {(0,), (0, 3)}
    got = _paths(_pct(L, E, W, 2, 1, 3, prefer={(1,), (1, 3)}))
    assert got == {(1,), (1, 3)}


def test_preferring_the_oracles_own_tree_changes_nothing():
    rng = np.random.default_rng(5)
    for _ in range(10):
        V, D, r = 7, 3, 3
        L = rng.normal(0, 1, (D, V)).round(1)           # coarse values: many exact ties
        E, W = rng.normal(0, 0.3, (V, r)), rng.normal(0, 0.3, (r, V))
        ref = _pct(L, E, W, 3, 4, 9)
        got = _pct(L, E, W, 3, 4, 9, prefer=_paths(ref))
        np.testing.assert_array_equal(got.tok, ref.tok)
        np.testing.assert_array_equal(got.parent, ref.parent)


def test_tree_from_perturbed_inputs_is_reproduced():
    """Inputs with many exact ties, perturbed by at most 1e-6: the tree built on
    the perturbed inputs differs from the unperturbed one only by near-tie
    flips, and resolving the unperturbed oracle's near ties toward it gives it
    back exactly (several of the cases do flip)."""
    rng = np.random.default_rng(11)
    flipped = 0
    for _ in range(40):
        V, D, r = 6, 3, 2
        L = rng.integers(-4, 4, (D, V)) / 4.0
        E, W = np.zeros((V, r)), np.zeros((r, V))
        Lp = L + rng.uniform(-1e-6, 1e-6, L.shape)
        ref = _pct(L, E, W, 2, 3, 7)
        per = _pct(Lp, E, W, 2, 3, 7)
        want = _paths(per)
        flipped += want != _paths(ref)
        got = _pct(L, E, W, 2, 3, 7, prefer=want)
        assert _paths(got) == want
    assert flipped >= 5


def _cadd(L, n_max, cost, prefer=None, ell=0):
    L = np.asarray(L, float)[None]
    return oracle.cadd_tree_grow(L, np.array([0]), np.array([ell]), n_max, **cost,
                                 prefer=None if prefer is None else [prefer])


def test_cadd_near_tie_pop_follows_preference():
    # stop disabled (c = e = 0), room for two nodes. After (0,) is added, the
    # candidates are its sibling (1,) and its child (0, 0); their scores differ
    # by gap. (Within one row the order is that of the input values on both
    # sides, so the near ties that matter are between different parents.)
    cost = dict(C_d=1.0, a=1.0, b=0.0, c=0.0, e=0.0)
    q2_0 = -math.log(1.0 + math.exp(-2.0) + math.exp(-30.0))     # log q_2(0)
    for gap, follows in ((3e-5, True), (3e-4, False)):
        delta = -q2_0 + gap                                        # q_1(0) - q_1(1)
        L = [[0.0, -delta, -30.0], [0.0, -2.0, -30.0]]
        assert _paths(_cadd(L, 3, cost)) == {(0,), (0, 0)}
        got = _paths(_cadd(L, 3, cost, prefer=({(0,), (1,)}, 3)))
        assert got == ({(0,), (1,)} if follows else {(0,), (0, 0)})


def test_cadd_stop_near_flip_follows_preferred_count():
    # one depth, uniform over V tokens: every candidate has p = 1/V. With C(n) =
    # 1 + c n the first node is added iff 1/V > (1 + Phi) c / (1 + c); choose c
    # so that the two sides differ by 1e-5 in log (inside 2 tol)
    V = 10
    p = 1.0 / V
    # log p - log(c / (1 + c)) = delta  ->  c / (1 + c) = p e^-delta
    for delta, default_n in ((+1e-5, 2), (-1e-5, 1)):
        x = p * math.exp(-delta)
        c = x / (1 - x)
        cost = dict(C_d=0.0, a=1.0, b=0.0, c=c, e=0.0)
        ref = _cadd(np.zeros((1, V)), 2, cost)
        assert int(ref.count[0]) == default_n
        other = 3 - default_n
        got = _cadd(np.zeros((1, V)), 2, cost, prefer=({(0,)}, other))
        assert int(got.count[0]) == other
    # far from the flip (delta = 0.1): the preferred count is ignored
    x = p * math.exp(-0.1)
    cost = dict(C_d=0.0, a=1.0, b=0.0, c=x / (1 - x), e=0.0)
    assert int(_cadd(np.zeros((1, V)), 2, cost, prefer=({(0,)}, 1)).count[0]) == 2
