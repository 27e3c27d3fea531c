"""Metamorphic pins of the oracle (CPU only): transformations of the inputs whose
effect on the outputs follows from the definitions, whatever the values.

* Token relabeling. A permutation pi of the vocabulary applied everywhere maps
  each tree onto itself with relabeled tokens. It acts on the columns of the
  logits, the rows of E and the columns of W, the anchor, and the columns of
  the target logits. Scores, counts and acceptance lengths are unchanged.
  Nothing in PCTree, CaDDTree or greedy verification depends on token ids
  except through these inputs and the tie order, and random inputs have no
  ties. This catches index mistakes that value-based pins can miss.
* Per-depth shifts. Adding a constant to every logit of one depth leaves that
  depth's log-softmax, and so every tree, unchanged (PCTree article, the
  softmax over the vocabulary in the path score; CaDDTree summary, the
  marginals q_d).
"""
import numpy as np
import pytest

import oracle


def _paths(res, b):
    """{token path: score} of request b's tree (path excludes the root)."""
    n = int(res.count[b])
    paths = {0: ()}
    out = {}
    for i in range(1, n):
        p = paths[int(res.parent[b, i])] + (int(res.tok[b, i]),)
        paths[i] = p
        out[p] = float(res.score[b, i])
    return out


def _relabel(paths, perm):
    return {tuple(int(perm[v]) for v in p): s for p, s in paths.items()}


def _same(a, b, atol=1e-9):
    assert set(a) == set(b)
    for p in a:
        assert abs(a[p] - b[p]) <= atol, (p, a[p], b[p])


@pytest.mark.parametrize("seed", range(6))
def test_pctree_token_relabeling(seed):
    rng = np.random.default_rng(900 + seed)
    V, D, r, k, beam, N = 24, 4, 3, 3, 5, 14
    L = rng.normal(0, 2.0, size=(2, D, V))
    E = rng.normal(0, 0.7, size=(V, r))
    W = rng.normal(0, 0.7, size=(r, V))
    anchor = rng.integers(0, V, 2)
    perm = rng.permutation(V)
    inv = np.argsort(perm)
    L2 = L[:, :, inv]              # L2[..., perm[v]] = L[..., v]
    E2 = E[inv]
    W2 = W[:, inv]
    a = oracle.pct_tree_build(L, anchor, E, W, k, beam, N)
    b = oracle.pct_tree_build(L2, perm[anchor], E2, W2, k, beam, N)
    for q in range(2):
        assert a.count[q] == b.count[q]
        _same(_relabel(_paths(a, q), perm), _paths(b, q))


@pytest.mark.parametrize("seed", range(6))
def test_caddtree_token_relabeling(seed):
    rng = np.random.default_rng(950 + seed)
    V, D = 40, 5
    L = rng.normal(0, 1.5, size=(3, D, V))
    L[np.arange(3)[:, None], np.arange(D)[None, :], rng.integers(0, V, (3, D))] += 4.0
    anchor = rng.integers(0, V, 3)
    ctx = np.array([512, 4096, 32768])
    perm = rng.permutation(V)
    L2 = L[:, :, np.argsort(perm)]
    cost = dict(C_d=1.0, a=2.0, b=1e-4, c=5e-3, e=1e-5)
    a = oracle.cadd_tree_grow(L, anchor, ctx, 64, **cost)
    b = oracle.cadd_tree_grow(L2, perm[anchor], ctx, 64, **cost)
    np.testing.assert_array_equal(a.count, b.count)
    np.testing.assert_allclose(a.phi, b.phi, rtol=1e-12)
    for q in range(3):
        _same(_relabel(_paths(a, q), perm), _paths(b, q))


@pytest.mark.parametrize("seed", range(4))
def test_log_softmax_shift_per_depth(seed):
    rng = np.random.default_rng(990 + seed)
    V, D, r = 20, 4, 2
    L = rng.normal(0, 2.0, size=(1, D, V))
    E = rng.normal(0, 0.7, size=(V, r))
    W = rng.normal(0, 0.7, size=(r, V))
    shift = rng.normal(0, 30.0, size=(1, D, 1))
    a = oracle.pct_tree_build(L, [3], E, W, 3, 4, 12)
    b = oracle.pct_tree_build(L + shift, [3], E, W, 3, 4, 12)
    _same(_paths(a, 0), _paths(b, 0))
    c1 = oracle.cadd_tree_grow(L, [3], [1000], 32, 1.0, 2.0, 1e-4, 5e-3, 1e-5)
    c2 = oracle.cadd_tree_grow(L + shift, [3], [1000], 32, 1.0, 2.0, 1e-4, 5e-3, 1e-5)
    assert c1.count[0] == c2.count[0]
    _same(_paths(c1, 0), _paths(c2, 0))


@pytest.mark.parametrize("seed", range(4))
def test_verify_token_relabeling(seed):
    rng = np.random.default_rng(1010 + seed)
    V, n, Dm = 30, 16, 5
    # a random tree: parent[i] < i, depth <= Dm, distinct sibling tokens
    par = [-1]
    dep = [0]
    tok = [int(rng.integers(0, V))]
    for i in range(1, n):
        cand = [j for j in range(i) if dep[j] < Dm]
        p = int(rng.choice(cand))
        used = {tok[c] for c in range(1, i) if par[c] == p}
        t = int(rng.choice([v for v in range(V) if v not in used]))
        par.append(p); dep.append(dep[p] + 1); tok.append(t)
    tok, par = np.array([tok], np.int32), np.array([par], np.int32)
    cnt = np.array([n], np.int32)
    T = rng.normal(0, 2.0, size=(1, n, V))
    # plant the walk along a few children so that acceptance goes deep
    cur = 0
    for _ in range(3):
        kids = [c for c in range(1, n) if par[0, c] == cur]
        if not kids:
            break
        c = int(rng.choice(kids))
        T[0, cur, tok[0, c]] = 20.0
        cur = c
    perm = rng.permutation(V).astype(np.int32)
    a = oracle.tree_verify_accept(tok, par, cnt, T, max_depth=Dm)
    b = oracle.tree_verify_accept(perm[tok], par, cnt, T[:, :, np.argsort(perm)], max_depth=Dm)
    assert a.accept_len[0] == b.accept_len[0] and a.accept_len[0] >= 1
    np.testing.assert_array_equal(a.accept_path, b.accept_path)
    assert perm[a.correction[0]] == b.correction[0]
    np.testing.assert_array_equal(perm[a.argmax[0, :n]], b.argmax[0, :n])
