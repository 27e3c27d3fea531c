"""Pins of oracle.row_topk: each row's k largest logits, value descending,
equal values to the lower token id.

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science),
"Method: CaDDTree": growth is best-first by prefix probability, so a
position's tokens are taken by decreasing marginal, i.e. by decreasing logit.
"""
import numpy as np
import pytest

import oracle


def _rank_brute(row):
    """Position of every token in the order: the tokens that come before it."""
    V = len(row)
    return [sum(1 for u in range(V) if row[u] > row[v] or (row[u] == row[v] and u < v))
            for v in range(V)]


@pytest.mark.parametrize("seed", range(12))
def test_matches_pairwise_count(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(1, 24))
    k = int(rng.integers(1, 12))
    row = rng.integers(-3, 4, V).astype(np.float64)      # many exact ties
    if V > 2:
        row[rng.integers(0, V)] = -np.inf
    got = oracle.row_topk(row[None], k)[0]
    rank = _rank_brute(row)
    for j in range(k):
        if j < V:
            assert rank[got[j]] == j, (row, got)
        else:
            assert got[j] == -1


def test_ties_go_to_the_lower_token():
    row = np.array([1.0, 5.0, 5.0, 2.0, 5.0])
    np.testing.assert_array_equal(oracle.row_topk(row[None], 4)[0], [1, 2, 4, 3])


def test_shape_and_padding():
    L = np.zeros((2, 3, 4))
    out = oracle.row_topk(L, 6)
    assert out.shape == (2, 3, 6) and out.dtype == np.int32
    np.testing.assert_array_equal(out[1, 2], [0, 1, 2, 3, -1, -1])


@pytest.mark.parametrize("seed", range(4))
def test_agrees_with_best_first_children_of_the_root(seed):
    """D = 1 and the stop disabled (c = e = 0): the tree of n_max = k + 1 nodes
    is the root and its k best children, which are the row's k best tokens."""
    rng = np.random.default_rng(100 + seed)
    V, k = 50, 7
    L = rng.normal(0, 2, (1, 1, V))
    tree = oracle.cadd_tree_grow(L, np.array([0]), np.array([512]), k + 1, C_d=1.0, a=2.0,
                                 b=0.0, c=0.0, e=0.0)
    assert tree.count[0] == k + 1
    assert set(tree.tok[0, 1:].tolist()) == set(oracle.row_topk(L, k)[0, 0].tolist())


def test_planted_mistake_is_caught():
    """Ties broken toward the higher token id: the pairwise count tells."""
    def mutant(L, k):
        row = np.asarray(L, dtype=np.float64)[0]
        V = len(row)
        order = (V - 1 - np.argsort(-row[::-1], kind="stable"))[:k]
        return order[None]

    row = np.array([1.0, 5.0, 5.0, 2.0, 5.0])
    rank = _rank_brute(row)
    got = mutant(row[None], 3)[0]
    assert any(rank[got[j]] != j for j in range(3))
    good = oracle.row_topk(row[None], 3)[0]
    assert all(rank[good[j]] == j for j in range(3))
