"""Pins of the acceptance-simulation oracle.

* Philox4x32-10 against the published known answers of the generator (Salmon
  et al., "Parallel random numbers: as easy as 1, 2, 3", SC 2011).
* Walks worked out by hand: a chain whose every child has probability 1 is
  always accepted to the end; probability 0 is never entered; a root with two
  children of probability 0.25 each is left for one of them in about half the
  walks.
* E[accepted] = Phi(T) (CaDDTree summary, "Method: CaDDTree") within four
  standard errors, on PCTree and CaDDTree trees from the tree oracles, with the
  target equal to the drafter (p(child) = exp(s(child) - s(parent))).
"""
import numpy as np

import oracle
from oracle.accept_sim import accept_sim, philox4x32_10, uniform24


def _hex(ctr, key):
    return ["%08x" % v for v in philox4x32_10(np.array(ctr, np.uint32), np.array(key, np.uint32))]


def test_philox_known_answers():
    assert _hex([0, 0, 0, 0], [0, 0]) == ["6627e8d5", "e169c58d", "bc57ac4c", "9b00dbd8"]
    assert _hex([0xffffffff] * 4, [0xffffffff] * 2) == ["408f276d", "41c83b0e", "a20bc7c6", "6d5451fd"]
    assert _hex([0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344], [0xa4093822, 0x299f31d0]) == \
        ["d16cfe09", "94fdcceb", "5001e420", "24126ea1"]


def test_uniform_is_exact_and_in_range():
    w = np.array([0, 255, 256, 0xffffffff], np.uint32)
    u = uniform24(w)
    assert u.dtype == np.float32
    assert list(u) == [0.0, 0.0, np.float32(2.0 ** -24), np.float32(1 - 2.0 ** -24)]


def test_hand_walks():
    # chain 0 -> 1 -> 2 -> 3 with p = 1: every walk accepts 3; a fourth child with p = 0 is never entered
    parent = np.array([[-1, 0, 1, 2, 2]])
    p = np.array([[0, 1, 1, 1, 0]], np.float32)
    h = accept_sim(parent, [5], p, trials=500, seed=3, max_depth=6)
    assert h[0, 3] == 500 and h.sum() == 500
    # the cap: max_depth 2 stops the same chain at 2
    h = accept_sim(parent, [5], p, trials=100, seed=3, max_depth=2)
    assert h[0, 2] == 100
    # root with two leaves of 0.25 each: about half of the walks accept one draft
    parent = np.array([[-1, 0, 0]])
    p = np.array([[0, 0.25, 0.25]], np.float32)
    h = accept_sim(parent, [3], p, trials=20000, seed=9, max_depth=3)
    assert abs(h[0, 1] / 20000 - 0.5) < 4 * np.sqrt(0.25 / 20000)


def _p_child(tok, parent, score, count):
    p = np.zeros(tok.shape, np.float32)
    for b in range(tok.shape[0]):
        for c in range(1, int(count[b])):
            p[b, c] = np.float32(np.exp(score[b, c] - score[b, parent[b, c]]))
    return p


def _phi(score, count):
    return np.array([np.exp(score[b, 1:int(count[b])]).sum() for b in range(score.shape[0])])


def _check_identity(res, trials, seed):
    p = _p_child(res.tok, res.parent, res.score, res.count)
    D = int(res.depth.max())
    h = accept_sim(res.parent, res.count, p, trials, seed, max_depth=D + 1)
    lens = np.arange(h.shape[1])
    mean = (h * lens).sum(1) / trials
    var = (h * lens ** 2).sum(1) / trials - mean ** 2
    phi = _phi(res.score, res.count)
    assert (np.abs(mean - phi) <= 4 * np.sqrt(var / trials) + 1e-9).all(), (mean, phi)


def test_identity_on_pctree_trees():
    rng = np.random.default_rng(1)
    V, D, r = 12, 4, 3
    L = rng.normal(0, 1.5, (2, D, V))
    E, W = rng.normal(0, 0.7, (V, r)), rng.normal(0, 0.7, (r, V))
    res = oracle.pct_tree_build(L, np.array([0, 5]), E, W, k=3, beam=6, n_nodes=14)
    _check_identity(res, trials=20000, seed=42)


def test_identity_on_caddtree_trees():
    rng = np.random.default_rng(2)
    L = rng.normal(0, 1.0, (2, 4, 10))
    L[:, :, 3] += 3.0
    res = oracle.cadd_tree_grow(L, np.array([1, 2]), np.array([0, 0]), 12, C_d=1.0, a=1.0,
                                b=0.0, c=0.0, e=0.0)
    _check_identity(res, trials=20000, seed=7)


def test_planted_mistake_breaks_the_identity():
    """Walking into a child with the parent's own probability (a wrong index)
    shifts the mean far outside the bound: the identity test is sensitive."""
    rng = np.random.default_rng(1)
    V, D, r = 12, 4, 3
    L = rng.normal(0, 1.5, (1, D, V))
    E, W = rng.normal(0, 0.7, (V, r)), rng.normal(0, 0.7, (r, V))
    res = oracle.pct_tree_build(L, np.array([0]), E, W, k=3, beam=6, n_nodes=14)
    p = _p_child(res.tok, res.parent, res.score, res.count)
    wrong = np.roll(p, 1, axis=1)
    h = accept_sim(res.parent, res.count, wrong, 20000, 5, max_depth=D + 1)
    mean = (h * np.arange(h.shape[1])).sum(1) / 20000
    assert abs(mean[0] - _phi(res.score, res.count)[0]) > 0.02
