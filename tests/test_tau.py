"""The acceptance simulator (host side) against identities that fix its mean.

DSpark explainer (xiaohu-jiedu), one round: the walk accepts drafts while the
target's token matches a child, and the first miss ends it. When the target
draws every position from the drafter's own distribution, the probability that
the walk passes a node is that node's prefix probability. So the expected
number of accepted drafts is Phi(T) = sum over non-root nodes of exp(score)
("Cost-Aware Diffusion Draft Trees for Speculative Decoding", gist.science
summary, "Method: CaDDTree"; PCTree article, qiita, for the parent-conditioned
head, where the score is the path's log-probability under that head).
"""
import numpy as np

import oracle
from speculative_decoding_draft_07_b200 import tau


def _mean_within(x, want, sigmas=4.0):
    se = x.std(ddof=1) / np.sqrt(x.size)
    assert abs(x.mean() - want) <= sigmas * se + 1e-12, (x.mean(), want, se)


def test_marginal_target_mean_is_phi_on_caddtree_trees():
    rng = np.random.default_rng(31)
    batch, D, V = 3, 6, 50
    L = rng.normal(0, 1.5, size=(batch, D, V))
    L[np.arange(batch)[:, None], np.arange(D)[None, :], rng.integers(0, V, (batch, D))] += 3.0
    anchor = rng.integers(0, V, batch)
    t = oracle.cadd_tree_grow(L, anchor, np.full(batch, 2000), 48, 1.0, 2.0, 1e-4, 5e-3, 1e-5)
    for b in range(batch):
        n = int(t.count[b])
        acc = tau.simulate_accept(t.tok[b], t.parent[b], n, V, 40000, rng, marginal_logits=L[b])
        phi = tau.expected_accept_marginal(t.score[b], n)
        assert abs(phi - t.phi[b]) < 1e-9
        _mean_within(acc.astype(np.float64), phi)


def test_conditioned_target_mean_is_phi_on_pctree_trees():
    rng = np.random.default_rng(32)
    D, V, r = 4, 40, 3
    L = rng.normal(0, 1.5, size=(1, D, V))
    E = rng.normal(0, 0.8, size=(V, r))
    W = rng.normal(0, 0.8, size=(r, V))
    t = oracle.pct_tree_build(L, [5], E, W, k=4, beam=6, n_nodes=20)
    n = int(t.count[0])
    cond = lambda d, u: L[0, d - 1] + E[u] @ W
    acc = tau.simulate_accept(t.tok[0], t.parent[0], n, V, 40000, rng, conditioned_logits=cond)
    _mean_within(acc.astype(np.float64), tau.expected_accept_marginal(t.score[0], n))


def test_deterministic_target_walks_exactly():
    """A chain 7 -> 3 -> 1 -> 4 plus a side branch; the target's argmax (one-hot
    logits) follows the chain for two steps and then names a token with no child."""
    tok = np.array([7, 3, 9, 1, 4])
    parent = np.array([-1, 0, 0, 1, 3])
    V = 12
    M = np.full((4, V), -1e4)
    M[0, 3] = M[1, 1] = 0.0      # depth 1 -> node 1, depth 2 -> node 3
    M[2, 5] = 0.0                # depth 3: token 5, node 3 has only child 4 -> miss
    M[3, 0] = 0.0
    acc = tau.simulate_accept(tok, parent, 5, V, 100, np.random.default_rng(0), marginal_logits=M)
    assert (acc == 2).all()
    M[2, 4] = 0.0
    M[2, 5] = -1e4
    acc = tau.simulate_accept(tok, parent, 5, V, 100, np.random.default_rng(0), marginal_logits=M)
    assert (acc == 3).all()       # the whole chain; depth 4 has no node


def test_root_only_tree_accepts_nothing():
    acc = tau.simulate_accept(np.array([2]), np.array([-1]), 1, 8, 50, np.random.default_rng(1),
                              marginal_logits=np.zeros((3, 8)))
    assert (acc == 0).all()


def test_mean_tau_on_a_batch_is_one_plus_phi():
    rng = np.random.default_rng(33)
    batch, D, V = 2, 5, 30
    L = rng.normal(0, 1.0, size=(batch, D, V))
    L[:, :, 4] += 3.0
    t = oracle.cadd_tree_grow(L, [1, 2], [100, 100], 32, 1.0, 2.0, 1e-4, 5e-3, 1e-5)
    m = tau.mean_tau(t, V, 40000, rng, marginal_logits=L)
    for b in range(batch):
        assert abs(m[b] - (1.0 + t.phi[b])) < 0.05
