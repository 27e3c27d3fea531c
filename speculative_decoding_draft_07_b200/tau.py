"""Synthetic acceptance-length (tau) simulation of a round (host side).

The acceptance rule follows the DSpark explainer (xiaohu-jiedu), one round
from drafting to confirmation: drafts are checked from the head, consecutive
matches are kept, the first miss ends the round, and the target adds one token
of its own. On a tree, the walk starts at the root. At each node it draws the
target's token for the next position and moves to the child carrying that
token, if there is one. tau = accepted drafts + 1.

The target here is synthetic: per position, a distribution given by logits.
Either one row per depth (marginal targets, as CaDDTree's drafter assumes),
or one row per (depth, token of the current node) through a callback
(parent-conditioned targets, as PCTree's Markov head assumes). When the target
equals the drafter's own distribution, the expected number of accepted drafts
is Phi(T), the sum of the prefix probabilities of the tree's non-root nodes
("Cost-Aware Diffusion Draft Trees for Speculative Decoding", gist.science
summary, "Method: CaDDTree"). The tests pin the simulation to that identity.
"""
from __future__ import annotations

from typing import Callable, Optional

import numpy as np

__all__ = ["simulate_accept", "expected_accept_marginal", "mean_tau"]


def _children_index(tok: np.ndarray, parent: np.ndarray, count: int, V: int):
    """Sorted keys parent * V + token of the tree's edges, and the child per key."""
    c = np.arange(1, count)
    keys = parent[1:count].astype(np.int64) * V + tok[1:count].astype(np.int64)
    order = np.argsort(keys, kind="stable")
    return keys[order], c[order]


def _softmax_cdf(logits: np.ndarray) -> np.ndarray:
    z = np.asarray(logits, dtype=np.float64)
    z = z - z.max()
    p = np.exp(z)
    cdf = np.cumsum(p)
    return cdf / cdf[-1]


def simulate_accept(tok: np.ndarray, parent: np.ndarray, count: int, V: int, draws: int,
                    rng: np.random.Generator, marginal_logits: Optional[np.ndarray] = None,
                    conditioned_logits: Optional[Callable[[int, int], np.ndarray]] = None,
                    max_depth: Optional[int] = None) -> np.ndarray:
    """Accepted-draft counts of `draws` independent rounds on one tree.

    tok, parent: the tree's node tables (root at 0, parent[i] < i); count: its size.
    Exactly one target model:
      marginal_logits [D][V]: the target's token at depth d is drawn from
        softmax(marginal_logits[d - 1]), whatever came before;
      conditioned_logits(d, u) -> [V]: the target's logits at depth d given the
        token u of the node the walk stands on (depth 1: u is the root's token).
    Returns an int array [draws]; tau of each round is the value + 1.
    """
    if (marginal_logits is None) == (conditioned_logits is None):
        raise ValueError("give exactly one of marginal_logits and conditioned_logits")
    keys, child = _children_index(np.asarray(tok), np.asarray(parent), int(count), V)
    # no walk goes deeper than the tree's deepest node (a draw below it always
    # misses), nor past the last row of marginal targets
    par = np.asarray(parent)
    node_depth = np.zeros(max(int(count), 1), dtype=np.int64)
    for i in range(1, int(count)):
        node_depth[i] = node_depth[par[i]] + 1
    depth_cap = int(node_depth.max())
    if max_depth is not None:
        depth_cap = min(depth_cap, int(max_depth))
    if marginal_logits is not None:
        depth_cap = min(depth_cap, marginal_logits.shape[0])
    node = np.zeros(draws, dtype=np.int64)          # every round starts at the root
    alive = np.ones(draws, dtype=bool)
    accepted = np.zeros(draws, dtype=np.int64)
    cdf_cache = {}
    for d in range(1, depth_cap + 1):
        idx = np.nonzero(alive)[0]
        if idx.size == 0 or keys.size == 0:
            break
        cur = node[idx]
        y = np.empty(idx.size, dtype=np.int64)
        if marginal_logits is not None:
            if ("m", d) not in cdf_cache:
                cdf_cache[("m", d)] = _softmax_cdf(marginal_logits[d - 1])
            y[:] = np.searchsorted(cdf_cache[("m", d)], rng.random(idx.size), side="right")
        else:
            toks = np.asarray(tok)[cur]
            for t in np.unique(toks):
                sel = toks == t
                key = ("c", d, int(t))
                if key not in cdf_cache:
                    cdf_cache[key] = _softmax_cdf(conditioned_logits(d, int(t)))
                y[sel] = np.searchsorted(cdf_cache[key], rng.random(int(sel.sum())), side="right")
        y = np.minimum(y, V - 1)
        want = cur * V + y
        pos = np.minimum(np.searchsorted(keys, want), keys.size - 1)
        hit = keys[pos] == want
        node[idx[hit]] = child[pos[hit]]
        accepted[idx[hit]] += 1
        alive[idx[~hit]] = False
    return accepted


def expected_accept_marginal(score: np.ndarray, count: int) -> float:
    """Phi(T) from a tree's log prefix probabilities (root first): the expected
    number of accepted drafts when the target draws each position from the
    drafter's own marginals."""
    return float(np.exp(np.asarray(score[1:count], dtype=np.float64)).sum())


def mean_tau(tree, V: int, draws: int, rng: np.random.Generator,
             marginal_logits: Optional[np.ndarray] = None,
             conditioned_logits: Optional[Callable[[int, int, int], np.ndarray]] = None) -> np.ndarray:
    """Mean tau (accepted drafts + 1) per request of a batch of trees.

    tree: node tables with tok, parent, count (torch tensors from the library or
    numpy arrays), [batch][N]. marginal_logits [batch][D][V], or
    conditioned_logits(b, d, u) -> [V] for request b."""
    def host(x):
        return x.detach().cpu().numpy() if hasattr(x, "detach") else np.asarray(x)
    tok, parent, count = host(tree.tok), host(tree.parent), host(tree.count)
    out = np.zeros(tok.shape[0])
    for b in range(tok.shape[0]):
        if marginal_logits is not None:
            acc = simulate_accept(tok[b], parent[b], int(count[b]), V, draws, rng,
                                  marginal_logits=np.asarray(marginal_logits[b], dtype=np.float64))
        else:
            acc = simulate_accept(tok[b], parent[b], int(count[b]), V, draws, rng,
                                  conditioned_logits=lambda d, u, b=b: conditioned_logits(b, d, u))
        out[b] = acc.mean() + 1.0
    return out


def drafter_child_probs(tree):
    """p(child) for a target equal to the drafter: exp(s(child) - s(parent)),
    0 at the root and past count (torch tensors on the tree's device). This is
    the input of the library's device simulation (``tree_accept_sim``)."""
    import torch
    par = tree.parent.to(torch.int64).clamp(min=0)
    p = torch.exp(tree.score - tree.score.gather(1, par))
    return torch.where(tree.parent >= 0, p, torch.zeros_like(p)).contiguous()


def mean_tau_device(tree, trials: int, seed: int, max_depth: int, p_child=None):
    """Mean tau (accepted drafts + 1) per request, walked on the GPU by
    ``tree_accept_sim`` (the drafter as the target unless p_child is given).
    Returns (mean tau [batch], histogram [batch][max_depth + 1]) as numpy."""
    from ._lib import tree_accept_sim
    p = drafter_child_probs(tree) if p_child is None else p_child
    hist, status = tree_accept_sim(tree.parent, tree.count, p, trials, seed, max_depth)
    h = hist.cpu().numpy().astype(np.float64)
    if (status.cpu().numpy() != 0).any():
        raise ValueError("tree_accept_sim flagged a malformed tree")
    lens = np.arange(h.shape[1])
    return (h * lens).sum(1) / np.maximum(h.sum(1), 1) + 1.0, h
