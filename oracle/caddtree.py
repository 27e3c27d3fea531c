"""CaDDTree oracle: cost-aware best-first draft tree (test infrastructure only).

Source: "Cost-Aware Diffusion Draft Trees for Speculative Decoding"
(gist.science summary), technical summary, "Method: CaDDTree":

* throughput objective: a round costs C(T; l) = C_d + C_v(|T|; l); the tree
  maximises (1 + Phi(T)) / C(T; l), where 1 + Phi(T) is the expected number of
  tokens the round yields;
* decomposition: for a fixed size n the best tree is the greedy best-first tree
  that takes the nodes of highest prefix probability (as in DDTree);
* unimodality and greedy stop: with a convex C_v the objective is unimodal in
  the size, so nodes are added one at a time and growth stops at the first
  non-positive marginal gain;
* the budget n* therefore adapts per round to the drafter's marginals and to
  the context length l through C_v.

Readings taken where the summary leaves a step open:

* the drafter gives per-position marginals q_d = softmax(L_d), d = 1..D, one
  forward for the whole block (block-diffusion drafter); a node's prefix
  probability is P(u) = prod_{j <= depth(u)} q_j(v_j), and s(u) = log P(u);
* Phi(T) = sum of P(u) over the non-root nodes of T (the expected number of
  accepted draft tokens when each position's target token is drawn from q_d);
* |T| counts the root; C_v(n; l) = a + b l + c n + e n^2 (the cost model of the
  benchmark configuration; convex when c, e >= 0);
* growth starts from T = {root}; at size n the best remaining candidate c (the
  best not-yet-added child of any tree node, same total order as PCTree:
  higher s, then lower depth, then the lexicographically smaller token path)
  is added unless f(n + 1) <= f(n), with f(n) = (1 + Phi_n) / C(n); growth also
  stops at n = n_max or when no candidate is left;
* output in canonical BFS order, scores s(u) = log P(u), count = n*, and Phi.

Near ties. A request is excluded when the last node added and the first
candidate not added differ by less than ``tol`` in s (unless their per-depth
logits are identical), or when the stop test at any step was within ``2 tol``
of flipping (|s - log((1 + Phi) dC(n) / C(n))| < 2 tol).

Near ties resolved toward a given tree. With ``prefer`` (per request, a set of
token paths and a node count, e.g. a tree built elsewhere) growth takes, at
each step, the best candidate in the set instead of the best candidate overall
when their scores differ by less than ``tol``, and a stop test within ``2 tol``
of flipping stops exactly when the tree has the given count. The result is the
tree this algorithm grows when its near ties fall the preferred way. Without
``prefer`` nothing changes.
"""
from __future__ import annotations

import heapq
import math
from dataclasses import dataclass, field

import numpy as np

from .numerics import row_log_softmax


def cadd_cost(n, ell, C_d, a, b, c, e):
    """Round cost C(n; l) = C_d + C_v(n; l), C_v = a + b l + c n + e n^2."""
    return C_d + a + b * ell + c * n + e * n * n


@dataclass
class CaddResult:
    tok: np.ndarray        # [batch][n_max] int32
    parent: np.ndarray
    depth: np.ndarray
    score: np.ndarray      # float64 log prefix probability
    count: np.ndarray      # n*
    phi: np.ndarray        # float64
    excluded: np.ndarray   # bool
    stop_reason: list = field(default_factory=list)   # "gain", "n_max" or "exhausted"
    f_values: list = field(default_factory=list)      # f(1..n*) per request


def _grow_one(L, anchor, ell, n_max, C_d, a, b, c, e, tol, prefer=None):
    D, V = L.shape
    q, _ = row_log_softmax(L)                           # log q_d(v), [D][V]
    order = [np.argsort(-q[d], kind="stable") for d in range(D)]   # (q desc, v asc)

    def C(n):
        return cadd_cost(n, ell, C_d, a, b, c, e)

    # tree nodes: (tok, depth, s, path, vals); the heap holds candidates keyed by
    # the total order, with the parent's node index and the child's rank in its row
    nodes = [(int(anchor), 0, 0.0, (), ())]
    heap = []

    def push_child(parent_idx, rank):
        ptok, pdepth, ps, ppath, pvals = nodes[parent_idx]
        d = pdepth + 1
        if d > D or rank >= V:
            return
        v = int(order[d - 1][rank])
        s = ps + q[d - 1][v]
        heapq.heappush(heap, (-s, d, ppath + (v,), parent_idx, rank, pvals + (L[d - 1][v],)))

    push_child(0, 0)
    phi, n = 0.0, 1
    excluded = False
    fvals = [(1.0 + phi) / C(1)]
    last_s, last_vals, last_depth = None, None, None
    reason = "n_max"
    while n < n_max:
        if not heap:
            reason = "exhausted"
            break
        pick = 0
        if prefer is not None and heap[0][2] not in prefer[0]:
            # a preferred candidate within tol of the best takes its place
            best = -heap[0][0]
            near = [j for j, h in enumerate(heap) if h[2] in prefer[0] and -h[0] > best - tol]
            if near:
                pick = min(near, key=lambda j: heap[j][:3])
        negs, d, path, pidx, rank, vals = heap[pick]
        s = -negs
        p = math.exp(s)
        dC = C(n + 1) - C(n)
        flip = False
        if dC > 0:
            margin = s - math.log((1.0 + phi) * dC / C(n))
            if abs(margin) < 2 * tol:
                excluded = True
                flip = prefer is not None
        stop = (1.0 + phi + p) / C(n + 1) <= (1.0 + phi) / C(n)
        if flip:
            stop = n >= prefer[1]
        if stop:
            reason = "gain"
            break
        heap[pick] = heap[-1]
        heap.pop()
        heapq.heapify(heap)
        nodes.append((path[-1], d, s, path, vals))
        phi += p
        n += 1
        fvals.append((1.0 + phi) / C(n))
        last_s, last_vals, last_depth = s, vals, d
        push_child(pidx, rank + 1)          # next sibling
        push_child(len(nodes) - 1, 0)       # first child
    if last_s is not None and heap and reason in ("gain", "n_max"):
        negs, d, path, pidx, rank, vals = heap[0]
        if abs(last_s - (-negs)) < tol and not (d == last_depth and vals == last_vals):
            excluded = True

    out = [nodes[0]] + sorted(nodes[1:], key=lambda t: (t[1], t[3]))
    index = {t[3]: i for i, t in enumerate(out)}
    return out, index, phi, excluded, reason, fvals


def cadd_tree_grow(L, anchor, ctx_len, n_max: int, C_d: float, a: float, b: float,
                   c: float, e: float, tol: float = 1e-4, prefer=None) -> CaddResult:
    """CaDDTree over a batch of independent requests.

    L: float64 [batch][D][V] marginal logits; anchor: int [batch]; ctx_len: the
    context length l per request. Output arrays are [batch][n_max].
    ``prefer``: None, or per request a pair (set of token paths below the root,
    node count) toward which near ties are resolved (module docstring).
    """
    L = np.asarray(L, dtype=np.float64)
    batch = L.shape[0]
    tok = np.full((batch, n_max), -1, np.int32)
    par = np.full((batch, n_max), -1, np.int32)
    dep = np.full((batch, n_max), -1, np.int32)
    score = np.full((batch, n_max), -np.inf, np.float64)
    count = np.zeros(batch, np.int32)
    phi = np.zeros(batch, np.float64)
    excl = np.zeros(batch, bool)
    reasons, fv = [], []
    for r in range(batch):
        out, index, ph, ex, why, f = _grow_one(L[r], anchor[r], float(ctx_len[r]), n_max,
                                               C_d, a, b, c, e, tol,
                                               None if prefer is None else prefer[r])
        for i, (t, d, s, path, _) in enumerate(out):
            tok[r, i], dep[r, i], score[r, i] = t, d, s
            par[r, i] = -1 if d == 0 else index[path[:-1]]
        count[r], phi[r], excl[r] = len(out), ph, ex
        reasons.append(why)
        fv.append(f)
    return CaddResult(tok, par, dep, score, count, phi, excl, reasons, fv)


def row_topk(L, k: int):
    """The k largest logits of every row of L [..][V] as token ids, value
    descending, equal values to the lower token id; -1 past V.

    Best-first growth expands a position's tokens in this order (the children
    of a node at depth d are taken by decreasing q_d, i.e. by decreasing
    logit), so these are the first k children any node of depth d - 1 offers.
    Plain definition: a stable sort of the row by decreasing value.
    """
    L = np.asarray(L, dtype=np.float64)
    V = L.shape[-1]
    flat = L.reshape(-1, V)
    out = np.full((flat.shape[0], k), -1, np.int32)
    for i, row in enumerate(flat):
        order = np.argsort(-row, kind="stable")[:k]
        out[i, :len(order)] = order
    return out.reshape(L.shape[:-1] + (k,))

