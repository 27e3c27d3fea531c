"""PCTree oracle: the parent-conditioned drafting tree, step by step (test infrastructure only).

Source: PCTree article (qiita), section on the chain draft's weakness and the
tree built in its place; DSpark's semi-autoregressive block is introduced in the
section before it. What the article fixes, in its notation:

* the DSpark chain picks, position by position, the best token of
  z_d = L_d + Markov(y_{d-1});
* PCTree instead scores every frontier parent p separately,
  z_d(p) = L_d + Markov(p), all parents in one batched Markov call;
* each parent keeps its local top-k children;
* candidates are ranked by the path log-probability s(c) = sum log pi(v|u);
* each depth is pruned to the best few ("top-k pruning at every depth",
  called the beam here), and a final global top-N keeps the tree inside the
  verification budget.

Readings taken where the article leaves a step open (all listed in the design
notes of this repository):

* the block has an anchor (depth 0, the root, a known token) and D = B - 1
  drafted depths; L has D rows, row d-1 serving depth d;
* one Markov head serves every depth and conditions depth 1 on the anchor;
* pi(.|u) = softmax over the vocabulary of z_d(u); s(root) = 0;
* per depth: every frontier parent contributes its k best children; the best
  ``beam`` candidates (by s) form the next frontier; after depth D the global
  top-(N-1) by s over the union of all kept nodes, plus the root, is the tree;
* total order everywhere: higher s first, then lower depth, then the
  lexicographically smaller token path (for siblings: the lower token id);
* output in canonical BFS order: root at 0, then by depth, then by (parent
  index, token); parent[0] = -1; slots at or past ``count`` hold tok = -1,
  parent = -1, depth = -1, score = -inf.

Near ties. The GPU computes in fp32 and this oracle in float64, so two
competing scores closer than ``tol`` may be ordered differently. A request is
marked excluded when such a pair sits at a selection boundary that can change
the output: a local top-k cut, a beam cut, or the global top-N cut. Pairs whose
per-depth inputs (drafter logit, Markov value, row log-sum-exp) are identical
are exact ties resolved by the total order on both sides and are not excluded.
A local top-k or beam boundary whose better score lies more than ``2 tol``
below the global cut cannot change the output (every node it could add or drop
scores below every selected node, and so do all its descendants) and is not
counted.

Near ties resolved toward a given tree. When two candidates differ by less
than ``tol``, either may be kept: both orders are correct to the tolerance. With
``prefer`` (a set of token paths, e.g. the nodes of a tree built elsewhere)
every cut keeps its usual members except that a rejected candidate in
``prefer`` replaces a kept one that is not in ``prefer`` when their scores
differ by less than ``tol``. The result is the tree this algorithm builds when
its near ties fall the preferred way; a tree equal to it is therefore a valid
output of the algorithm. Without ``prefer`` nothing changes.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .numerics import row_log_softmax


@dataclass
class PCTreeResult:
    tok: np.ndarray        # [batch][N] int32
    parent: np.ndarray     # [batch][N] int32
    depth: np.ndarray      # [batch][N] int32
    score: np.ndarray      # [batch][N] float64
    count: np.ndarray      # [batch] int32
    excluded: np.ndarray   # [batch] bool, near tie at a boundary that matters
    frontier_sizes: list = field(default_factory=list)   # per request: |F_d|, d=1..D
    kept: list = field(default_factory=list)             # per request: nodes kept by all beams


class _Node:
    __slots__ = ("tok", "depth", "s", "path", "vals")

    def __init__(self, tok, depth, s, path, vals):
        self.tok, self.depth, self.s, self.path, self.vals = tok, depth, s, path, vals


def score_parents(L_d, parent_tok, E, W, k, extra=1):
    """One depth of batched parent scoring for one request.

    For every parent token p: z = L_d + E[p] . W (all parents in one matrix
    product), log pi = z - lse(z), and the k + extra best children in the
    order (z desc, token asc). Returns (z, markov, log_pi, lse, order) with
    order holding the first min(k + extra, V) token ids of each row.
    """
    toks = np.asarray(parent_tok, dtype=np.int64)
    markov = E[toks] @ W                                       # [|F|][V]
    Z = L_d[None, :] + markov                                  # z_d(p)
    logpi, lse = row_log_softmax(Z)
    # stable sort of -z keeps the lower token first among equal z
    order = np.argsort(-Z, axis=1, kind="stable")[:, : min(k + extra, Z.shape[1])]
    return Z, markov, logpi, lse, order


def _near_tie_keep(ranked, keep, score, preferred, tol):
    """The first ``keep`` of ``ranked`` (best first), except that each rejected
    item in ``preferred`` takes the place of the lowest-ranked kept item not in
    ``preferred`` whose score is within ``tol`` of its own."""
    kept, rest = list(ranked[:keep]), ranked[keep:]
    if not kept or preferred is None:
        return kept
    floor = score(kept[-1]) - tol
    for y in rest:
        if score(y) <= floor:
            break
        if not preferred(y):
            continue
        for j in range(len(kept) - 1, -1, -1):
            x = kept[j]
            if not preferred(x) and abs(score(x) - score(y)) < tol:
                kept[j] = y
                break
    return kept


def _build_one(L, anchor, E, W, k, beam, n_nodes, tol, prefer=None):
    D, V = L.shape
    root = _Node(int(anchor), 0, 0.0, (), ())
    frontier = [root]
    levels = []
    boundaries = []            # (better score, worse score, identical inputs?)
    kk = min(k, V)
    pref = None if prefer is None else (lambda c: c.path in prefer)
    for d in range(1, D + 1):
        # one batched Markov call for every frontier parent: E[tok(p)] . W
        Z, markov, logpi, lse, order = score_parents(L[d - 1], [p.tok for p in frontier], E, W, k,
                                                     extra=1 if prefer is None else 8)
        cands = []
        for i, p in enumerate(frontier):
            row = [_Node(int(v), d, p.s + logpi[i, v], p.path + (int(v),),
                         p.vals + ((L[d - 1][v], markov[i, v], lse[i]),)) for v in order[i]]
            cands.extend(_near_tie_keep(row, kk, lambda c: c.s, pref, tol))
            if kk < V:
                vi, vo = int(order[i, kk - 1]), int(order[i, kk])
                same = (L[d - 1][vi] == L[d - 1][vo]) and (markov[i, vi] == markov[i, vo])
                boundaries.append((p.s + logpi[i, vi], p.s + logpi[i, vo], same))
        cands.sort(key=lambda c: (-c.s, c.path))
        if len(cands) > beam:
            a, b = cands[beam - 1], cands[beam]
            boundaries.append((a.s, b.s, a.vals == b.vals))
        kept = sorted(_near_tie_keep(cands, beam, lambda c: c.s, pref, tol),
                      key=lambda c: c.path)                   # canonical order
        levels.append(kept)
        frontier = kept

    union = [n for lvl in levels for n in lvl]
    ranked = sorted(union, key=lambda c: (-c.s, c.depth, c.path))
    chosen = {id(c) for c in _near_tie_keep(ranked, n_nodes - 1, lambda c: c.s, pref, tol)}
    sel = [c for c in ranked if id(c) in chosen]
    excluded = False
    if len(ranked) > n_nodes - 1:
        s_cut = sel[-1].s if sel else np.inf
        if sel:
            a, b = sel[-1], ranked[n_nodes - 1]
            if abs(a.s - b.s) < tol and not (a.depth == b.depth and a.vals == b.vals):
                excluded = True
    else:
        s_cut = -np.inf
    for better, worse, same in boundaries:
        if better >= s_cut - 2 * tol and abs(better - worse) < tol and not same:
            excluded = True

    out = [root] + sorted(sel, key=lambda c: (c.depth, c.path))
    index = {n.path: i for i, n in enumerate(out)}
    return out, index, excluded, [len(l) for l in levels], union


def pct_tree_build(L, anchor, E, W, k: int, beam: int, n_nodes: int,
                   tol: float = 1e-4, prefer=None) -> PCTreeResult:
    """PCTree over a batch of independent requests.

    L: float64 [batch][D][V] drafter logits (decoded); anchor: int [batch];
    E: float64 [V][r]; W: float64 [r][V]. Returns the node tables in canonical
    BFS order with float64 scores. ``prefer``: None, or one set of token paths
    per request (tuples of tokens below the root) toward which near ties are
    resolved (module docstring).
    """
    L = np.asarray(L, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    batch = L.shape[0]
    tok = np.full((batch, n_nodes), -1, np.int32)
    par = np.full((batch, n_nodes), -1, np.int32)
    dep = np.full((batch, n_nodes), -1, np.int32)
    score = np.full((batch, n_nodes), -np.inf, np.float64)
    count = np.zeros(batch, np.int32)
    excl = np.zeros(batch, bool)
    sizes, kept = [], []
    for b in range(batch):
        out, index, ex, fs, union = _build_one(L[b], anchor[b], E, W, k, beam, n_nodes, tol,
                                               None if prefer is None else prefer[b])
        for i, n in enumerate(out):
            tok[b, i] = n.tok
            dep[b, i] = n.depth
            score[b, i] = n.s
            par[b, i] = -1 if n.depth == 0 else index[n.path[:-1]]
        count[b] = len(out)
        excl[b] = ex
        sizes.append(fs)
        kept.append(union)
    return PCTreeResult(tok, par, dep, score, count, excl, sizes, kept)
