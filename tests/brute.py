"""Exhaustive enumerations used to pin the oracle on tiny inputs.

Written independently of ``oracle/``: plain Python loops and ``math`` only, no
numpy routines shared with it. Every path of depth <= D over a vocabulary of V
tokens is listed and scored from its definition.
"""
from __future__ import annotations

import itertools
import math


def _logsumexp(xs):
    m = max(xs)
    return m + math.log(sum(math.exp(x - m) for x in xs))


def conditioned_path_scores(L, anchor, E, W):
    """PCTree's path score for every path, from the definition.

    z_j(u)[v] = L[j-1][v] + sum_i E[u][i] * W[i][v]; the token before depth 1
    is the anchor; s(path) = sum_j (z_j(y_{j-1})[y_j] - lse z_j(y_{j-1})).
    Returns {path tuple: score}.
    """
    D, V = len(L), len(L[0])
    r = len(W)

    def z_row(j, u):
        return [L[j - 1][v] + sum(E[u][i] * W[i][v] for i in range(r)) for v in range(V)]

    cache = {}
    out = {}
    for d in range(1, D + 1):
        for path in itertools.product(range(V), repeat=d):
            s = 0.0
            prev = anchor
            for j, y in enumerate(path, start=1):
                key = (j, prev)
                if key not in cache:
                    row = z_row(j, prev)
                    cache[key] = (row, _logsumexp(row))
                row, lse = cache[key]
                s += row[y] - lse
                prev = y
            out[path] = s
    return out


def marginal_path_scores(L):
    """Prefix log-probability of every path under per-position marginals.

    s(path) = sum_j (L[j-1][y_j] - lse L[j-1]). Returns {path tuple: score}.
    """
    D, V = len(L), len(L[0])
    lse = [_logsumexp(L[j]) for j in range(D)]
    out = {}
    for d in range(1, D + 1):
        for path in itertools.product(range(V), repeat=d):
            out[path] = sum(L[j][y] - lse[j] for j, y in enumerate(path))
    return out


def ranked(scores):
    """Paths in the total order: higher score, lower depth, smaller token path."""
    return sorted(scores, key=lambda p: (-scores[p], len(p), p))


def canonical_table(anchor, paths, scores):
    """Root + paths in canonical BFS order: (tok, parent, depth, score) lists."""
    order = [()] + sorted(paths, key=lambda p: (len(p), p))
    index = {p: i for i, p in enumerate(order)}
    tok = [anchor] + [p[-1] for p in order[1:]]
    parent = [-1] + [index[p[:-1]] for p in order[1:]]
    depth = [len(p) for p in order]
    score = [0.0] + [scores[p] for p in order[1:]]
    return tok, parent, depth, score


def pruned_selection(scores, z_of, V, D, k, beam, N):
    """PCTree with finite k and beam, from predicates over every path.

    A path p of depth d is eligible when its parent p[:-1] is kept and its last
    token is among the k best children of that parent by z (ties: lower token
    id); kept at depth d are the `beam` best eligible paths of that depth in
    the total order (score desc, then the smaller token path). The tree is the
    root plus the N-1 best kept paths of all depths in the total order (score
    desc, lower depth, smaller token path). z_of(parent_path, token) gives z.
    Returns (selected paths, per-depth kept counts).
    """
    kept = {(): True}
    all_kept, sizes = [], []
    for d in range(1, D + 1):
        eligible = []
        for p in itertools.product(range(V), repeat=d):
            par = p[:-1]
            if par not in kept:
                continue
            zs = [(z_of(par, v), -v) for v in range(V)]
            mine = zs[p[-1]]
            better = sum(1 for t in zs if t > mine)
            if better < k:
                eligible.append(p)
        eligible.sort(key=lambda p: (-scores[p], p))
        layer = eligible[:beam]
        for p in layer:
            kept[p] = True
        all_kept.extend(layer)
        sizes.append(len(layer))
    sel = sorted(all_kept, key=lambda p: (-scores[p], len(p), p))[: max(N - 1, 0)]
    return sel, sizes


def conditioned_z(L, anchor, E, W):
    """z_of(parent_path, v) for the conditioned head: L[d-1][v] + Markov(last token)[v]."""
    r = len(W)

    def z_of(par, v):
        d = len(par) + 1
        u = par[-1] if par else anchor
        return L[d - 1][v] + sum(E[u][i] * W[i][v] for i in range(r))
    return z_of
