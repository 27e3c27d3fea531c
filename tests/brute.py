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
