"""DDTree fixed-budget trees and the fixed-versus-adaptive budget sweep (host side).

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
summary), technical summary, "Method: CaDDTree":
- A round costs C(n; l) = C_d + a + b l + c n + e n^2 and yields 1 + Phi_n tokens
  in expectation.
- For a fixed size n the best tree is the best-first tree of the n - 1 nodes of
  highest prefix probability, which is DDTree's tree with budget n.
- CaDDTree stops growing at the first size whose successor does not raise
  (1 + Phi_n) / C(n).

The best-first order does not depend on the cost. So one fixed-budget tree per
round gives Phi_n for every n up to its size, and from it, on the host, the
objective of every fixed budget and the adaptive size under any cost. The sweep
compares the best single fixed budget over a set of rounds with the per-round
adaptive size, optionally with the planner misestimating the cost.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np
import torch

from ._lib import TreeOut, cadd_tree_grow

__all__ = ["ddtree_grow", "phi_curve", "round_cost", "objective_curve", "adaptive_size",
           "budget_sweep"]


def ddtree_grow(L: torch.Tensor, anchor: torch.Tensor, n: int, out: Optional[TreeOut] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> TreeOut:
    """Best-first tree of n nodes per request (root included): the CaDDTree growth
    with the stop disabled. With c = e = 0, dC(n) = 0, so no node of positive
    probability has a non-positive gain. A request stops short of n only when its
    candidates run out. Node tables [batch][n], scores are log prefix probabilities."""
    ctx = torch.zeros(L.shape[0], dtype=torch.int64, device=L.device)
    return cadd_tree_grow(L, anchor, ctx, n, 1.0, 0.0, 0.0, 0.0, 0.0, out=out,
                          workspace=workspace, stream=stream)


def phi_curve(score: np.ndarray, count: int) -> np.ndarray:
    """Phi_n for n = 1..count (entry n - 1) of one best-first tree.

    score holds the tree's log prefix probabilities, root first, in any node
    order. Best-first growth adds nodes in decreasing prefix probability, so
    Phi_n is the running sum of the n - 1 largest, accumulated largest first.
    """
    s = np.sort(np.asarray(score[1:count], dtype=np.float64))[::-1]
    phi = np.zeros(max(int(count), 1), dtype=np.float64)
    acc = 0.0
    for i, x in enumerate(s):
        acc += math.exp(float(x))
        phi[i + 1] = acc
    return phi


def round_cost(n, ell, C_d: float, a: float, b: float, c: float, e: float):
    """C(n; l) = C_d + C_v(n; l), C_v = a + b l + c n + e n^2 (n counts the root)."""
    return C_d + a + b * ell + c * n + e * n * n


def objective_curve(phi: np.ndarray, ell: float, C_d: float, a: float, b: float, c: float,
                    e: float) -> np.ndarray:
    """f(n) = (1 + Phi_n) / C(n; l) for n = 1..len(phi) (entry n - 1)."""
    n = np.arange(1, len(phi) + 1, dtype=np.float64)
    return (1.0 + phi) / round_cost(n, ell, C_d, a, b, c, e)


def adaptive_size(phi: np.ndarray, ell: float, C_d: float, a: float, b: float, c: float,
                  e: float, n_max: Optional[int] = None) -> int:
    """CaDDTree's greedy size: starting from the root alone, the next node is added
    while (1 + Phi_{n+1}) / C(n + 1) > (1 + Phi_n) / C(n). Growth stops at n_max or
    when the tree's candidates (the end of phi) run out."""
    top = len(phi) if n_max is None else min(int(n_max), len(phi))
    n = 1
    while n < top:
        if (1.0 + phi[n]) / round_cost(n + 1, ell, C_d, a, b, c, e) <= \
                (1.0 + phi[n - 1]) / round_cost(n, ell, C_d, a, b, c, e):
            break
        n += 1
    return n


def budget_sweep(phis: Sequence[np.ndarray], ells: Sequence[float], cost: Sequence[float],
                 plan_cost: Optional[Sequence[float]] = None,
                 sizes: Optional[Sequence[int]] = None) -> dict:
    """Tokens per unit cost over a set of rounds: every fixed budget, and the adaptive size.

    phis: Phi curves, one per round; ells: the context length of each round.
    cost: the true (C_d, a, b, c, e). plan_cost: the cost the adaptive planner
    uses to choose its sizes (default: the true one); the rates always use the
    true cost. A round whose tree is smaller than a budget uses its whole tree.
    The rate of a policy is the sum over rounds of 1 + Phi divided by the sum of
    the rounds' costs.
    """
    plan = tuple(cost if plan_cost is None else plan_cost)
    longest = max(len(p) for p in phis)
    sizes = list(range(1, longest + 1)) if sizes is None else [int(n) for n in sizes]

    def rate(chosen):
        tok = sum(1.0 + p[m - 1] for p, m in zip(phis, chosen))
        cst = sum(round_cost(m, ell, *cost) for m, ell in zip(chosen, ells))
        return tok / cst

    fixed = {n: rate([min(n, len(p)) for p in phis]) for n in sizes}
    best_n = max(fixed, key=lambda n: (fixed[n], -n))
    adaptive = np.array([adaptive_size(p, ell, *plan) for p, ell in zip(phis, ells)])
    adaptive_rate = rate(list(adaptive))
    return {"fixed": fixed, "best_fixed_n": best_n, "best_fixed_rate": fixed[best_n],
            "adaptive_sizes": adaptive, "adaptive_size_mean": float(adaptive.mean()),
            "adaptive_size_std": float(adaptive.std()), "adaptive_rate": adaptive_rate,
            "gain": adaptive_rate / fixed[best_n]}
