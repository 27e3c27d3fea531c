"""CPU oracle for the draft-tree hot path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference legs of ``bench.py`` may import, call or execute anything
in this package. The product library (``speculative_decoding_draft_07_b200``)
never does, and this package never imports the product library: the two share
no code. Inputs come from ``workloads`` (seeded generators only).

Everything here is a plain, slow, float64 restatement of what the three source
pages define, written step by step in their order and notation:

* ``pctree.pct_tree_build``   -- Parent-Conditioned Drafting Tree (PCTree
  article on qiita, section on the chain draft's weakness and the tree that
  replaces it): per-parent scores z_d(p) = L_d + Markov(p), log-softmax over
  the vocabulary, local top-k per parent, path score s(c) = sum log pi(v|u),
  per-depth pruning to a beam, global top-N.
* ``caddtree.cadd_tree_grow`` -- Cost-Aware Diffusion Draft Trees (gist.science
  summary, technical summary, "Method: CaDDTree"): best-first growth by prefix
  probability, greedy stop at the first non-positive marginal gain of
  (1 + Phi(T)) / (C_d + C_v(n; l)).
* ``verify.tree_verify_accept`` -- DSpark explainer (xiaohu-jiedu), section on
  one round from drafting to confirmation: greedy argmax per node, accept the
  longest matching root path, append the target's own token.
* ``verify.tree_ancestor_mask`` -- the self-plus-ancestors mask used for tree
  attention in the verification forward.
* ``costfit.cost_fit`` -- the non-negative least-squares fit of the
  verification cost C_v(n; l) = a + b l + c n + e n^2 to latency samples
  (CaDDTree summary, "Method": convex, non-decreasing cost profiled offline),
  by exhaustive search over the 16 free sets.

Parity status of each function (what pins it, other than itself, is in
``tests/test_oracle_*.py``):

* ``pct_tree_build``: pinned by brute-force enumeration of every path (k = V,
  unbounded beam), by the pruned tree defined by predicates over every path
  for finite k and beam (eligible = child of a kept path among its parent's k
  best; kept = the beam best eligible paths of a depth; V <= 5, D <= 4), by the
  DSpark greedy chain (k = 1, N = B), by agreement with the best-first tree
  when the Markov term is zero, and by a hand-derived finite beam example.
* ``cadd_tree_grow``: pinned by brute force (the top prefix-probability nodes
  for every n), by an exhaustive scan of the throughput objective over n, by a
  closed form on uniform marginals, and by Monte Carlo acceptance.
* ``tree_verify_accept``: pinned by the pages' worked round (4 accepted drafts
  plus 1 correction) and by planted paths.
* ``cost_fit``: pinned by SciPy's NNLS on random problems, by the KKT
  conditions and by exact recovery of noiseless convex costs.
* ``tree_ancestor_mask``: pinned by an independent transitive closure of the
  parent relation.
* ``row_topk``: each row's k largest logits (value descending, ties to the
  lower token id), the order best-first growth takes a position's tokens in;
  pinned by a brute-force pairwise count of the tokens that precede each token
  and by the children the best-first tree takes at depth 1.
* ``accept_sim``: Monte Carlo walks of greedy verification on a tree (the
  acceptance length tau); pinned by the generator's published known answers,
  by walks worked out by hand, and by the identity E[accepted] = Phi(T) when the
  target is the drafter itself.
"""
from .numerics import decode_bf16, to_f64, row_log_softmax
from .pctree import pct_tree_build, PCTreeResult, score_parents
from .caddtree import cadd_tree_grow, CaddResult, cadd_cost, row_topk
from .verify import tree_verify_accept, tree_ancestor_mask, VerifyResult
from .accept_sim import accept_sim, philox4x32_10, uniform24
from .costfit import cost_fit

__all__ = [
    "decode_bf16", "to_f64", "row_log_softmax",
    "pct_tree_build", "PCTreeResult", "score_parents",
    "cadd_tree_grow", "CaddResult", "cadd_cost",
    "tree_verify_accept", "tree_ancestor_mask", "VerifyResult",
    "accept_sim", "philox4x32_10", "uniform24",
    "cost_fit",
]
