"""B200-native (sm_100a) per-round hot path of tree-based speculative decoding.

* ``pct_tree_build``     -- PCTree: parent-conditioned drafting tree (batched
  Markov scoring on tcgen05 tensor cores, log-softmax, local top-k, beam,
  global top-N).
* ``cadd_tree_grow``     -- CaDDTree: cost-aware best-first tree with a greedy
  stop on (1 + Phi) / (C_d + C_v(n; l)).
* ``tree_ancestor_mask`` -- self-plus-ancestor bitmask for tree attention.
* ``tree_verify_accept`` -- greedy verification: argmax per node, accept walk,
  correction token.
* ``pct_score_parents``  -- one depth of PCTree's batched parent scoring.
* ``ddtree_grow`` and ``budget`` -- the fixed-budget best-first tree (CaDDTree's
  growth with the stop disabled) and the host-side sweep of fixed budgets
  against CaDDTree's adaptive size.
* ``tau`` -- Monte Carlo acceptance length of a round's trees against a synthetic
  target (marginal or parent-conditioned), host side.
* ``costfit`` -- non-negative (convex, non-decreasing) fit of the verification
  cost C_v(n; l) = a + b l + c n + e n^2 to latency samples, host side.

All compute runs in ``libpctree.so`` (CUDA C++ behind a C ABI, declared in
``include/pctree.h``); this package only marshals torch tensors to it.
"""
from ._lib import (  # noqa: F401
    BuildDesc, CaddDesc, PctError, TreeOut, VerifyOut, LIB_PATH, EXPORTED,
    PCT_OK, PCT_EINVAL, PCT_EWORKSPACE, PCT_ECUDA, PCT_EDEVICE, PCT_ETIMEOUT, PCT_EUNSUPPORTED,
    PCT_F32, PCT_BF16, DEV_BAD_PARENT, DEV_BAD_TOKEN, DEV_BAD_COUNT, DEV_DEPTH_OVERFLOW,
    DEV_BAD_COST, DEV_TIMEOUT,
    lib, build_desc, cadd_desc, pct_tree_build_workspace, pct_tree_build, pct_score_parents,
    cadd_tree_grow, tree_ancestor_mask, tree_verify_accept, trace_enable, trace_reset,
    trace_read, version,
)
from . import budget  # noqa: F401,E402
from .budget import ddtree_grow  # noqa: F401,E402
from . import tau  # noqa: F401,E402
from . import costfit  # noqa: F401,E402
