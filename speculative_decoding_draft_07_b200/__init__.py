"""B200-native (sm_100a) per-round hot path of tree-based speculative decoding.

The hot path, all of it in ``libpctree.so`` (CUDA C++ for sm_100a behind the
C ABI declared in ``include/pctree.h``); the functions here only check shapes,
allocate outputs and pass pointers (``_lib.py``), and raise if the library is
missing:

* ``pct_tree_build``     -- PCTree: parent-conditioned drafting tree (batched
  Markov scoring on tcgen05 tensor cores, log-softmax, local top-k, beam,
  global top-N). With ``seeds=`` (and optionally ``Wt=markov_transpose(W)``)
  the gates of its top-k start from given columns instead of a pass over L.
* ``cadd_tree_grow``     -- CaDDTree: cost-aware best-first tree with a greedy
  stop on (1 + Phi) / (C_d + C_v(n; l)). With ``top_tok=`` its row pass also
  writes each row's top-k tokens, which can seed the PCTree on the same L.
* ``tree_ancestor_mask`` -- self-plus-ancestor bitmask for tree attention.
* ``tree_verify_accept`` -- greedy verification: argmax per node, accept walk,
  correction token.
* ``tree_verify_walk``   -- the same acceptance reading only the rows the walk
  reaches.
* ``tree_accept_sim``    -- Monte Carlo acceptance length (tau) of a batch of
  trees against a synthetic target given per node.
* ``pct_score_parents``  -- one depth of PCTree's batched parent scoring.
* ``cadd_cost_fit``      -- the non-negative fit of CaDDTree's verification cost
  C_v(n; l) = a + b l + c n + e n^2 to latency samples, on the device.
* ``budget.ddtree_grow`` -- the fixed-budget best-first tree (CaDDTree's growth
  with the stop disabled), a call of ``cadd_tree_grow``.

Host-side tools around the hot path (numpy on the host, not part of it and not
marshalling): ``budget`` (Phi curves, the greedy size and the sweep of fixed
budgets against the adaptive size, evaluated from the library's trees),
``tau`` (Monte Carlo acceptance length of a round's trees against a synthetic
target) and ``costfit`` (the same non-negative fit as ``cadd_cost_fit``, by
the Lawson-Hanson method on the host).
"""
from ._lib import (  # noqa: F401
    BuildDesc, CaddDesc, PctError, TreeOut, VerifyOut, LIB_PATH, EXPORTED,
    PCT_OK, PCT_EINVAL, PCT_EWORKSPACE, PCT_ECUDA, PCT_EDEVICE, PCT_ETIMEOUT, PCT_EUNSUPPORTED,
    PCT_F32, PCT_BF16, DEV_BAD_PARENT, DEV_BAD_TOKEN, DEV_BAD_COUNT, DEV_DEPTH_OVERFLOW,
    DEV_BAD_COST, DEV_TIMEOUT,
    lib, build_desc, cadd_desc, pct_tree_build_workspace, pct_tree_build, pct_score_parents,
    cadd_tree_grow, tree_ancestor_mask, tree_verify_accept, tree_verify_walk, tree_accept_sim,
    cadd_cost_fit, markov_transpose, trace_enable, trace_reset,
    trace_read, version,
)
from . import budget  # noqa: F401,E402
from .budget import ddtree_grow  # noqa: F401,E402
from . import tau  # noqa: F401,E402
from . import costfit  # noqa: F401,E402
