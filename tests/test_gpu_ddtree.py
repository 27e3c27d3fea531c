"""GPU parity of the fixed-budget (DDTree) trees and of the budget sweep built on them.

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
summary), "Method: CaDDTree" and "Experiments": for a fixed size the best tree
is the best-first tree of highest prefix probability (DDTree with that budget);
CaDDTree's adaptive size is compared with the best fixed budget.

ddtree_grow is cadd_tree_grow with c = e = 0: the stop never fires, no token
of a row can be filtered out, and the library's exact selection of each row's
n_max - 1 best tokens runs over the whole vocabulary.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import compare_all, f64, host, oracle_map
from speculative_decoding_draft_07_b200 import budget

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
STOP_OFF = dict(C_d=1.0, a=0.0, b=0.0, c=0.0, e=0.0)


def _ddtree_vs_oracle(L, anchor, n, label, max_unresolved=0):
    out = budget.ddtree_grow(L.to(DEV), torch.as_tensor(anchor, dtype=torch.int32, device=DEV), n)
    torch.cuda.synchronize()
    Lh, an = L.cpu(), np.asarray(anchor)
    zero = np.zeros(1)

    def grow(b, prefer=None):
        return oracle.cadd_tree_grow(f64(Lh[b:b + 1]), an[b:b + 1], zero, n, **STOP_OFF,
                                     prefer=None if prefer is None else [prefer])

    rows = list(range(L.shape[0]))
    refs = oracle_map(grow, rows)
    cnt = host(out.count)
    compare_all(out, refs, lambda j, paths: grow(j, (paths, int(cnt[j]))), rows, label,
                max_unresolved=max_unresolved, phi=True)
    assert (host(out.status) == 0).all()
    return out, refs


@pytest.mark.slow
def test_ddtree_full_size_every_request():
    """V = 151936, D = 15, n = 512, 64 requests (the CaDDTree workload's marginals)."""
    w = workloads.CADDTREE
    d = workloads.cadd_inputs(w, 0, device=DEV)
    out, refs = _ddtree_vs_oracle(d["L"], host(d["anchor"]), w.n_max, "ddtree n=512",
                                  max_unresolved=1)
    assert (host(out.count) == w.n_max).all()


def test_ddtree_candidates_run_out_before_the_budget():
    """V = 3, D = 2 holds 3 + 9 = 12 paths: a budget of 40 nodes stops at 13."""
    g = torch.Generator().manual_seed(3)
    L = (torch.randn((4, 2, 3), generator=g) * 2).to(torch.bfloat16)
    out, refs = _ddtree_vs_oracle(L, [0, 1, 2, 0], 40, "ddtree exhausted")
    assert (host(out.count) == 13).all()


def test_budget_sweep_on_gpu_trees_matches_oracle_trees():
    """Phi_n for every n from the GPU's fixed-budget trees, then the sweep of
    fixed budgets against the adaptive size (and with a misestimated planner
    cost): the same sizes and rates as from the oracle's trees."""
    w = workloads.CADDTREE
    d = workloads.cadd_inputs(w, 0, device=DEV, batch=12)
    L = d["L"][:, :6].contiguous()                  # six depths keep the oracle quick
    n = 128
    out, refs = _ddtree_vs_oracle(L, host(d["anchor"]), n, "ddtree sweep trees")
    ells = [512, 4096, 32768] * 4
    cost = (w.C_d, w.a, w.b, w.c, w.e)
    sc, cnt = host(out.score), host(out.count)
    g_phis = [budget.phi_curve(sc[b], int(cnt[b])) for b in range(12)]
    o_phis = [budget.phi_curve(r.score[0], int(r.count[0])) for r in refs]
    for gp, op in zip(g_phis, o_phis):
        np.testing.assert_allclose(gp, op, rtol=1e-4, atol=1e-7)
    for plan in (None, (w.C_d, w.a * 1.5, w.b, w.c * 0.5, w.e * 2)):
        gs = budget.budget_sweep(g_phis, ells, cost, plan_cost=plan)
        os_ = budget.budget_sweep(o_phis, ells, cost, plan_cost=plan)
        np.testing.assert_array_equal(gs["adaptive_sizes"], os_["adaptive_sizes"])
        assert gs["best_fixed_n"] == os_["best_fixed_n"]
        assert abs(gs["gain"] - os_["gain"]) < 1e-4 * os_["gain"]
    # the adaptive size under the true cost is CaDDTree's own n* for these rounds
    for b in range(12):
        ref = oracle.cadd_tree_grow(f64(L[b:b + 1].cpu()), host(d["anchor"])[b:b + 1],
                                    np.array([ells[b]]), n, *cost)
        if not ref.excluded[0]:     # a stop test within 2e-4 of flipping may go either way
            assert budget.adaptive_size(g_phis[b], ells[b], *cost) == int(ref.count[0])
