"""GPU parity of one full round at full size: PCTree build (64 requests, N = 256,
V = 151936, D = 15), ancestor mask and greedy verification on planted target logits.

Every request is rebuilt by the oracle (in parallel over the host cores) and
compared element by element; a request with a near tie at a selection boundary
is compared against the oracle's tree with that near tie resolved toward the
GPU's nodes. Verification and the mask are compared on the ORACLE's trees
(target logits planted along them), so no oracle input comes from the GPU.
The chained round (GPU build, then GPU mask and verify on the GPU's trees) is
checked for consistency on every request.
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_draft_07_b200 as pct
import workloads
from gpu_util import (check_tree_invariants, compare_all, f64, host, oracle_map, report)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = torch.device("cuda")


def test_full_round_every_request():
    w = workloads.FULL_ROUND
    d = workloads.drafter_inputs(w, device=DEV)
    out = pct.pct_tree_build(d["L"], d["anchor"], d["E"], d["W"], w.k, w.beam, w.n_nodes)
    torch.cuda.synchronize()
    anchor = host(d["anchor"])
    check_tree_invariants(out, anchor, w.n_nodes, "full round")
    assert (host(out.count) == w.n_nodes).all()          # N = 256 binds (456 nodes kept)
    assert (host(out.status) == 0).all()

    B, N = w.batch, w.n_nodes
    E, Wm = f64(d["E"]), f64(d["W"])
    Lh = d["L"].cpu()

    def build(b, prefer=None):
        return oracle.pct_tree_build(f64(Lh[b:b + 1]), anchor[b:b + 1], E, Wm, w.k, w.beam,
                                     w.n_nodes, prefer=None if prefer is None else [prefer])

    refs = oracle_map(build, range(B))
    compare_all(out, refs, lambda j, paths: build(j, paths), list(range(B)), "full round build")

    # oracle trees, and target logits planted along them
    rtok = np.stack([r.tok[0] for r in refs])
    rpar = np.stack([r.parent[0] for r in refs])
    rcnt = np.array([r.count[0] for r in refs], np.int32)
    T = workloads.target_logits(B, N, w.vocab, workloads.FULL_ROUND_TARGET_SIGMA,
                                seed=w.seed + 1000, device=DEV)
    walked, paths, ends = workloads.plant_path(T, rtok, rpar, rcnt, seed=w.seed + 1001)

    # verification and mask on the oracle's trees
    dt, dp, dc = (torch.from_numpy(x).to(DEV) for x in (rtok, rpar, rcnt))
    mask, mstat = pct.tree_ancestor_mask(dp, dc)
    v = pct.tree_verify_accept(dt, dp, dc, T, max_depth=w.depth)
    torch.cuda.synchronize()
    assert (host(mstat) == 0).all() and (host(v.status) == 0).all()
    Th = T.cpu()
    rvers = oracle_map(lambda b: oracle.tree_verify_accept(rtok[b:b + 1], rpar[b:b + 1],
                                                           rcnt[b:b + 1], Th[b:b + 1],
                                                           max_depth=w.depth), range(B))
    rmask = oracle.tree_ancestor_mask(rpar, rcnt, N)
    np.testing.assert_array_equal(host(mask).view(np.uint32), rmask)
    for b, rv in enumerate(rvers):
        np.testing.assert_array_equal(host(v.argmax)[b], rv.argmax[0], err_msg=f"argmax {b}")
        assert host(v.accept_len)[b] == rv.accept_len[0] == walked[b]
        np.testing.assert_array_equal(host(v.accept_path)[b], rv.accept_path[0])
        assert host(v.correction)[b] == rv.correction[0] == ends[b]
    report("full round verify + mask", B, B, 0, 0)

    # the lazy walk on the same trees: same acceptance, argmax of the walked rows only
    lw = pct.tree_verify_walk(dt, dp, dc, T, max_depth=w.depth)
    torch.cuda.synchronize()
    assert (host(lw.status) == 0).all()
    np.testing.assert_array_equal(host(lw.accept_len), host(v.accept_len))
    np.testing.assert_array_equal(host(lw.accept_path), host(v.accept_path))
    np.testing.assert_array_equal(host(lw.correction), host(v.correction))
    lam = host(lw.argmax)
    for b, rv in enumerate(rvers):
        walked = [0] + [int(x) for x in rv.accept_path[0, : rv.accept_len[0]]]
        want = np.full(N, -1, np.int32)
        want[walked] = rv.argmax[0, walked]
        np.testing.assert_array_equal(lam[b], want, err_msg=f"walk argmax {b}")
    report("full round lazy walk", B, B, 0, 0)

    # the chained round on the GPU's own trees: the walk follows the GPU's argmax
    mask2, _ = pct.tree_ancestor_mask(out.parent, out.count)
    v2 = pct.tree_verify_accept(out.tok, out.parent, out.count, T, max_depth=w.depth)
    torch.cuda.synchronize()
    tok, par, am = host(out.tok), host(out.parent), host(v2.argmax)
    alen, apath, corr = host(v2.accept_len), host(v2.accept_path), host(v2.correction)
    gm, dep = host(mask2).view(np.uint32), host(out.depth)
    for b in range(B):
        u = 0
        for i in range(alen[b]):
            c = apath[b, i]
            assert par[b, c] == u and tok[b, c] == am[b, u]
            u = c
        kids = np.nonzero(par[b] == u)[0]
        assert not (tok[b, kids] == am[b, u]).any()
        assert corr[b] == am[b, u]
        pop = np.unpackbits(gm[b].view(np.uint8), axis=1).sum(axis=1)
        np.testing.assert_array_equal(pop, dep[b] + 1)     # popcount = depth + 1
    del T
    torch.cuda.empty_cache()
