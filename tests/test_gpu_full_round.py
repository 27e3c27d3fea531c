"""GPU parity of one full round at full size: PCTree build (64 requests, N = 256,
V = 151936, D = 15), ancestor mask and greedy verification on planted target logits.

Two sampled requests are rebuilt by the oracle; the target logits of those
requests are planted along the ORACLE's trees, so no oracle input comes from
the GPU. Every other request is checked for the output invariants and for a
walk that is consistent with the GPU's own argmax.
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_draft_07_b200 as pct
import workloads
from gpu_util import check_tree_invariants, compare_trees, f64, host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = torch.device("cuda")


def test_full_round_sampled():
    w = workloads.FULL_ROUND
    d = workloads.drafter_inputs(w, device=DEV)
    out = pct.pct_tree_build(d["L"], d["anchor"], d["E"], d["W"], w.k, w.beam, w.n_nodes)
    torch.cuda.synchronize()
    check_tree_invariants(out, host(d["anchor"]), w.n_nodes, "full round")
    assert (host(out.count) == w.n_nodes).all()          # N = 256 binds (456 nodes kept)

    sample = [0, 37]
    ref = oracle.pct_tree_build(f64(d["L"][sample]), host(d["anchor"])[sample], f64(d["E"]),
                                f64(d["W"]), w.k, w.beam, w.n_nodes)
    n = compare_trees(out, ref, rows=sample, label="full round")
    assert n >= 1

    # planting trees: the oracle's for the sampled requests, the bare root elsewhere
    B, N = w.batch, w.n_nodes
    ptok = np.full((B, N), -1, np.int32)
    ppar = np.full((B, N), -1, np.int32)
    pcnt = np.ones(B, np.int32)
    ptok[:, 0] = host(d["anchor"])
    for j, b in enumerate(sample):
        ptok[b], ppar[b], pcnt[b] = ref.tok[j], ref.parent[j], ref.count[j]
    T = workloads.target_logits(B, N, w.vocab, workloads.FULL_ROUND_TARGET_SIGMA,
                                seed=w.seed + 1000, device=DEV)
    walked, paths, ends = workloads.plant_path(T, ptok, ppar, pcnt, seed=w.seed + 1001)

    mask, mstat = pct.tree_ancestor_mask(out.parent, out.count)
    v = pct.tree_verify_accept(out.tok, out.parent, out.count, T, max_depth=w.depth)
    torch.cuda.synchronize()
    assert (host(mstat) == 0).all() and (host(v.status) == 0).all()

    rmask = oracle.tree_ancestor_mask(ref.parent, ref.count, N)
    rver = oracle.tree_verify_accept(ref.tok, ref.parent, ref.count, T[sample], max_depth=w.depth)
    gm = host(mask).view(np.uint32)
    for j, b in enumerate(sample):
        if ref.excluded[j]:
            continue
        np.testing.assert_array_equal(gm[b], rmask[j])
        np.testing.assert_array_equal(host(v.argmax)[b], rver.argmax[j])
        assert host(v.accept_len)[b] == rver.accept_len[j] == walked[b]
        np.testing.assert_array_equal(host(v.accept_path)[b], rver.accept_path[j])
        assert host(v.correction)[b] == rver.correction[j] == ends[b]

    # every request: the walk follows the GPU's own argmax through the GPU's tree
    tok, par, am = host(out.tok), host(out.parent), host(v.argmax)
    alen, apath, corr = host(v.accept_len), host(v.accept_path), host(v.correction)
    for b in range(B):
        u = 0
        for i in range(alen[b]):
            c = apath[b, i]
            assert par[b, c] == u and tok[b, c] == am[b, u]
            u = c
        kids = np.nonzero(par[b] == u)[0]
        assert not (tok[b, kids] == am[b, u]).any()
        assert corr[b] == am[b, u]
        words = gm[b]
        for i in range(N):   # mask invariant: popcount = depth + 1
            assert sum(bin(int(x)).count("1") for x in words[i]) == host(out.depth)[b, i] + 1
    del T
    torch.cuda.empty_cache()
