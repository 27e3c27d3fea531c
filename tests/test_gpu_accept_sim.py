"""GPU parity of the acceptance simulation (tau = accepted drafts + 1).

DSpark explainer (xiaohu-jiedu), one round from drafting to confirmation; PCTree
article (qiita), numbers table (tau). The kernel and the oracle draw the same
Philox numbers, so every walk is the same on both sides: the histograms must be
equal. On full-size trees with the drafter as the target, the mean accepted
length must match Phi(T) ("Cost-Aware Diffusion Draft Trees for Speculative
Decoding", gist.science summary, "Method: CaDDTree") within four standard
errors.
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_draft_07_b200 as pct
import workloads
from gpu_util import host

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _random_probs(par, cnt, seed, mass=0.9):
    """Per-node probabilities whose children sums are at most `mass`."""
    rng = np.random.default_rng(seed)
    p = np.zeros(par.shape, np.float32)
    for b in range(par.shape[0]):
        n = int(cnt[b])
        for u in range(n):
            kids = np.nonzero(par[b, :n] == u)[0]
            if len(kids):
                w = rng.dirichlet(np.ones(len(kids) + 1))[: len(kids)] * mass
                p[b, kids] = w.astype(np.float32)
    return p


@pytest.mark.parametrize("n_stride,D,trials,seed", [(60, 8, 3000, 11), (256, 15, 2000, 1 << 40),
                                                     (7, 3, 5000, 5)])
def test_histograms_equal_oracle(n_stride, D, trials, seed):
    batch = 5
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, 50, D, seed=n_stride)
    p = _random_probs(par, cnt, seed=n_stride + 1)
    hist, st = pct.tree_accept_sim(torch.from_numpy(par).to(DEV), torch.from_numpy(cnt).to(DEV),
                                   torch.from_numpy(p).to(DEV), trials, seed, D)
    torch.cuda.synchronize()
    ref = oracle.accept_sim(par, cnt, p, trials, seed, D)
    np.testing.assert_array_equal(host(hist), ref)
    assert (host(st) == 0).all()


def test_bad_tree_is_flagged():
    par = np.array([[-1, 0, 5, -1], [-1, 0, 1, 2]], np.int32)
    cnt = np.array([3, 9], np.int32)
    p = np.full(par.shape, 0.5, np.float32)
    hist, st = pct.tree_accept_sim(torch.from_numpy(par).to(DEV), torch.from_numpy(cnt).to(DEV),
                                   torch.from_numpy(p).to(DEV), 100, 1, 4)
    torch.cuda.synchronize()
    s = host(st)
    assert s[0] & pct.DEV_BAD_PARENT and s[1] & pct.DEV_BAD_COUNT
    assert (host(hist) == 0).all()


@pytest.mark.slow
def test_identity_on_full_size_caddtree_trees():
    """64 requests, V = 151936, D = 15, n_max = 512 (context 32768): the drafter as
    the target, p(child) = exp(s(child) - s(parent)); 2e5 walks per request."""
    w = workloads.CADDTREE
    d = workloads.cadd_inputs(w, 32768, device=DEV)
    out = pct.cadd_tree_grow(d["L"], d["anchor"], d["ctx_len"], w.n_max,
                             C_d=w.C_d, a=w.a, b=w.b, c=w.c, e=w.e)
    par = out.parent.to(torch.int64).clamp(min=0)
    p = torch.where(out.parent >= 0, torch.exp(out.score - out.score.gather(1, par)),
                    torch.zeros_like(out.score)).contiguous()
    trials = 200000
    hist, st = pct.tree_accept_sim(out.parent, out.count, p, trials, 2024, w.depth)
    torch.cuda.synchronize()
    assert (host(st) == 0).all()
    h = host(hist).astype(np.float64)
    lens = np.arange(h.shape[1])
    mean = (h * lens).sum(1) / trials
    var = (h * lens ** 2).sum(1) / trials - mean ** 2
    phi = host(out.phi).astype(np.float64)
    assert (np.abs(mean - phi) <= 4 * np.sqrt(var / trials) + 1e-6).all()
    # and walk by walk on two requests against the oracle (same numbers)
    sub = [0, 63]
    hs, _ = pct.tree_accept_sim(out.parent[sub].contiguous(), out.count[sub].contiguous(),
                                p[sub].contiguous(), 3000, 77, w.depth)
    torch.cuda.synchronize()
    ref = oracle.accept_sim(host(out.parent)[sub], host(out.count)[sub], host(p)[sub], 3000, 77,
                            w.depth)
    # the request index is part of the counter: request j of the sub-batch
    np.testing.assert_array_equal(host(hs), ref)
