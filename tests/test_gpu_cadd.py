"""GPU parity: CaDDTree best-first growth with the greedy stop against the oracle.

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science),
"Method: CaDDTree".
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_draft_07_b200 as pct
import workloads
from gpu_util import compare_all, f64, host, oracle_map

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
COST = dict(C_d=1.0, a=2.0, b=1e-4, c=5e-3, e=1e-5)


def _sharp_logits(batch, D, V, seed, dtype="bf16", sigma=1.0, peak=(8.0, 16.0)):
    g = torch.Generator().manual_seed(seed)
    L = torch.randn((batch, D, V), generator=g) * sigma
    tok = torch.randint(0, V, (batch, D), generator=g)
    h = torch.rand((batch, D), generator=g) * (peak[1] - peak[0]) + peak[0]
    L.scatter_add_(2, tok[..., None], h[..., None])
    return L.to(torch.bfloat16 if dtype == "bf16" else torch.float32)


def _cadd_oracle(L, anchor, ctx, n_max, cost):
    """Per-request oracle runs (in parallel) and the near-tie rebuild."""
    anchor, ctx = np.asarray(anchor), np.asarray(ctx)

    def grow(b, prefer=None):
        return oracle.cadd_tree_grow(f64(L[b:b + 1]), anchor[b:b + 1], ctx[b:b + 1], n_max, **cost,
                                     prefer=None if prefer is None else [prefer])
    return grow


def _run(L, anchor, ctx, n_max, cost, label="", max_unresolved=0):
    """GPU growth of every request, each compared with the oracle (node tables
    bit-exact, scores within 1e-4, Phi within 1e-4 relative; near ties resolved
    toward the GPU's tree)."""
    out = pct.cadd_tree_grow(L.to(DEV), torch.as_tensor(anchor, dtype=torch.int32, device=DEV),
                             torch.as_tensor(ctx, dtype=torch.int64, device=DEV), n_max, **cost)
    torch.cuda.synchronize()
    grow = _cadd_oracle(L, anchor, ctx, n_max, cost)
    rows = list(range(len(anchor)))
    refs = oracle_map(grow, rows)
    cnt = host(out.count)
    compare_all(out, refs, lambda j, paths: grow(j, (paths, int(cnt[j]))), rows, label,
                max_unresolved=max_unresolved, phi=True)
    assert (host(out.status) == 0).all()

    class Ref:   # the batch's oracle results, stacked (for the callers' extra checks)
        count = np.array([r.count[0] for r in refs])
    return out, Ref


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("V,D,n_max", [(512, 6, 64), (1000, 15, 512), (64, 4, 200), (3000, 8, 32)])
def test_sharp_marginals_deep_trees(dtype, V, D, n_max):
    batch = 8
    L = _sharp_logits(batch, D, V, seed=V + D, dtype=dtype)
    anchor = np.arange(batch) % V
    ctx = np.array([512, 4096, 32768, 0, 100, 2000, 50000, 7] * (batch // 8 + 1))[:batch]
    out, ref = _run(L, anchor, ctx, n_max, COST, label=f"sharp V={V}")
    assert ref.count.max() > 3      # trees actually grow


@pytest.mark.parametrize("seed", range(3))
def test_random_convex_costs(seed):
    rng = np.random.default_rng(seed)
    batch, D, V = 12, 10, 2048
    L = _sharp_logits(batch, D, V, seed=100 + seed, sigma=float(rng.uniform(0.5, 2)),
                      peak=(float(rng.uniform(0, 6)), float(rng.uniform(6, 20))))
    cost = dict(C_d=float(rng.uniform(0.2, 2)), a=float(rng.uniform(0, 3)), b=float(rng.uniform(0, 1e-3)),
                c=float(rng.uniform(0, 0.02)), e=float(rng.uniform(0, 1e-4)))
    _run(L, np.arange(batch), rng.integers(0, 40000, batch), 256, cost, label=f"cost{seed}")


def test_stop_disabled_uses_exact_selection_fallback():
    """c = e = 0: no threshold applies, every token survives the filter (more than the
    2048-entry buffer), so the exact radix selection of the n_max - 1 best runs."""
    batch, D, V = 4, 5, 6000
    L = _sharp_logits(batch, D, V, seed=7, sigma=1.0, peak=(0.0, 3.0))
    L[0, 0, :] = 0.25          # a row of identical values: ties resolved by token id
    cost = dict(C_d=1.0, a=1.0, b=0.0, c=0.0, e=0.0)
    out, ref = _run(L, np.arange(batch), np.zeros(batch), 40, cost, label="fallback")
    assert (ref.count == 40).all()


def test_many_rows_mixed_overflow():
    """240 rows of one segment each: in flat rows (std 0.05) more values pass than the
    finishing kernel sorts, so they take the exact selection; sharply peaked rows (std
    2, peak +40) keep one survivor; the two interleaved at random in row order."""
    batch, D, V = 16, 15, 4096
    L = _sharp_logits(batch, D, V, seed=21, sigma=0.05, peak=(0.0, 0.5)).float()
    g = torch.Generator().manual_seed(22)
    sharp = torch.rand((batch, D), generator=g) < 0.5
    tok = torch.randint(0, V, (batch, D), generator=g)
    for b in range(batch):
        for d in range(D):
            if sharp[b, d]:
                L[b, d] *= 40.0
                L[b, d, tok[b, d]] += 40.0
    L = L.to(torch.bfloat16)
    cost = dict(C_d=1.0, a=1.0, b=0.0, c=1e-6, e=0.0)
    out, ref = _run(L, np.arange(batch), np.arange(batch) * 1000, 32, cost, label="mixed overflow")
    assert (ref.count == 32).all()


@pytest.mark.parametrize("seed", [51, 52])
def test_multi_segment_rows(seed):
    """V = 47784: each row splits into five segments of the row pass (four of 1280
    16-byte groups and one of 853), each marking the groups above its own threshold
    for the finishing kernel to test against the row's; the short last segment takes
    the bounds-checked loads."""
    batch, D, V = 8, 6, 47784
    L = _sharp_logits(batch, D, V, seed=seed, sigma=2.0, peak=(0.0, 6.0))
    ctx = np.array([512, 4096, 32768, 0, 100, 2000, 50000, 7])
    out, ref = _run(L, np.arange(batch), ctx, 128, COST, label=f"segments {seed}")
    assert ref.count.max() > 30


@pytest.mark.parametrize("V", [20488, 183520])
def test_segment_edges(V):
    """V = 20488: a last segment of one 16-byte group; V = 183520: eighteen segments,
    a bitmap of 717 words per row."""
    batch, D = 2, 3
    L = _sharp_logits(batch, D, V, seed=V % 97, sigma=2.0, peak=(0.0, 6.0))
    ctx = np.array([4096, 32768])
    out, ref = _run(L, np.arange(batch), ctx, 128, COST, label=f"segment edges V={V}")
    assert ref.count.max() > 30


def test_multi_segment_overflow():
    """Five segments per row: flat rows mark more groups than the finishing kernel lists
    (exact selection over the row), interleaved with sharply peaked rows."""
    batch, D, V = 6, 5, 47784
    L = _sharp_logits(batch, D, V, seed=41, sigma=0.05, peak=(0.0, 0.5)).float()
    g = torch.Generator().manual_seed(42)
    sharp = torch.rand((batch, D), generator=g) < 0.5
    tok = torch.randint(0, V, (batch, D), generator=g)
    for b in range(batch):
        for d in range(D):
            if sharp[b, d]:
                L[b, d] *= 40.0
                L[b, d, tok[b, d]] += 40.0
    L = L.to(torch.bfloat16)
    cost = dict(C_d=1.0, a=1.0, b=0.0, c=1e-6, e=0.0)
    out, ref = _run(L, np.arange(batch), np.arange(batch) * 1000, 32, cost, label="segment overflow")
    assert (ref.count == 32).all()


def test_exhausted_small_vocab():
    L = _sharp_logits(3, 2, 3, seed=3, sigma=0.5, peak=(0.0, 0.1))
    cost = dict(C_d=1.0, a=0.0, b=0.0, c=0.0, e=0.0)
    out, ref = _run(L, [0, 1, 2], [0, 0, 0], 100, cost, label="exhausted")
    assert (ref.count == 13).all()


def test_bad_cost_flagged():
    L = _sharp_logits(2, 3, 256, seed=4)
    cost = dict(C_d=-10.0, a=0.0, b=0.0, c=0.01, e=0.0)     # C(n) <= 0 for small n
    out = pct.cadd_tree_grow(L.to(DEV), torch.tensor([0, 1], dtype=torch.int32, device=DEV),
                             torch.zeros(2, dtype=torch.int64, device=DEV), 16, **cost)
    torch.cuda.synchronize()
    assert (host(out.status) & pct.DEV_BAD_COST).all()


@pytest.mark.slow
@pytest.mark.parametrize("ell", workloads.CADDTREE.ells)
def test_caddtree_workload_full_size(ell):
    """64 requests, V = 151936, D = 15, n_max = 512: every request against the oracle."""
    w = workloads.CADDTREE
    d = workloads.cadd_inputs(w, ell, device=DEV)
    cost = dict(C_d=w.C_d, a=w.a, b=w.b, c=w.c, e=w.e)
    out, ref = _run(d["L"].cpu(), host(d["anchor"]), host(d["ctx_len"]), w.n_max, cost,
                    label=f"caddtree l={ell} (cfg 3)", max_unresolved=1)
    counts = host(out.count)
    assert (counts >= 2).all() and (counts <= w.n_max).all()
