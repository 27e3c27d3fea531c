"""GPU parity: PCTree (batched parent scoring, log-softmax, local top-k, beam,
global top-N) against the oracle.

PCTree article (qiita), section on the chain draft's weakness and the tree
built in its place.
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_draft_07_b200 as pct
import workloads
from gpu_util import SCORE_TOL, check_tree_invariants, compare_all, f64, host, oracle_map

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _problem(batch, D, V, r, seed, dtype="bf16", sigma=2.0, peak=(2.0, 10.0), ew=0.3):
    g = torch.Generator().manual_seed(seed)
    L = torch.randn((batch, D, V), generator=g) * sigma
    pt = torch.randint(0, V, (batch, D), generator=g)
    ph = torch.rand((batch, D), generator=g) * (peak[1] - peak[0]) + peak[0]
    L.scatter_add_(2, pt[..., None], ph[..., None])
    E = torch.randn((V, r), generator=g) * ew
    W = torch.randn((r, V), generator=g) * ew
    anchor = torch.randint(0, V, (batch,), generator=g, dtype=torch.int64).to(torch.int32)
    t = torch.bfloat16 if dtype == "bf16" else torch.float32
    return L.to(t), anchor, E.to(t), W.to(t)


def _score_ref(L_row, ptok, E, W, k):
    """Oracle per-parent scoring for every request; returns lse, top tokens, log pi,
    and a mask of rows whose k-th / (k+1)-th values are closer than the tolerance."""
    Lf, Ef, Wf = f64(L_row), f64(E), f64(W)
    lse_all, tok_all, lp_all, near_all = [], [], [], []
    for b in range(Lf.shape[0]):
        Z, markov, logpi, lse, order = oracle.score_parents(Lf[b], ptok[b], Ef, Wf, k)
        rows = np.arange(Z.shape[0])[:, None]
        top = order[:, :k]
        lse_all.append(lse)
        tok_all.append(top)
        lp_all.append(logpi[rows, top])
        if order.shape[1] > k:
            zk, zk1 = Z[rows[:, 0], order[:, k - 1]], Z[rows[:, 0], order[:, k]]
            near = (np.abs(zk - zk1) < SCORE_TOL)
        else:
            near = np.zeros(Z.shape[0], bool)
        # near ties inside the top-k permute tokens too; compare those rows as sets
        zs = Z[rows, order[:, :k]]
        near_in = (np.abs(np.diff(zs, axis=1)) < SCORE_TOL).any(axis=1) if k > 1 else np.zeros_like(near)
        near_all.append((near, near_in))
    return (np.stack(lse_all), np.stack(tok_all), np.stack(lp_all), near_all)


def _score_parents_case(dtype, V, r, k, batch, n_par, logits_dtype=None):
    L, _, E, W = _problem(batch, 1, V, r, seed=V + r + k, dtype=dtype)
    L = L[:, 0, :].contiguous()
    if logits_dtype is not None:
        L = L.to(logits_dtype)
    g = torch.Generator().manual_seed(k)
    ptok = torch.randint(0, V, (batch, n_par), generator=g, dtype=torch.int64).to(torch.int32)
    lse, tt, tl, st = pct.pct_score_parents(L.to(DEV), ptok.to(DEV), E.to(DEV), W.to(DEV), k)
    torch.cuda.synchronize()
    rl, rt, rlp, near = _score_ref(L, ptok.numpy(), E, W, k)
    np.testing.assert_allclose(host(lse), rl, rtol=0, atol=SCORE_TOL)
    gt, gl = host(tt), host(tl)
    skipped = 0
    for b in range(batch):
        nb, nin = near[b]
        for p in range(n_par):
            if nb[p]:
                skipped += 1
                continue
            if nin[p]:
                assert sorted(gt[b, p]) == sorted(rt[b, p])
            else:
                np.testing.assert_array_equal(gt[b, p], rt[b, p], err_msg=f"row {b},{p}")
            np.testing.assert_allclose(gl[b, p], rlp[b, p], rtol=0, atol=SCORE_TOL)
    assert skipped <= max(1, batch * n_par // 50)
    assert (host(st) == 0).all()


@pytest.mark.parametrize("dtype,V,r,k,batch,n_par", [
    ("bf16", 1024, 64, 4, 1, 1), ("bf16", 1024, 16, 8, 3, 40), ("bf16", 2048, 100, 8, 2, 200),
    ("bf16", 4096, 256, 16, 3, 100), ("bf16", 64, 64, 1, 2, 5), ("bf16", 1000, 256, 8, 1, 130),
    ("f32", 1000, 16, 4, 2, 7), ("f32", 777, 33, 8, 3, 20)])
def test_score_parents_matches_oracle(dtype, V, r, k, batch, n_par):
    _score_parents_case(dtype, V, r, k, batch, n_par)


@pytest.mark.parametrize("batch,n_par,mode", [
    (3, 40, "fold, one row tile"), (4, 64, "fold, two row tiles"),
    (5, 100, "fold, requests straddle CTAs"), (16, 16, "fold, 16 requests per CTA"),
    (24, 2, "staged tiles, 24 requests per CTA"), (80, 1, "global loads, 80 requests per CTA"),
    (40, 4, "CTA pairs, global loads, 40 requests per pair"),
    (2, 65, "CTA pairs, fold, second CTA nearly empty")])
def test_score_parents_logits_modes(batch, n_par, mode):
    """The tensor-core path adds L_d in the MMA (at most 16 requests per CTA or
    CTA pair), in the epilogue from staged shared-memory tiles (at most 64, up to
    128 rows), or from global memory (more); more than 128 rows run on CTA pairs.
    Each mode against the oracle."""
    _score_parents_case("bf16", 3000, 128, 8, batch, n_par)


@pytest.mark.parametrize("batch,n_par", [(3, 30), (3, 60)])
def test_score_parents_fp32_logits_bf16_markov(batch, n_par):
    _score_parents_case("bf16", 2000, 64, 8, batch, n_par, logits_dtype=torch.float32)


def _build_and_compare(L, anchor, E, W, k, beam, N, label="", max_unresolved=0, seeds=None):
    """GPU build of every request, each compared with the oracle (near ties
    resolved toward the GPU's nodes; at most ``max_unresolved`` requests may
    stay unmatched). seeds: the gate columns of pct_tree_build_seeded."""
    out = pct.pct_tree_build(L.to(DEV), anchor.to(DEV), E.to(DEV), W.to(DEV), k, beam, N,
                             seeds=None if seeds is None else seeds.to(DEV))
    torch.cuda.synchronize()
    check_tree_invariants(out, anchor.numpy(), N, label)
    Ef, Wf, an = f64(E), f64(W), anchor.numpy()

    def build(b, prefer=None):
        return oracle.pct_tree_build(f64(L[b:b + 1]), an[b:b + 1], Ef, Wf, k, beam, N,
                                     prefer=None if prefer is None else [prefer])

    rows = list(range(L.shape[0]))
    refs = oracle_map(build, rows)
    compare_all(out, refs, lambda j, paths: build(j, paths), rows, label,
                max_unresolved=max_unresolved)
    assert (host(out.status) == 0).all()
    return out, refs


def test_tiny_workload_fp32():
    w = workloads.WORKLOADS["tiny"]
    d = workloads.drafter_inputs(w)
    out, ref = _build_and_compare(d["L"], d["anchor"], d["E"], d["W"], w.k, w.beam, w.n_nodes,
                                  label="tiny (cfg 0)")
    assert host(out.count)[0] == 25


@pytest.mark.parametrize("dtype,V,D,r,k,beam,N,batch", [
    ("bf16", 2048, 4, 64, 4, 8, 32, 4), ("bf16", 1024, 6, 256, 8, 16, 64, 3),
    ("bf16", 4096, 5, 100, 8, 32, 128, 5), ("bf16", 512, 8, 32, 2, 5, 40, 6),
    ("bf16", 3000, 3, 16, 16, 64, 200, 2), ("f32", 1500, 5, 24, 4, 8, 40, 4),
    ("f32", 1000, 6, 16, 3, 6, 30, 3)])
def test_small_builds_match_oracle(dtype, V, D, r, k, beam, N, batch):
    L, anchor, E, W = _problem(batch, D, V, r, seed=V + D + r, dtype=dtype)
    _build_and_compare(L, anchor, E, W, k, beam, N, label=f"small {dtype} V={V} D={D}")


def test_k1_is_the_greedy_chain_on_gpu():
    L, anchor, E, W = _problem(4, 6, 1024, 64, seed=9)
    out, ref = _build_and_compare(L, anchor, E, W, 1, 4, 7, label="chain")
    assert (host(out.count) == 7).all()
    assert (host(out.parent)[:, 1:] == np.arange(6)).all()


def test_zero_markov_exact_ties():
    """W = 0: every parent of a depth sees the same row, many exact ties in bf16."""
    L, anchor, E, W = _problem(3, 5, 1024, 64, seed=11, sigma=1.0)
    W = torch.zeros_like(W)
    L[0, 1, 10:20] = 6.0          # ten identical peaks
    _build_and_compare(L, anchor, E, W, 8, 16, 64, label="zero markov, exact ties")


def test_seeded_gate_with_ties_across_slices():
    """W = 0 and twelve equal peaks spread over the vocabulary: each row's k-th
    value is a tie held by columns in different V-slices, and the row's seeded
    gate sits just below it (the rounding allowance); the lower token ids win."""
    L, anchor, E, W = _problem(2, 3, 8192, 64, seed=21, sigma=1.0)
    W = torch.zeros_like(W)
    for b in range(2):
        for d in range(3):
            L[b, d, torch.arange(12) * 677 + 5 + d] = 6.0
    _build_and_compare(L, anchor, E, W, 8, 16, 40, label="ties across slices")


def test_strong_markov_loose_seed():
    """Markov term several times larger than the drafter logits: the drafter's
    best columns are not the parents' best, so every seed is loose."""
    L, anchor, E, W = _problem(8, 4, 4096, 128, seed=23, sigma=0.5, ew=0.6)
    _build_and_compare(L, anchor, E, W, 8, 16, 64, label="strong markov")


def test_vocab_too_small_for_seed_columns():
    """V = 64 has eight 8-column groups, fewer than k = 16 seed columns: the
    rows are scored without seeds."""
    L, anchor, E, W = _problem(2, 3, 64, 32, seed=25)
    _build_and_compare(L, anchor, E, W, 16, 32, 60, label="v64 no seeds")


def test_repeated_builds_are_bit_identical():
    L, anchor, E, W = _problem(4, 6, 2048, 64, seed=13)
    Ld, ad, Ed, Wd = L.to(DEV), anchor.to(DEV), E.to(DEV), W.to(DEV)
    first = pct.pct_tree_build(Ld, ad, Ed, Wd, 8, 16, 64)
    ref = [host(x).copy() for x in (first.tok, first.parent, first.score, first.count)]
    for _ in range(10):
        o = pct.pct_tree_build(Ld, ad, Ed, Wd, 8, 16, 64)
        for x, y in zip(ref, (o.tok, o.parent, o.score, o.count)):
            np.testing.assert_array_equal(x, host(y))


@pytest.mark.slow
def test_qwen3_4b_scale_workload():
    """V = 151936, B = 7, r = 256, k = 8, beam 16, N = 64, one request."""
    w = workloads.WORKLOADS["qwen3_4b_scale"]
    d = workloads.drafter_inputs(w, device=DEV)
    L, a, E, W = (d[x].cpu() for x in ("L", "anchor", "E", "W"))
    _build_and_compare(L, a, E, W, w.k, w.beam, w.n_nodes, label="qwen3-4b scale (cfg 1)")


@pytest.mark.slow
def test_long_block_workload_every_request():
    """V = 151936, B = 16, r = 256, k = 8, beam 32, N = 128, 32 requests: all of
    them against the oracle."""
    w = workloads.WORKLOADS["long_block"]
    d = workloads.drafter_inputs(w, device=DEV)
    L, a, E, W = (d[x].cpu() for x in ("L", "anchor", "E", "W"))
    _build_and_compare(L, a, E, W, w.k, w.beam, w.n_nodes, label="long block (cfg 2)",
                       max_unresolved=1)


# ---------------------------------------------------------------------------
# The persistent small-frontier path (one launch for all depths: at most 16
# requests, 128 parent rows per depth, beam <= 32, bf16 logits and Markov
# parameters) and the multi-launch path on the same small problems.
def _kernels_of(fn):
    pct.trace_enable(True)
    pct.trace_reset()
    out = fn()
    torch.cuda.synchronize()
    names = set(pct.trace_read())
    pct.trace_enable(False)
    return out, names


@pytest.mark.parametrize("V,D,r,k,beam,N,batch", [
    (3000, 4, 64, 4, 8, 32, 4),      # 4 -> 32 rows: four copies per lane quarter; 24 CTAs
    (8192, 5, 96, 8, 24, 60, 2),     # up to 48 rows: two copies; r = 96 (zero K past r)
    (4096, 4, 256, 8, 32, 80, 4),    # 128 rows: one copy; full K
    (2048, 6, 128, 16, 32, 100, 1),  # k = 16
    (1024, 6, 64, 1, 4, 7, 5),       # k = 1: chains
    (20488, 3, 256, 8, 8, 20, 16),   # 16 requests: every request row of the folded L_d
])
def test_persistent_path_matches_oracle(V, D, r, k, beam, N, batch):
    L, anchor, E, W = _problem(batch, D, V, r, seed=V + 3 * D + k)
    out, names = _kernels_of(lambda: pct.pct_tree_build(L.to(DEV), anchor.to(DEV), E.to(DEV),
                                                        W.to(DEV), k, beam, N))
    assert "pct_chain" in names and "pct_score_umma" not in names, names
    _build_and_compare(L, anchor, E, W, k, beam, N, label=f"persistent V={V} k={k} b={batch}")


def test_persistent_path_qwen3_scale_is_used():
    w = workloads.WORKLOADS["qwen3_4b_scale"]
    d = workloads.drafter_inputs(w, device=DEV)
    _, names = _kernels_of(lambda: pct.pct_tree_build(d["L"], d["anchor"], d["E"], d["W"], w.k,
                                                      w.beam, w.n_nodes))
    assert "pct_chain" in names, names


@pytest.mark.parametrize("V,D,r,k,beam,N", [(3000, 4, 64, 4, 8, 32), (4096, 5, 128, 8, 16, 64)])
def test_multi_launch_path_on_small_problems(V, D, r, k, beam, N):
    """17 requests are past the persistent path's 16: the per-depth launches run."""
    L, anchor, E, W = _problem(17, D, V, r, seed=V + D + 77)
    out, names = _kernels_of(lambda: pct.pct_tree_build(L.to(DEV), anchor.to(DEV), E.to(DEV),
                                                        W.to(DEV), k, beam, N))
    assert "pct_chain" not in names and "pct_merge_beam" in names, names
    _build_and_compare(L, anchor, E, W, k, beam, N, label=f"multi-launch V={V}")


def test_persistent_path_flags_bad_anchor():
    L, anchor, E, W = _problem(3, 3, 2048, 64, seed=5)
    anchor[1] = 2048                  # outside the vocabulary
    out = pct.pct_tree_build(L.to(DEV), anchor.to(DEV), E.to(DEV), W.to(DEV), 4, 8, 20)
    torch.cuda.synchronize()
    st = host(out.status)
    assert st[1] & pct.DEV_BAD_TOKEN and st[0] == 0 and st[2] == 0


def test_persistent_path_repeated_builds_are_bit_identical():
    L, anchor, E, W = _problem(2, 6, 4096, 128, seed=31)
    Ld, ad, Ed, Wd = L.to(DEV), anchor.to(DEV), E.to(DEV), W.to(DEV)
    first = pct.pct_tree_build(Ld, ad, Ed, Wd, 8, 16, 64)
    ref = [host(x).copy() for x in (first.tok, first.parent, first.score, first.count)]
    for _ in range(20):
        o = pct.pct_tree_build(Ld, ad, Ed, Wd, 8, 16, 64)
        for x, y in zip(ref, (o.tok, o.parent, o.score, o.count)):
            np.testing.assert_array_equal(x, host(y))
