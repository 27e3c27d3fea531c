"""GPU parity: one pass over the drafter logits serving both trees.

cadd_tree_grow_topk writes, beside the CaDDTree, each row's top-k tokens by
logit; they are compared with oracle.row_topk exactly and the trees with
cadd_tree_grow's bit for bit. pct_tree_build_seeded takes such columns as the
seeds of its top-k gate; the gate only decides which values a parent's
running top-k looks at, so the trees must equal the unseeded build's bit for
bit (and the oracle's), whatever the seeds.

"Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science),
"Method: CaDDTree" (best-first by marginal); PCTree article (qiita), section
on the tree that replaces the chain draft (local top-k of z_d(p) = L_d +
Markov(p)).
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_draft_07_b200 as pct
import workloads
from gpu_util import f64, host
from test_gpu_cadd import _sharp_logits
from test_gpu_pctree import _build_and_compare, _kernels_of, _problem

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
COST = dict(C_d=1.0, a=2.0, b=1e-4, c=5e-3, e=1e-5)


def _grow_both(L, anchor, ctx, n_max, cost, top_k):
    """cadd_tree_grow and cadd_tree_grow_topk on the same inputs."""
    Ld = L.to(DEV)
    a = torch.as_tensor(anchor, dtype=torch.int32, device=DEV)
    c = torch.as_tensor(ctx, dtype=torch.int64, device=DEV)
    plain = pct.cadd_tree_grow(Ld, a, c, n_max, **cost)
    top = torch.full((L.shape[0], L.shape[1], top_k), -7, dtype=torch.int32, device=DEV)
    withk = pct.cadd_tree_grow(Ld, a, c, n_max, **cost, top_tok=top)
    torch.cuda.synchronize()
    return plain, withk, host(top)


def _same_tree(x, y, phi=False):
    for f in ("tok", "parent", "depth", "score", "count", "status") + (("phi",) if phi else ()):
        np.testing.assert_array_equal(host(getattr(x, f)), host(getattr(y, f)), err_msg=f)


def _check_topk(L, anchor, ctx, n_max, cost, top_k):
    plain, withk, top = _grow_both(L, anchor, ctx, n_max, cost, top_k)
    _same_tree(plain, withk, phi=True)
    np.testing.assert_array_equal(top, oracle.row_topk(f64(L), top_k))
    return top


@pytest.mark.parametrize("dtype,V,D,batch,n_max,top_k", [
    ("bf16", 20000, 4, 3, 64, 8),      # two segments per row
    ("bf16", 20000, 4, 3, 64, 32),
    ("bf16", 4096, 6, 5, 200, 16),     # one segment
    ("f32", 3000, 5, 4, 128, 16),      # the single-kernel row pass
    ("bf16", 3001, 3, 2, 64, 8),       # V % 8 != 0: the single-kernel row pass
])
def test_grow_topk_is_each_rows_top_k(dtype, V, D, batch, n_max, top_k):
    L = _sharp_logits(batch, D, V, seed=V + D + top_k, dtype=dtype)
    _check_topk(L, np.arange(batch), np.arange(batch) * 3000 + 512, n_max, COST, top_k)


def test_grow_topk_rows_with_few_survivors():
    """Sharply peaked rows keep one value above the threshold, fewer than top_k:
    their top_k is selected exactly over the row; flat rows overflow the sorted
    buffer and take the exact selection of n_max - 1 (more than top_k)."""
    batch, D, V = 8, 6, 4096
    L = _sharp_logits(batch, D, V, seed=3, sigma=0.05, peak=(0.0, 0.5)).float()
    g = torch.Generator().manual_seed(4)
    sharp = torch.rand((batch, D), generator=g) < 0.5
    tok = torch.randint(0, V, (batch, D), generator=g)
    for b in range(batch):
        for d in range(D):
            if sharp[b, d]:
                L[b, d] *= 40.0
                L[b, d, tok[b, d]] += 40.0
    L = L.to(torch.bfloat16)
    _check_topk(L, np.arange(batch), np.arange(batch) * 1000, 32, dict(C_d=1.0, a=1.0, b=0.0,
                                                                       c=1e-6, e=0.0), 8)


@pytest.mark.parametrize("n_max,top_k", [(1, 8), (5, 16), (40, 8)])
def test_grow_topk_exact_paths(n_max, top_k):
    """n_max = 1: no candidates at all; stop disabled (c = e = 0): every value
    survives and the exact selection keeps n_max - 1, below or above top_k. A
    row of equal values: ties go to the lower token ids."""
    batch, D, V = 3, 4, 6000
    L = _sharp_logits(batch, D, V, seed=n_max + top_k, sigma=1.0, peak=(0.0, 3.0))
    L[0, 0, :] = 0.25
    _check_topk(L, np.arange(batch), np.zeros(batch), n_max,
                dict(C_d=1.0, a=1.0, b=0.0, c=0.0, e=0.0), top_k)


def test_grow_topk_vocab_smaller_than_k():
    L = _sharp_logits(2, 3, 16, seed=5, dtype="f32")
    top = _check_topk(L, np.arange(2), np.zeros(2), 8, COST, 32)
    assert (top[..., 16:] == -1).all()


def test_grow_topk_rejects_bad_k():
    L = _sharp_logits(1, 2, 64, seed=6).to(DEV)
    a = torch.zeros(1, dtype=torch.int32, device=DEV)
    c = torch.zeros(1, dtype=torch.int64, device=DEV)
    for k in (0, 33):
        with pytest.raises(pct.PctError):
            pct.cadd_tree_grow(L, a, c, 8, **COST,
                               top_tok=torch.zeros((1, 2, k), dtype=torch.int32, device=DEV))


# ---------------------------------------------------------------------------
def _unseeded_and_seeded(L, anchor, E, W, k, beam, N, seeds, transposed=False):
    args = (L.to(DEV), anchor.to(DEV), E.to(DEV), W.to(DEV), k, beam, N)
    plain = pct.pct_tree_build(*args)
    Wt = pct.markov_transpose(args[3]) if transposed else None
    seeded, names = _kernels_of(lambda: pct.pct_tree_build(*args, seeds=seeds.to(DEV), Wt=Wt))
    return plain, seeded, names


def _cadd_seeds(L, k):
    """Seeds as the round makes them: cadd_tree_grow_topk on the same logits."""
    batch = L.shape[0]
    _, _, top = _grow_both(L, np.zeros(batch), np.full(batch, 4096), 256, COST, k)
    return torch.as_tensor(top)


def _odd_seeds(batch, D, k, V, seed):
    """Columns outside [0, V), repeats and -1 among in-range columns."""
    g = torch.Generator().manual_seed(seed)
    s = torch.randint(-3, V + 3, (batch, D, k), generator=g, dtype=torch.int32)
    s[..., 1] = s[..., 0]
    s[0, 0, :] = -1
    return s


@pytest.mark.parametrize("kind", ["cadd", "cadd_wt", "odd", "odd_wt", "none"])
@pytest.mark.parametrize("V,D,r,k,beam,N,batch", [
    (4096, 5, 128, 8, 16, 64, 17),     # per-depth launches (more than 16 requests)
    (8192, 4, 96, 8, 24, 60, 2),       # the persistent small-frontier launch
])
def test_seeded_build_is_the_unseeded_build(kind, V, D, r, k, beam, N, batch):
    """_wt: the seeds' W columns read from markov_transpose(W) (r = 96: zero
    padding past r inside the transposed rows)."""
    L, anchor, E, W = _problem(batch, D, V, r, seed=V + D + batch)
    seeds = {"cadd": lambda: _cadd_seeds(L, k),
             "odd": lambda: _odd_seeds(batch, D, k, V, V),
             "none": lambda: torch.full((batch, D, k), -1, dtype=torch.int32)}[kind.split("_")[0]]()
    plain, seeded, names = _unseeded_and_seeded(L, anchor, E, W, k, beam, N, seeds,
                                                transposed=kind.endswith("_wt"))
    assert "seed_columns" in names and "drafter_topk" not in names, names
    torch.cuda.synchronize()
    _same_tree(plain, seeded)


@pytest.mark.parametrize("V,r", [(64, 1), (1000, 64), (4096, 100), (20488, 256), (151936, 256)])
def test_markov_transpose_layout(V, r):
    """Wt[v][j] = W[j][v] for j < r, zero for r <= j < r_pad (r rounded up to 64)."""
    g = torch.Generator().manual_seed(V + r)
    W = (torch.randn((r, V), generator=g)).to(torch.bfloat16).to(DEV)
    Wt = pct.markov_transpose(W)
    torch.cuda.synchronize()
    r_pad = (r + 63) // 64 * 64
    assert tuple(Wt.shape) == (V, r_pad)
    ref = torch.zeros((V, r_pad), dtype=torch.bfloat16, device=DEV)
    ref[:, :r] = W.t()
    assert torch.equal(Wt.view(torch.int16), ref.view(torch.int16))


def test_seeded_build_matches_oracle():
    L, anchor, E, W = _problem(17, 5, 4096, 100, seed=41)
    seeds = _cadd_seeds(L, 8)
    _build_and_compare(L, anchor, E, W, 8, 32, 128, label="seeded from cadd", seeds=seeds)


def test_seeded_build_f32_markov_ignores_seeds():
    L, anchor, E, W = _problem(3, 4, 1500, 24, seed=43, dtype="f32")
    plain, seeded, _ = _unseeded_and_seeded(L, anchor, E, W, 4, 8, 40,
                                            _odd_seeds(3, 4, 4, 1500, 44))
    _same_tree(plain, seeded)


def test_seeded_build_rejects_bad_seed_shape():
    L, anchor, E, W = _problem(2, 3, 1024, 64, seed=45)
    with pytest.raises(ValueError):
        pct.pct_tree_build(L.to(DEV), anchor.to(DEV), E.to(DEV), W.to(DEV), 8, 8, 20,
                           seeds=torch.zeros((2, 3, 4), dtype=torch.int32, device=DEV))


def test_full_round_one_pass_serves_both_trees():
    """The round's shapes: 64 requests, V = 151936, D = 15, k = 8. The CaDDTree
    on the drafter logits writes each row's top 8; seeded with them (W columns
    from W or from its transpose), the PCTree equals the unseeded build bit for
    bit; the top 8 of sampled rows equal the oracle's."""
    w, C = workloads.FULL_ROUND, workloads.CADDTREE
    d = workloads.drafter_inputs(w, device=DEV)
    L, anchor, E, W = d["L"], d["anchor"], d["E"], d["W"]
    batch, D, V = L.shape
    ctx = torch.tensor([C.ells[b % len(C.ells)] for b in range(batch)], dtype=torch.int64,
                       device=DEV)
    cost = dict(C_d=C.C_d, a=C.a, b=C.b, c=C.c, e=C.e)
    top = torch.empty((batch, D, w.k), dtype=torch.int32, device=DEV)
    withk = pct.cadd_tree_grow(L, anchor, ctx, C.n_max, **cost, top_tok=top)
    plain_c = pct.cadd_tree_grow(L, anchor, ctx, C.n_max, **cost)
    plain = pct.pct_tree_build(L, anchor, E, W, w.k, w.beam, w.n_nodes)
    seeded = pct.pct_tree_build(L, anchor, E, W, w.k, w.beam, w.n_nodes, seeds=top)
    seeded_t = pct.pct_tree_build(L, anchor, E, W, w.k, w.beam, w.n_nodes, seeds=top,
                                  Wt=pct.markov_transpose(W))
    torch.cuda.synchronize()
    _same_tree(plain_c, withk, phi=True)
    _same_tree(plain, seeded)
    _same_tree(plain, seeded_t)
    topn = host(top)
    rng = np.random.default_rng(7)
    for b, dd in zip(rng.integers(0, batch, 24), rng.integers(0, D, 24)):
        np.testing.assert_array_equal(topn[b, dd], oracle.row_topk(f64(L[b, dd].cpu()), w.k))


@pytest.mark.parametrize("V,top_k", [(20488, 1), (10240, 32), (10248, 16), (183520, 8)])
def test_grow_topk_segment_edges(V, top_k):
    """Segment boundaries (a last segment of one 16-byte group, exactly one full
    segment, eighteen segments) and the extreme top_k; every row of a flat batch
    (sigma 0.05, stop disabled) is left to the exact selection, in 16 parts at the
    largest V."""
    L = _sharp_logits(2, 3, V, seed=V % 89 + top_k, sigma=2.0, peak=(0.0, 6.0))
    _check_topk(L, np.arange(2), np.array([4096, 32768]), 64, COST, top_k)
    flat = _sharp_logits(2, 3, V, seed=V % 83, sigma=0.05, peak=(0.0, 0.1))
    _check_topk(flat, np.arange(2), np.zeros(2), 1, dict(C_d=1.0, a=1.0, b=0.0, c=0.0, e=0.0),
                top_k)


def test_grow_topk_repeated_calls_reuse_the_workspace():
    """The exact selection's counters and row list are reset by every call: ten
    calls on one workspace, alternating flat rows (every row left to the exact
    selection) and wide rows (none left)."""
    batch, D, V = 4, 5, 30000
    La = _sharp_logits(batch, D, V, seed=51, sigma=0.05, peak=(0.0, 0.5))
    Lb = _sharp_logits(batch, D, V, seed=52, sigma=2.0, peak=(0.0, 6.0))   # hundreds above θ
    a = torch.arange(batch, dtype=torch.int32, device=DEV)
    c = torch.full((batch,), 4096, dtype=torch.int64, device=DEV)
    cost = dict(C_d=1.0, a=1.0, b=0.0, c=1e-3, e=0.0)
    cdesc = pct.cadd_desc(batch, D, V, 32, pct.PCT_BF16, *cost.values())
    import ctypes
    ws = torch.empty(int(pct.lib().cadd_tree_grow_workspace(ctypes.byref(cdesc))), dtype=torch.uint8,
                     device=DEV)
    refs = {id(La): oracle.row_topk(f64(La), 8), id(Lb): oracle.row_topk(f64(Lb), 8)}
    Ld = {id(La): La.to(DEV), id(Lb): Lb.to(DEV)}
    for i in range(10):
        L = La if i % 2 == 0 else Lb
        top = torch.full((batch, D, 8), -7, dtype=torch.int32, device=DEV)
        pct.cadd_tree_grow(Ld[id(L)], a, c, 32, **cost, workspace=ws, top_tok=top)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(top), refs[id(L)], err_msg=f"call {i}")


@pytest.mark.parametrize("k,beam,N", [(16, 32, 200), (1, 4, 7)])
def test_seeded_build_extreme_k(k, beam, N):
    """k = 16 (the largest: sixteen seed columns per row) and k = 1 (chains)."""
    L, anchor, E, W = _problem(17, 5, 4096, 64, seed=60 + k)
    seeds = _cadd_seeds(L, k)
    plain, seeded, names = _unseeded_and_seeded(L, anchor, E, W, k, beam, N, seeds,
                                                transposed=True)
    torch.cuda.synchronize()
    _same_tree(plain, seeded)
    _build_and_compare(L, anchor, E, W, k, beam, N, label=f"seeded k={k}", seeds=seeds)


def test_one_pass_round_in_a_cuda_graph():
    """cadd_tree_grow_topk forks its exact selection to the library's second
    stream and joins it back: captured in a graph with the seeded build, the
    replay gives the eager results bit for bit (new inputs copied in between)."""
    import ctypes
    batch, D, V, r, k = 17, 5, 4096, 64, 8
    L, anchor, E, W = _problem(batch, D, V, r, seed=71)
    L2, _, _, _ = _problem(batch, D, V, r, seed=72)
    Ld, ad, Ed, Wd = L.to(DEV), anchor.to(DEV), E.to(DEV), W.to(DEV)
    ctx = torch.full((batch,), 4096, dtype=torch.int64, device=DEV)
    Wt = pct.markov_transpose(Wd)
    top = torch.empty((batch, D, k), dtype=torch.int32, device=DEV)
    cdesc = pct.cadd_desc(batch, D, V, 64, pct.PCT_BF16, *COST.values())
    ws_c = torch.empty(int(pct.lib().cadd_tree_grow_workspace(ctypes.byref(cdesc))), dtype=torch.uint8,
                       device=DEV)
    bdesc = pct.build_desc(batch, D, V, r, k, 16, 64, pct.PCT_BF16, pct.PCT_BF16)
    ws_t = torch.empty(pct.pct_tree_build_workspace(bdesc), dtype=torch.uint8, device=DEV)
    cad = pct.cadd_tree_grow(Ld, ad, ctx, 64, **COST, workspace=ws_c, top_tok=top)
    tree = pct.pct_tree_build(Ld, ad, Ed, Wd, k, 16, 64, workspace=ws_t, seeds=top, Wt=Wt)
    torch.cuda.synchronize()

    def eager(Lx):
        t2 = torch.empty_like(top)
        c = pct.cadd_tree_grow(Lx.to(DEV), ad, ctx, 64, **COST, top_tok=t2)
        b = pct.pct_tree_build(Lx.to(DEV), ad, Ed, Wd, k, 16, 64, seeds=t2, Wt=Wt)
        torch.cuda.synchronize()
        return c, b, host(t2)

    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            pct.cadd_tree_grow(Ld, ad, ctx, 64, **COST, out=cad, workspace=ws_c, top_tok=top,
                               stream=s)
            pct.pct_tree_build(Ld, ad, Ed, Wd, k, 16, 64, out=tree, workspace=ws_t, seeds=top,
                               Wt=Wt, stream=s)
    for Lx in (L2, L):
        Ld.copy_(Lx.to(DEV))
        g.replay()
        torch.cuda.synchronize()
        c, b, t2 = eager(Lx)
        _same_tree(c, cad, phi=True)
        _same_tree(b, tree)
        np.testing.assert_array_equal(host(top), t2)


def test_grow_topk_from_two_host_threads():
    """Two host threads, each on its own stream and workspace, call
    cadd_tree_grow_topk at the same time (the second stream and its events are
    shared under a lock): every result equals the single-threaded one."""
    import threading
    batch, D, V = 6, 4, 20000
    Ls = [_sharp_logits(batch, D, V, seed=80 + i, sigma=0.05 if i % 2 else 2.0,
                        peak=(0.0, 0.5 if i % 2 else 6.0)) for i in range(2)]
    refs = [oracle.row_topk(f64(x), 8) for x in Ls]
    a = torch.arange(batch, dtype=torch.int32, device=DEV)
    c = torch.full((batch,), 4096, dtype=torch.int64, device=DEV)
    errors = []
    torch.cuda.synchronize()

    def work(i):
        try:
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                Ld = Ls[i].to(DEV)
                for _ in range(20):
                    top = torch.full((batch, D, 8), -7, dtype=torch.int32, device=DEV)
                    pct.cadd_tree_grow(Ld, a, c, 32, **COST, top_tok=top, stream=st)
                    st.synchronize()
                    np.testing.assert_array_equal(host(top), refs[i])
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append(e)

    th = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
