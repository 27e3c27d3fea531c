"""Benchmark: draft-tree rounds/sec (build + verify) at V = 151936 on B200.

One step is one round of the whole hot path over a batch of 64 requests
(synthetic inputs resident in HBM when the timed region starts):
  * CaDDTree grow on the drafter logits (as marginals) with C_d = 1,
    C_v = 2 + 1e-4 l + 5e-3 n + 1e-5 n^2, n_max = 512, context lengths cycling
    through 512 / 4096 / 32768 over the requests; its row pass also writes each
    row's top 8 tokens (cadd_tree_grow_topk);
  * PCTree build on the same logits: V = 151936, B = 16 (D = 15), bf16 logits
    ~ N(0, 2) + peak U[0, 6], bf16 Markov rank 256, k = 8, beam 32, N = 256,
    its top-k gates seeded with those tokens (pct_tree_build_seeded), so the
    logits are streamed once for both trees;
  * ancestor mask of the PCTree trees (256 x 256 bits per request);
  * greedy verification against bf16 target logits [64][256][V] (4.98 GB), with
    an argmax planted along a random root path of each tree.
The 4.98 GB of target logits stream through L2 every step, so no step starts
with a warm L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0). For N > 1 (torchrun, one process per GPU) every
rank runs its own independent batch (weak scaling, no data-path collective);
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "draft-tree rounds/sec (build+verify) at V=151936; HBM GB/s vs roofline"
W = workloads.FULL_ROUND
C = workloads.CADDTREE
COST = dict(C_d=C.C_d, a=C.a, b=C.b, c=C.c, e=C.e)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def set_requests(n):
    """Use n requests per round instead of the workload's 64 (profiling captures only)."""
    global W
    import dataclasses
    W = dataclasses.replace(workloads.FULL_ROUND, batch=int(n))


def workload_config():
    return {
        "workload": "full_round: CaDDTree grow (n_max=512, l in {512,4096,32768}; also each "
                    "row's top 8) + PCTree build seeded with them (V=151936, B=16, r=256, k=8, "
                    "beam=32, N=256) + ancestor mask + greedy verify of bf16 target logits "
                    "[64][256][V]",
        "requests": W.batch, "vocab": W.vocab, "block": W.block, "rank": W.rank, "k": W.k,
        "beam": W.beam, "n_nodes": W.n_nodes, "cadd_n_max": C.n_max,
        "l2": "inputs larger than L2: 4.98 GB of target logits stream through L2 each step",
        "seed": W.seed,
    }


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# algorithmic work per step (counted from the method, not from the kernels)
def frontier_sizes():
    F = [1]
    for _ in range(W.depth):
        F.append(min(W.beam, F[-1] * W.k))
    return F


# The library scores depths of more than 128 parent rows with the CTA-pair
# kernel and smaller ones with the single-CTA kernel.
PAIR_ROWS_MIN = 129


def merge_bytes_per_step():
    """Algorithmic bytes of the per-depth beam merge over the round: per request
    and depth, the |F|k candidates (token, score: 8 B) read, the beam's
    (token, parent, score: 12 B) written, and the next depth's Markov operand
    rows (beam x r bf16) gathered and written."""
    F = frontier_sizes()
    tot = 0.0
    for d in range(1, W.depth + 1):
        c = F[d - 1] * W.k
        kept = F[d]
        tot += W.batch * (8.0 * c + 12.0 * kept + (4.0 * kept * W.rank if d < W.depth else 0.0))
    return tot


def algorithmic_work():
    F = frontier_sizes()
    rows = [W.batch * F[d - 1] for d in range(1, W.depth + 1)]
    flop = lambda ms: sum(2.0 * W.rank * W.vocab * m for m in ms)
    return {
        # tensor-core contraction E_g[M_d][r] . W[r][V] per depth, by the kernel that runs it
        "pct_score_pair": {"bound": "tensor", "flop": flop([m for m in rows if m >= PAIR_ROWS_MIN])},
        "pct_score_umma": {"bound": "tensor", "flop": flop([m for m in rows if m < PAIR_ROWS_MIN])},
        # every node row of target logits read once (bf16)
        "verify_argmax_walk": {"bound": "hbm", "bytes": float(W.batch * W.n_nodes * W.vocab * 2)},
        # every marginal row read once (bf16)
        "cadd_rowpass": {"bound": "hbm", "bytes": float(W.batch * W.depth * W.vocab * 2)},
        # admission seeds found by a pass over the drafter logits (the unseeded build)
        "drafter_topk": {"bound": "hbm", "bytes": float(W.batch * W.depth * W.vocab * 2)},
        # admission seeds from given columns: k rows of W's transpose (r bf16
        # values each, contiguous) per logits row read and written
        "seed_columns": {"bound": "latency",
                         "bytes": float(W.batch * W.depth * W.k * W.rank * 2 * 2)},
        # per-depth beam merge: a few KB per request and depth, bound by latency
        "pct_merge_beam": {"bound": "latency", "bytes": merge_bytes_per_step()},
    }


def source_sha(fname):
    p = os.path.join(ROOT, "speculative_decoding_draft_07_b200", "csrc", fname)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:12] if os.path.exists(p) else None


KERNEL_SOURCE = {"pct_score_pair": "pct_umma2.cu", "pct_score_umma": "pct_umma.cu",
                 "verify_argmax_walk": "verify.cu", "cadd_rowpass": "cadd.cu",
                 "drafter_topk": "pct_seed.cu", "pct_merge_beam": "pct_merge.cu",
                 "seed_columns": "pct_seed.cu"}


def ncu_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, if it matches the source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    want = source_sha(KERNEL_SOURCE.get(kernel, ""))
    for line in open(p):
        f = dict(x.split("=", 1) for x in line.split() if "=" in x)
        if f.get("kernel") == kernel and f.get("src_sha") == want:
            try:
                return float(f["bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock/throttle samples (every 200 ms) during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, ids):
        self.ids = ids
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.ids:
                cmd += ["-i", ",".join(self.ids)]
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def gpu_ids(dev):
    try:
        u = torch.cuda.get_device_properties(dev).uuid
        s = str(u)
        return ["GPU-" + s if not s.startswith("GPU-") else s]
    except Exception:
        return [str(dev.index or 0)]


# ---------------------------------------------------------------------------
class RoundInputs:
    """The round's seeded drafter inputs and context lengths (no library call)."""

    def __init__(self, dev, seed_offset=0):
        self.dev = dev
        d = workloads.drafter_inputs(W, device=dev, seed=W.seed + seed_offset)
        self.L, self.anchor, self.E, self.W = d["L"], d["anchor"], d["E"], d["W"]
        ells = np.array(C.ells)[np.arange(W.batch) % len(C.ells)]
        self.ctx = torch.as_tensor(ells, dtype=torch.int64, device=dev)


class Round(RoundInputs):
    """Inputs, outputs and workspaces of one round, all resident on one GPU."""

    def __init__(self, dev, seed_offset=0):
        import speculative_decoding_draft_07_b200 as pct
        super().__init__(dev, seed_offset)
        self.pct = pct
        # each row's top k from the CaDDTree's row pass seeds the PCTree's gates
        self.seeds = torch.empty((W.batch, W.depth, W.k), dtype=torch.int32, device=dev)
        # W transposed once (a model constant): the seeds' W columns are contiguous there
        self.Wt = pct.markov_transpose(self.W)
        self.cadd = pct.cadd_tree_grow(self.L, self.anchor, self.ctx, C.n_max, **COST,
                                       top_tok=self.seeds)
        self.tree = pct.pct_tree_build(self.L, self.anchor, self.E, self.W, W.k, W.beam, W.n_nodes,
                                       seeds=self.seeds, Wt=self.Wt)
        torch.cuda.synchronize(dev)
        # target logits planted along this batch's trees (drawn once, outside timing)
        self.T = workloads.target_logits(W.batch, W.n_nodes, W.vocab,
                                         workloads.FULL_ROUND_TARGET_SIGMA,
                                         seed=W.seed + seed_offset + 1000, device=dev)
        workloads.plant_path(self.T, self.tree.tok.cpu().numpy(), self.tree.parent.cpu().numpy(),
                             self.tree.count.cpu().numpy(), seed=W.seed + seed_offset + 1001)
        self.mask, self.mstat = pct.tree_ancestor_mask(self.tree.parent, self.tree.count)
        self.ver = pct.tree_verify_accept(self.tree.tok, self.tree.parent, self.tree.count, self.T,
                                          max_depth=W.depth)
        self.walk = pct.tree_verify_walk(self.tree.tok, self.tree.parent, self.tree.count, self.T,
                                         max_depth=W.depth)
        # preallocated workspaces so the timed region allocates nothing
        desc = pct.build_desc(W.batch, W.depth, W.vocab, W.rank, W.k, W.beam, W.n_nodes,
                              pct.PCT_BF16, pct.PCT_BF16)
        self.ws_tree = torch.empty(pct.pct_tree_build_workspace(desc), dtype=torch.uint8, device=dev)
        import ctypes
        cdesc = pct.cadd_desc(W.batch, W.depth, W.vocab, C.n_max, pct.PCT_BF16, *COST.values())
        self.ws_cadd = torch.empty(int(pct.lib().cadd_tree_grow_workspace(ctypes.byref(cdesc))),
                                   dtype=torch.uint8, device=dev)
        self.ws_ver = torch.empty(int(pct.lib().tree_verify_accept_workspace(W.batch, W.n_nodes)),
                                  dtype=torch.uint8, device=dev)
        torch.cuda.synchronize(dev)

    def step_lazy(self):
        """The same round with the lazy verification walk in place of the full
        argmax (identical acceptance; only the walked rows are read)."""
        pct = self.pct
        pct.cadd_tree_grow(self.L, self.anchor, self.ctx, C.n_max, **COST, out=self.cadd,
                           workspace=self.ws_cadd, top_tok=self.seeds)
        pct.pct_tree_build(self.L, self.anchor, self.E, self.W, W.k, W.beam, W.n_nodes,
                           out=self.tree, workspace=self.ws_tree, seeds=self.seeds, Wt=self.Wt)
        pct.tree_ancestor_mask(self.tree.parent, self.tree.count, mask=self.mask, status=self.mstat)
        pct.tree_verify_walk(self.tree.tok, self.tree.parent, self.tree.count, self.T,
                             max_depth=W.depth, out=self.walk)

    def step(self):
        pct = self.pct
        pct.cadd_tree_grow(self.L, self.anchor, self.ctx, C.n_max, **COST, out=self.cadd,
                           workspace=self.ws_cadd, top_tok=self.seeds)
        pct.pct_tree_build(self.L, self.anchor, self.E, self.W, W.k, W.beam, W.n_nodes,
                           out=self.tree, workspace=self.ws_tree, seeds=self.seeds, Wt=self.Wt)
        pct.tree_ancestor_mask(self.tree.parent, self.tree.count, mask=self.mask, status=self.mstat)
        pct.tree_verify_accept(self.tree.tok, self.tree.parent, self.tree.count, self.T,
                               max_depth=W.depth, out=self.ver, workspace=self.ws_ver)


def timed(fn, steps, dev):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize(dev)
    return s.elapsed_time(e)


def graph_step_ms(fn, steps, dev):
    """Milliseconds per step of fn captured once in a CUDA graph and replayed
    back to back (None if the capture fails)."""
    try:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize(dev)
        for _ in range(3):
            g.replay()
        ms = timed(g.replay, steps, dev) / steps
        del g
        return ms
    except Exception:
        torch.cuda.synchronize(dev)
        return None


def e2e_measure(rnd: Round, steps: int, dev):
    """Same metric through the public API with host buffers: every step copies its
    inputs from pinned host memory and reads its results back."""
    pct = rnd.pct
    hL = torch.empty(rnd.L.shape, dtype=rnd.L.dtype, pin_memory=True)
    hL.copy_(rnd.L)
    hT = torch.empty(rnd.T.shape, dtype=rnd.T.dtype, pin_memory=True)
    hT.copy_(rnd.T)
    ha = rnd.anchor.cpu().pin_memory()
    hc = rnd.ctx.cpu().pin_memory()
    outs = [rnd.tree.tok, rnd.tree.parent, rnd.tree.score, rnd.tree.count, rnd.cadd.tok,
            rnd.cadd.parent, rnd.cadd.count, rnd.cadd.phi, rnd.mask, rnd.ver.accept_len,
            rnd.ver.accept_path, rnd.ver.correction]
    houts = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    h2d = sum(t.numel() * t.element_size() for t in (hL, hT, ha, hc))
    d2h = sum(t.numel() * t.element_size() for t in houts)

    def one():
        rnd.L.copy_(hL, non_blocking=True)
        rnd.T.copy_(hT, non_blocking=True)
        rnd.anchor.copy_(ha, non_blocking=True)
        rnd.ctx.copy_(hc, non_blocking=True)
        rnd.step()
        for h, o in zip(houts, outs):
            h.copy_(o, non_blocking=True)

    one()
    ms = timed(one, steps, dev)
    del hL, hT
    return ms / steps, h2d, d2h


def host_cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def blas_threads(n):
    """Limit the BLAS pool of numpy to n threads inside the block (if possible)."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(n)
    except ImportError:  # pragma: no cover
        import contextlib
        return contextlib.nullcontext()


def oracle_requests(rnd: RoundInputs, req_ids, seed: int, threads: int):
    """The oracle, as it stands, on the given requests of the round: PCTree
    build, CaDDTree grow, mask and verify, one request per task over `threads`
    host threads (BLAS one thread each). Inputs are the round's drafter inputs;
    the target logits are drawn for these requests and planted along the
    ORACLE's own trees (untimed), so nothing comes from the GPU path.
    Returns (wall seconds, per-request PCTree results, per-request CaDDTree results)."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    E, Wm = oracle.to_f64(rnd.E), oracle.to_f64(rnd.W)
    Lh = rnd.L.cpu()
    anc = rnd.anchor.cpu().numpy()
    ctx = rnd.ctx.cpu().numpy()

    def build(b):
        Lb = oracle.to_f64(Lh[b:b + 1])
        ref = oracle.pct_tree_build(Lb, anc[b:b + 1], E, Wm, W.k, W.beam, W.n_nodes)
        cad = oracle.cadd_tree_grow(Lb, anc[b:b + 1], ctx[b:b + 1], C.n_max, **COST)
        oracle.tree_ancestor_mask(ref.parent, ref.count, W.n_nodes)
        return ref, cad

    with blas_threads(1), ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        built = list(ex.map(build, req_ids))
        t1 = time.perf_counter()
        Ts = []
        for j, (ref, _) in enumerate(built):       # untimed: targets along the oracle's trees
            T = workloads.target_logits(1, W.n_nodes, W.vocab, workloads.FULL_ROUND_TARGET_SIGMA,
                                        seed=seed + j)
            workloads.plant_path(T, ref.tok, ref.parent, ref.count, seed=seed + 500 + j)
            Ts.append(T)
        t2 = time.perf_counter()
        list(ex.map(lambda j: oracle.tree_verify_accept(built[j][0].tok, built[j][0].parent,
                                                         built[j][0].count, Ts[j],
                                                         max_depth=W.depth), range(len(built))))
        t3 = time.perf_counter()
    return (t1 - t0) + (t3 - t2), [b[0] for b in built], [b[1] for b in built]


def _gpu_paths(tok, par, n):
    paths, out = {0: ()}, set()
    for i in range(1, n):
        p = int(par[i])
        if p < 0 or p >= i:
            break
        paths[i] = paths[p] + (int(tok[i]),)
        out.add(paths[i])
    return out


def sample_parity(rnd, req_ids, refs, cads):
    """The GPU's trees of the sampled requests against the oracle's (untimed):
    node tables bit-exact, scores within 1e-4. A request the oracle marks as a
    near tie (two candidates closer than 1e-4 at a cut, so either order is
    correct) is compared against the oracle's tree with that tie resolved
    toward the GPU's nodes; `excluded` counts requests matched neither way."""
    import oracle
    E, Wm = oracle.to_f64(rnd.E), oracle.to_f64(rnd.W)
    Lh, anc, ctx = rnd.L.cpu(), rnd.anchor.cpu().numpy(), rnd.ctx.cpu().numpy()
    out = {}
    for name, gpu, res in (("pctree", rnd.tree, refs), ("caddtree", rnd.cadd, cads)):
        tok, par, sc, cnt = (t.cpu().numpy() for t in (gpu.tok, gpu.parent, gpu.score, gpu.count))

        def same(b, r):
            n = int(r.count[0])
            return bool(int(cnt[b]) == n and (tok[b] == r.tok[0]).all()
                        and (par[b] == r.parent[0]).all()
                        and np.abs(sc[b, :n] - r.score[0, :n]).max() <= 1e-4)

        exact = resolved = excluded = 0
        for b, r in zip(req_ids, res):
            if not r.excluded[0]:
                ok = same(b, r)
                exact += ok
                excluded += not ok
                continue
            paths = _gpu_paths(tok[b], par[b], int(cnt[b]))
            Lb = oracle.to_f64(Lh[b:b + 1])
            if name == "pctree":
                alt = oracle.pct_tree_build(Lb, anc[b:b + 1], E, Wm, W.k, W.beam, W.n_nodes,
                                            prefer=[paths])
            else:
                alt = oracle.cadd_tree_grow(Lb, anc[b:b + 1], ctx[b:b + 1], C.n_max, **COST,
                                            prefer=[(paths, int(cnt[b]))])
            ok = same(b, alt)
            resolved += ok
            excluded += not ok
        out[name] = {"requests": len(req_ids), "exact": exact, "near_tie_resolved": resolved,
                     "excluded": excluded}
    return out


def cpu_baseline(rnd: Round, n_multi: int = None):
    """The oracle on a bounded sample of the round, timed two ways on the host
    cores: one request on one thread, and one request per core on all cores."""
    cores = host_cores()
    n_multi = min(W.batch, cores) if n_multi is None else n_multi
    t1, _, _ = oracle_requests(rnd, [0], seed=W.seed + 7000, threads=1)
    ids = list(range(n_multi))
    tm, refs, cads = oracle_requests(rnd, ids, seed=W.seed + 7000, threads=cores)
    single = {"value": 1.0 / (t1 * W.batch), "unit": "rounds/s", "cores": 1,
              "sample": f"request 0 of the {W.batch}-request round on one thread "
                        f"({t1:.1f} s), scaled to the round"}
    line = {"value": n_multi / (tm * W.batch), "unit": "rounds/s", "cores": cores,
            "kind": "oracle",
            "sample": f"requests 0..{n_multi - 1} of the {W.batch}-request round (PCTree build, "
                      f"CaDDTree grow, mask, verify), one request per thread on {cores} host "
                      f"threads ({tm:.1f} s), scaled to the round; numpy float64",
            "single_thread": single}
    return line, sample_parity(rnd, ids, refs, cads)


def roofline_entry(name, launches, total_ms, steps, pk, pk_src, clocks=None):
    """One kernel's roofline: algorithmic work per launch over its mean launch time.

    Tensor-bound kernels are divided by the burst bf16 peak (the step runs for
    milliseconds at the sampled clock); the fraction of the sustained peak is
    given beside it. HBM-bound and latency-bound kernels are divided by the
    measured copy bandwidth."""
    work = algorithmic_work()[name]
    per_launch_ms = total_ms / max(launches, 1)
    per_step_launches = launches / steps
    extra = {}
    if work["bound"] == "tensor":
        units = work["flop"] / per_step_launches
        achieved = units / (per_launch_ms * 1e-3) / 1e12
        peak = float(pk.get("bf16_tflops", pk.get("bf16_tflops_sustained")))
        sus = float(pk.get("bf16_tflops_sustained", peak))
        extra = {"frac_of_sustained": round(achieved / sus, 4), "sustained_peak": sus}
        unit, src = "TFLOP/s", "burst bf16"
    else:
        units = work["bytes"] / per_step_launches
        achieved = units / (per_launch_ms * 1e-3) / 1e9
        peak = float(pk["hbm_gbs"])
        unit, src = "GB/s", "HBM copy"
    e = {"kernel": name, "bound": work["bound"], "achieved": round(achieved, 2),
         "peak": peak, "unit": unit, "frac": round(achieved / peak, 4),
         "peak_source": f"{pk_src} ({src})", "traffic": ncu_traffic(name),
         "launches_per_step": per_step_launches, "ms_per_launch": round(per_launch_ms, 4),
         "algorithmic_per_launch": units}
    e.update(extra)
    if clocks:
        e["sm_mhz"] = clocks.get("sm_mhz")
    return e


# ---------------------------------------------------------------------------
def rank_seed_offset(rank: int) -> int:
    """Seed offset of a rank's inputs: every rank draws its own batch of requests
    (weak scaling, no data-path collective)."""
    return 100 * rank


def max_over_ranks(x: float, dist=None, dev=None) -> float:
    """The slowest rank's value (device times are reported as the max over ranks)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, rank, world, budget_s: float = 150.0):
    """--impl reference: the CPU oracle on the same workload (rank 0 only).

    A step is a bounded sample of the round: one request per host core (cycling
    through the batch), every stage of the hot path, one request per thread.
    Steps run until K steps or about `budget_s` seconds, whichever comes first;
    the line reports the steps actually timed and the measured time per step."""
    if rank != 0:
        return 0
    if not torch.cuda.is_available():
        print(json.dumps({"impl": "reference", "unavailable": "no CUDA device to draw the inputs"}))
        return 0
    rnd = RoundInputs(torch.device("cuda", 0))
    cores = host_cores()
    per = min(cores, W.batch)
    times, spent = [], 0.0
    warm = min(args.warmup, 1)
    for i in range(warm + args.steps):
        ids = [(i * per + j) % W.batch for j in range(per)]
        dt, _, _ = oracle_requests(rnd, ids, seed=W.seed + 9000 + 100 * i, threads=cores)
        spent += dt
        if i >= warm:
            times.append(dt)
        if spent > budget_s and times:
            break
    ms = statistics.mean(times) * 1e3                     # one step: `per` requests
    value = per / (statistics.mean(times) * W.batch)      # 64-request rounds per second
    line = {"metric": METRIC, "value": value, "unit": "rounds/s", "n_gpus": 1,
            "steps": len(times), "steps_requested": args.steps, "warmup": warm,
            "ms_per_step": ms, "requests_per_step": per, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "rounds/s", "cores": cores, "kind": "oracle",
                             "sample": f"{per} of the {W.batch} requests per step, one per "
                                       f"thread on {cores} host threads, {len(times)} steps"},
            "e2e": {"value": value, "unit": "rounds/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


class L2Flush:
    """Writes a buffer twice the size of L2 between timed runs (untimed)."""

    def __init__(self, dev):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.zero_()


def warm_cold_ms(fn, dev, warm_runs, cold_runs, flush):
    """Mean milliseconds per run: back to back (warm: inputs that fit in L2 stay
    there) and with L2 flushed before every run (cold), each run bracketed by
    its own events on the launch stream."""
    fn()
    torch.cuda.synchronize(dev)
    warm = timed(fn, warm_runs, dev) / warm_runs
    tot = 0.0
    for _ in range(cold_runs):
        flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        e.synchronize()
        tot += s.elapsed_time(e)
    return warm, tot / cold_runs


def traced_kernels_us(fn, runs, dev):
    """Per-kernel device time of fn with L2 warm: two events around every launch
    on its stream (the library's trace), microseconds and launches per run."""
    import speculative_decoding_draft_07_b200 as pct
    pct.trace_enable(True)
    pct.trace_reset()
    for _ in range(runs):
        fn()
    torch.cuda.synchronize(dev)
    t = pct.trace_read()
    pct.trace_enable(False)
    return {n: {"launches": c / runs, "us": round(ms * 1e3 / runs, 2)} for n, (c, ms) in t.items()}


def oracle_legs(fn, batch):
    """The oracle on one request on one thread, and on min(batch, cores) requests
    one per thread on all host cores; rates scaled to the configuration's batch."""
    from concurrent.futures import ThreadPoolExecutor
    cores = host_cores()
    with blas_threads(1):
        t0 = time.perf_counter()
        fn(0)
        t1 = time.perf_counter() - t0
        n = min(batch, cores)
        with ThreadPoolExecutor(max_workers=n) as ex:
            t0 = time.perf_counter()
            list(ex.map(fn, range(n)))
            tm = time.perf_counter() - t0
    return {"single_thread": {"rounds_per_s": 1.0 / (t1 * batch), "cores": 1,
                              "sample": "1 request", "seconds": round(t1, 3)},
            "all_cores": {"rounds_per_s": n / (tm * batch), "cores": cores,
                          "sample": f"{n} requests, one per thread", "seconds": round(tm, 3)}}


def config_results(dev, pk, quick=False):
    """Every configuration of the hot path other than the full round: GPU rounds
    per second warm and cold (L2 flushed before every round), the dominant
    rate against its measured peak, and the oracle's rates (host cores)."""
    import oracle
    import speculative_decoding_draft_07_b200 as pct
    flush = L2Flush(dev)
    f64 = oracle.to_f64
    hbm, tc = float(pk["hbm_gbs"]), float(pk.get("bf16_tflops", pk.get("bf16_tflops_sustained")))
    res = {}
    for name in ("tiny", "qwen3_4b_scale", "long_block"):
        w = workloads.WORKLOADS[name]
        d = workloads.drafter_inputs(w, device=dev)
        L, a, E, Wm = d["L"], d["anchor"], d["E"], d["W"]
        out = pct.pct_tree_build(L, a, E, Wm, w.k, w.beam, w.n_nodes)
        ws = torch.empty(pct.pct_tree_build_workspace(pct.build_desc(
            w.batch, w.depth, w.vocab, w.rank, w.k, w.beam, w.n_nodes,
            pct.PCT_BF16 if L.dtype == torch.bfloat16 else pct.PCT_F32,
            pct.PCT_BF16 if E.dtype == torch.bfloat16 else pct.PCT_F32)), dtype=torch.uint8,
            device=dev)
        fn = lambda: pct.pct_tree_build(L, a, E, Wm, w.k, w.beam, w.n_nodes, out=out, workspace=ws)
        runs = 20 if name == "long_block" else 200
        warm, cold = warm_cold_ms(fn, dev, runs, max(runs // 4, 10), flush)
        F = [1]
        for _ in range(w.depth):
            F.append(min(w.beam, F[-1] * w.k))
        rows = sum(w.batch * F[i - 1] for i in range(1, w.depth + 1))
        flop = 2.0 * w.rank * w.vocab * rows
        esz = 2 if w.dtype == "bf16" else 4
        wbytes = float(w.depth * (w.rank * w.vocab + w.batch * w.vocab) * esz)   # W per depth + L
        e = {"workload": name, "requests": w.batch, "rounds_per_s_warm": 1e3 / warm,
             "rounds_per_s_cold": 1e3 / cold, "ms_per_round_cold": cold,
             "tflops_cold": flop / cold / 1e9, "frac_bf16_burst_cold": flop / cold / 1e9 / tc,
             "stream_gbs_cold": wbytes / cold / 1e6, "frac_hbm_cold": wbytes / cold / 1e6 / hbm,
             "stream_gbs_warm": wbytes / warm / 1e6,
             "bound": "tensor" if name == "long_block" else ("hbm" if name != "tiny" else "launch"),
             "kernels_warm": traced_kernels_us(fn, 10, dev)}
        if not quick:
            Lh, Eh, Wh, ah = L.cpu(), f64(E), f64(Wm), a.cpu().numpy()
            e["oracle"] = oracle_legs(lambda b: oracle.pct_tree_build(
                f64(Lh[b:b + 1]), ah[b:b + 1], Eh, Wh, w.k, w.beam, w.n_nodes), w.batch)
        res[name] = e
        del d, L, E, Wm, out, ws
    for ell in C.ells:
        d = workloads.cadd_inputs(C, ell, device=dev)
        L, a, ctx = d["L"], d["anchor"], d["ctx_len"]
        out = pct.cadd_tree_grow(L, a, ctx, C.n_max, **COST)
        fn = lambda: pct.cadd_tree_grow(L, a, ctx, C.n_max, **COST, out=out)
        warm, cold = warm_cold_ms(fn, dev, 100, 25, flush)
        nbytes = float(L.numel() * L.element_size())
        e = {"workload": f"caddtree_l{ell}", "requests": C.batch, "rounds_per_s_warm": 1e3 / warm,
             "rounds_per_s_cold": 1e3 / cold, "ms_per_round_cold": cold,
             "gbs_cold": nbytes / cold / 1e6, "frac_hbm_cold": nbytes / cold / 1e6 / hbm,
             "mean_nodes": float(out.count.float().mean()), "bound": "hbm",
             "kernels_warm": traced_kernels_us(fn, 10, dev)}
        if not quick:
            Lh, ah, ch = L.cpu(), a.cpu().numpy(), ctx.cpu().numpy()
            e["oracle"] = oracle_legs(lambda b: oracle.cadd_tree_grow(
                f64(Lh[b:b + 1]), ah[b:b + 1], ch[b:b + 1], C.n_max, **COST), C.batch)
        res[f"caddtree_l{ell}"] = e
        del d, L, out
    del flush
    torch.cuda.empty_cache()
    return {k: {kk: (round(vv, 6) if isinstance(vv, float) else vv) for kk, vv in v.items()}
            for k, v in res.items()}


def run_configs(args):
    """--configs: one line per configuration (not the default bench line)."""
    dev = torch.device("cuda", 0)
    pk, _ = peaks()
    for name, e in config_results(dev, pk).items():
        print(json.dumps(e))
    return 0


def run_stage(args):
    """One stage of the round, repeated, with only its own inputs on the device
    (the drafter logits and Markov parameters: about 0.45 GB), so that ncu
    captures of its kernels stay small."""
    import speculative_decoding_draft_07_b200 as pct
    dev = torch.device("cuda", 0)
    rnd = RoundInputs(dev)
    # as in the round: the CaDDTree's row pass writes each row's top k, which
    # seed the PCTree (W's transpose for their columns)
    seeds = torch.empty((W.batch, W.depth, W.k), dtype=torch.int32, device=dev)
    pct.cadd_tree_grow(rnd.L, rnd.anchor, rnd.ctx, C.n_max, **COST, top_tok=seeds)
    Wt = pct.markov_transpose(rnd.W)
    for _ in range(args.warmup + args.steps):
        if args.profile_stage == "pctree":
            out = pct.pct_tree_build(rnd.L, rnd.anchor, rnd.E, rnd.W, W.k, W.beam, W.n_nodes,
                                     seeds=seeds, Wt=Wt)
        else:
            out = pct.cadd_tree_grow(rnd.L, rnd.anchor, rnd.ctx, C.n_max, **COST, top_tok=seeds)
    torch.cuda.synchronize(dev)
    print(f"{args.profile_stage}: {args.warmup + args.steps} runs, status "
          f"{int(out.status.abs().sum().item())}, nodes {int(out.count.sum().item())}")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="leave the per-configuration results out of the bench line")
    ap.add_argument("--requests", type=int, default=W.batch,
                    help="requests per round (smaller only for profiling captures)")
    ap.add_argument("--profile-stage", default=None, choices=["pctree", "cadd"],
                    help="for profiler captures: run only this stage of the round on its "
                         "inputs, --warmup + --steps times, and print no bench line")
    ap.add_argument("--configs", action="store_true",
                    help="time every configuration of the hot path (one line each) instead of "
                         "the full round")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    set_requests(args.requests)
    if args.profile_stage is not None:
        return run_stage(args)
    if args.configs:
        return run_configs(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        import datetime
        dist = dist_mod
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import speculative_decoding_draft_07_b200 as pct
    pct.lib()

    rnd = Round(dev, seed_offset=rank_seed_offset(rank))
    for _ in range(args.warmup):
        rnd.step()
    torch.cuda.synchronize(dev)

    # timed region: the rounds back to back on the launch stream, clocks sampled alongside
    sampler = ClockSampler(gpu_ids(dev))
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.cudart().cudaProfilerStart()   # a profiler started with capture off records only this
    ms = timed(rnd.step, args.steps, dev)
    torch.cuda.cudart().cudaProfilerStop()
    # the same rounds again with every kernel bracketed by two events on its
    # stream: the per-kernel durations of the rooflines (the events lengthen
    # the round, so the headline comes from the region above)
    pct.trace_enable(True)
    pct.trace_reset()
    if dist is not None:
        dist.barrier()
    ms_traced = timed(rnd.step, args.steps, dev)
    clocks = sampler.stop()
    kernels = pct.trace_read()
    pct.trace_enable(False)
    ms = max_over_ranks(ms, dist, dev)
    ms_traced = max_over_ranks(ms_traced, dist, dev)
    ms_step = ms / args.steps
    value = world * 1e3 / ms_step
    graph_ms = graph_step_ms(rnd.step, args.steps, dev)
    if graph_ms is not None:
        graph_ms = max_over_ranks(graph_ms, dist, dev)

    # the same round with the lazy verification walk (argmax of the walked rows only)
    for _ in range(3):
        rnd.step_lazy()
    if dist is not None:
        dist.barrier()
    ms_lazy = max_over_ranks(timed(rnd.step_lazy, args.steps, dev), dist, dev) / args.steps
    pct.trace_enable(True)
    pct.trace_reset()
    if dist is not None:
        dist.barrier()
    timed(rnd.step_lazy, args.steps, dev)
    kl = pct.trace_read()
    pct.trace_enable(False)
    walked_rows = int((rnd.walk.accept_len.to(torch.int64) + 1).sum().item())

    # end-to-end through the public API with host buffers
    e2e_ms, h2d, d2h = e2e_measure(rnd, args.e2e_steps, dev)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)

    if rank == 0:
        pk, pk_src = peaks()
        launches = sum(v[0] for v in kernels.values())
        roofs = [roofline_entry(n, kernels[n][0], kernels[n][1], args.steps, pk, pk_src, clocks)
                 for n in algorithmic_work() if n in kernels]
        dominant = max(kernels, key=lambda n: kernels[n][1]) if kernels else None
        main_roof = next((r for r in roofs if r["kernel"] == dominant), roofs[0] if roofs else None)
        line = {
            "metric": METRIC, "value": value, "unit": "rounds/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(),
            "request_rounds_per_s": value * W.batch,
            "roofline": main_roof, "rooflines": roofs,
            "kernels": {n: {"launches_per_step": c / args.steps, "ms_per_step": t / args.steps}
                        for n, (c, t) in kernels.items()},
            "gpu_launches": launches,
            "traced_ms_per_step": ms_traced / args.steps,
            "cuda_graph": None if graph_ms is None else {
                "value": world * 1e3 / graph_ms, "unit": "rounds/s", "ms_per_step": graph_ms,
                "note": "the same round captured once in a CUDA graph and replayed"},
            "clocks": clocks,
            "e2e": {"value": world * 1e3 / e2e_ms, "unit": "rounds/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
        }
        wl = kl.get("verify_walk", (1, 0.0))
        walk_bytes = float(walked_rows * W.vocab * 2)
        line["lazy_verify"] = {
            "value": world * 1e3 / ms_lazy, "unit": "rounds/s", "ms_per_step": ms_lazy,
            "note": "the round with tree_verify_walk in place of the full argmax: same "
                    "acceptance, only the rows the walk reaches are read",
            "verify_walk_ms_per_step": wl[1] / args.steps,
            "walked_rows_per_step": walked_rows, "bytes_read_per_step": walk_bytes,
            "walk_gbs": walk_bytes / (wl[1] / args.steps * 1e-3) / 1e9 if wl[1] > 0 else None,
            "full_argmax_bytes_per_step": algorithmic_work()["verify_argmax_walk"]["bytes"]}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"], line["parity_sample"] = cpu_baseline(rnd)
            line["excluded"] = line["parity_sample"]["pctree"]["excluded"] + \
                line["parity_sample"]["caddtree"]["excluded"]
        if world == 1 and not args.no_configs:
            line["configs"] = config_results(dev, pk)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
