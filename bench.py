"""Benchmark: draft-tree rounds/sec (build + verify) at V = 151936 on B200.

One step is one round of the whole hot path over a batch of 64 requests
(synthetic inputs resident in HBM when the timed region starts):
  * PCTree build: V = 151936, B = 16 (D = 15), bf16 logits ~ N(0, 2) + peak
    U[0, 6], bf16 Markov rank 256, k = 8, beam 32, N = 256;
  * CaDDTree grow on the same drafter logits (as marginals) with C_d = 1,
    C_v = 2 + 1e-4 l + 5e-3 n + 1e-5 n^2, n_max = 512, context lengths cycling
    through 512 / 4096 / 32768 over the requests;
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
        "workload": "full_round: PCTree build (V=151936, B=16, r=256, k=8, beam=32, N=256) + "
                    "CaDDTree grow (n_max=512, l in {512,4096,32768}) + ancestor mask + "
                    "greedy verify of bf16 target logits [64][256][V]",
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
    }


def source_sha(fname):
    p = os.path.join(ROOT, "speculative_decoding_draft_07_b200", "csrc", fname)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:12] if os.path.exists(p) else None


KERNEL_SOURCE = {"pct_score_pair": "pct_umma2.cu", "pct_score_umma": "pct_umma.cu",
                 "verify_argmax_walk": "verify.cu",
                 "cadd_rowpass": "cadd.cu"}


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
        self.tree = pct.pct_tree_build(self.L, self.anchor, self.E, self.W, W.k, W.beam, W.n_nodes)
        self.cadd = pct.cadd_tree_grow(self.L, self.anchor, self.ctx, C.n_max, **COST)
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

    def step(self):
        pct = self.pct
        pct.pct_tree_build(self.L, self.anchor, self.E, self.W, W.k, W.beam, W.n_nodes,
                           out=self.tree, workspace=self.ws_tree)
        pct.cadd_tree_grow(self.L, self.anchor, self.ctx, C.n_max, **COST, out=self.cadd,
                           workspace=self.ws_cadd)
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


def oracle_round_sample(rnd: RoundInputs, req_ids, seed: int):
    """Seconds the oracle, as it stands, spends on the given requests of the
    round: PCTree build, CaDDTree grow, mask and verify. Inputs are the round's
    drafter inputs; the target logits are drawn for these requests and planted
    along the ORACLE's own trees (untimed), so nothing comes from the GPU path."""
    import oracle
    L = oracle.to_f64(rnd.L[req_ids])
    E, Wm = oracle.to_f64(rnd.E), oracle.to_f64(rnd.W)
    anc = rnd.anchor.cpu().numpy()[req_ids]
    ctx = rnd.ctx.cpu().numpy()[req_ids]
    t0 = time.perf_counter()
    ref = oracle.pct_tree_build(L, anc, E, Wm, W.k, W.beam, W.n_nodes)
    oracle.cadd_tree_grow(L, anc, ctx, C.n_max, **COST)
    oracle.tree_ancestor_mask(ref.parent, ref.count, W.n_nodes)
    t1 = time.perf_counter()
    T = workloads.target_logits(len(req_ids), W.n_nodes, W.vocab,
                                workloads.FULL_ROUND_TARGET_SIGMA, seed=seed)
    workloads.plant_path(T, ref.tok, ref.parent, ref.count, seed=seed + 1)
    t2 = time.perf_counter()
    oracle.tree_verify_accept(ref.tok, ref.parent, ref.count, T, max_depth=W.depth)
    t3 = time.perf_counter()
    return (t1 - t0) + (t3 - t2)


def host_cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def cpu_baseline(rnd: Round, n_req: int = 1):
    """The oracle on a bounded sample: n_req requests of the round."""
    dt = oracle_round_sample(rnd, list(range(n_req)), seed=W.seed + 7000)
    per_round = dt * W.batch / n_req
    return {"value": 1.0 / per_round, "unit": "rounds/s", "cores": host_cores(), "kind": "oracle",
            "sample": f"{n_req} of {W.batch} requests of one round (PCTree build, CaDDTree grow, "
                      f"mask, verify), scaled to the {W.batch}-request round; {dt:.1f} s of CPU "
                      "time; numpy float64, BLAS threads for the Markov matmul"}


def roofline_entry(name, kinfo, launches, total_ms, steps, pk, pk_src):
    work = algorithmic_work()[name]
    per_launch_ms = total_ms / max(launches, 1)
    per_step_launches = launches / steps
    if work["bound"] == "tensor":
        units = work["flop"] / per_step_launches
        achieved = units / (per_launch_ms * 1e-3) / 1e12
        peak = float(pk.get("bf16_tflops_sustained", pk.get("bf16_tflops")))
        unit = "TFLOP/s"
    else:
        units = work["bytes"] / per_step_launches
        achieved = units / (per_launch_ms * 1e-3) / 1e9
        peak = float(pk["hbm_gbs"])
        unit = "GB/s"
    return {"kernel": name, "bound": work["bound"], "achieved": round(achieved, 2),
            "peak": peak, "unit": unit, "frac": round(achieved / peak, 4),
            "peak_source": f"{pk_src} ({'sustained bf16' if unit == 'TFLOP/s' else 'HBM copy'})",
            "traffic": ncu_traffic(name), "launches_per_step": per_step_launches,
            "ms_per_launch": round(per_launch_ms, 4),
            "algorithmic_per_launch": units}


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


def run_reference(args, rank, world, budget_s: float = 120.0):
    """--impl reference: the CPU oracle on the same workload (rank 0 only).

    Each step is a bounded sample of the round: one request (cycling through the
    batch), all of its hot-path stages. Steps run until K steps or about
    `budget_s` seconds of oracle time, whichever comes first; the line reports
    the steps actually timed."""
    if rank != 0:
        return 0
    if not torch.cuda.is_available():
        print(json.dumps({"impl": "reference", "unavailable": "no CUDA device to draw the inputs"}))
        return 0
    rnd = RoundInputs(torch.device("cuda", 0))
    times, spent = [], 0.0
    warm = min(args.warmup, 1)
    for i in range(warm + args.steps):
        dt = oracle_round_sample(rnd, [i % W.batch], seed=W.seed + 9000 + i)
        spent += dt
        if i >= warm:
            times.append(dt)
        if spent > budget_s and times:
            break
    ms = statistics.mean(times) * W.batch * 1e3          # one 64-request round
    value = 1e3 / ms
    line = {"metric": METRIC, "value": value, "unit": "rounds/s", "n_gpus": 1,
            "steps": len(times), "steps_requested": args.steps, "warmup": warm,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_config(),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "rounds/s", "cores": host_cores(),
                             "kind": "oracle",
                             "sample": f"one request of the {W.batch}-request round per step, "
                                       f"{len(times)} steps, scaled to the round"},
            "e2e": {"value": value, "unit": "rounds/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_configs(args):
    """One line per configuration of the hot path (not the default bench line):
    GPU rounds/s over --steps timed runs after --warmup, the dominant kernel's
    rate against the measured peak, and the oracle timed on one request of the
    same inputs (host cores), scaled to the configuration's batch."""
    import oracle
    import speculative_decoding_draft_07_b200 as pct
    dev = torch.device("cuda", 0)
    pk, pk_src = peaks()
    f64 = lambda t: t.detach().cpu().double().numpy() if t.dtype != torch.bfloat16 else \
        t.detach().cpu().float().double().numpy()
    lines = []

    def gpu_rate(fn):
        for _ in range(args.warmup):
            fn()
        return args.steps / (timed(fn, args.steps, dev) / 1e3)

    def oracle_requests_per_s(fn):   # the oracle on one request
        t0 = time.perf_counter()
        fn()
        return 1.0 / (time.perf_counter() - t0)

    for name in ("tiny", "qwen3_4b_scale", "long_block"):
        w = workloads.WORKLOADS[name]
        d = workloads.drafter_inputs(w, device=dev)
        L, a, E, Wm = d["L"], d["anchor"], d["E"], d["W"]
        r = gpu_rate(lambda: pct.pct_tree_build(L, a, E, Wm, w.k, w.beam, w.n_nodes))
        F = [1]
        for _ in range(w.depth):
            F.append(min(w.beam, F[-1] * w.k))
        rows = sum(w.batch * F[d_ - 1] for d_ in range(1, w.depth + 1))
        flop = 2.0 * w.rank * w.vocab * rows
        wbytes = float(w.rank * w.vocab * (2 if w.dtype == "bf16" else 4) * w.depth)
        o_rate = oracle_requests_per_s(lambda: oracle.pct_tree_build(
            f64(L[:1]), a[:1].cpu().numpy(), f64(E), f64(Wm), w.k, w.beam, w.n_nodes))
        lines.append({"config": name, "rounds_per_s": r, "requests": w.batch,
                      "tflops": flop * r / 1e12, "frac_bf16_sustained": flop * r / 1e12 /
                      float(pk["bf16_tflops_sustained"]),
                      "w_stream_gbs": wbytes * r / 1e9,
                      "frac_hbm": wbytes * r / 1e9 / float(pk["hbm_gbs"]),
                      "oracle_rounds_per_s": o_rate / w.batch, "oracle_sample": "1 request"})
    for ell in C.ells:
        d = workloads.cadd_inputs(C, ell, device=dev)
        L, a, ctx = d["L"], d["anchor"], d["ctx_len"]
        r = gpu_rate(lambda: pct.cadd_tree_grow(L, a, ctx, C.n_max, **COST))
        nbytes = float(L.numel() * L.element_size())
        o_rate = oracle_requests_per_s(lambda: oracle.cadd_tree_grow(
            f64(L[:1]), a[:1].cpu().numpy(), ctx[:1].cpu().numpy(), C.n_max, **COST))
        lines.append({"config": f"caddtree_l{ell}", "rounds_per_s": r, "requests": C.batch,
                      "gbs": nbytes * r / 1e9, "frac_hbm": nbytes * r / 1e9 / float(pk["hbm_gbs"]),
                      "oracle_rounds_per_s": o_rate / C.batch, "oracle_sample": "1 request"})
    for ln in lines:
        print(json.dumps({k: (round(v, 6) if isinstance(v, float) else v) for k, v in ln.items()}))
    return 0


def run_stage(args):
    """One stage of the round, repeated, with only its own inputs on the device
    (the drafter logits and Markov parameters: about 0.45 GB), so that ncu
    captures of its kernels stay small."""
    import speculative_decoding_draft_07_b200 as pct
    dev = torch.device("cuda", 0)
    rnd = RoundInputs(dev)
    for _ in range(args.warmup + args.steps):
        if args.profile_stage == "pctree":
            out = pct.pct_tree_build(rnd.L, rnd.anchor, rnd.E, rnd.W, W.k, W.beam, W.n_nodes)
        else:
            out = pct.cadd_tree_grow(rnd.L, rnd.anchor, rnd.ctx, C.n_max, **COST)
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

    # timed region: per-kernel events on the launch stream, clocks sampled alongside
    pct.trace_enable(True)
    pct.trace_reset()
    sampler = ClockSampler(gpu_ids(dev))
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    ms = timed(rnd.step, args.steps, dev)
    clocks = sampler.stop()
    kernels = pct.trace_read()
    pct.trace_enable(False)
    ms = max_over_ranks(ms, dist, dev)
    ms_step = ms / args.steps
    value = world * 1e3 / ms_step

    # end-to-end through the public API with host buffers
    e2e_ms, h2d, d2h = e2e_measure(rnd, args.e2e_steps, dev)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)

    if rank == 0:
        pk, pk_src = peaks()
        launches = sum(v[0] for v in kernels.values())
        roofs = [roofline_entry(n, None, kernels[n][0], kernels[n][1], args.steps, pk, pk_src)
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
            "clocks": clocks,
            "e2e": {"value": world * 1e3 / e2e_ms, "unit": "rounds/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(rnd, n_req=2)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
