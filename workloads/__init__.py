"""Seeded synthetic inputs for the draft-tree hot path.

This module is shared by the CPU oracle, the GPU tests and the benchmark. It
only draws random numbers and lays them out; it holds none of the arithmetic of
the method (no softmax, no scoring, no selection, no verification). Both sides
of every parity check receive the very same tensors from here.

Workloads (sizes follow the hot path's five configurations):

* ``tiny``            V=1000, block B=7, fp32 drafter logits ~ N(0, 3) plus one
                      peaked token per position (+U[2, 10]), Markov rank 16 with
                      E, W ~ N(0, 0.1), k=4, beam 4, N=32, one request, seed 0.
* ``qwen3_4b_scale``  V=151936, B=7, bf16 logits ~ N(0, 2) + peak U[2, 10],
                      bf16 Markov rank 256 with E, W ~ N(0, 0.05), k=8,
                      beam 16, N=64, one request.
* ``long_block``      V=151936, B=16, as above with peak U[0, 6], k=8, beam 32,
                      N=128, 32 requests.
* ``caddtree``        per-position marginals only (no Markov), V=151936, B=16,
                      logits as ``long_block``, n_max=512, C_d=1, C_v(n; l) =
                      a + b l + c n + e n^2 with a=2, b=1e-4, c=5e-3, e=1e-5,
                      l in {512, 4096, 32768}, 64 requests.
* ``full_round``      PCTree build as ``long_block`` with N=256 and 64 requests,
                      then bf16 target logits [N][V] ~ N(0, 2) per request with
                      an argmax of 20.0 planted along a random root path whose
                      length is drawn from U{0..16}.

Reading adopted for "N(mu, x)": x is the standard deviation. A block of size B
has one anchor (depth 0) and D = B - 1 drafted depths.

Draw order from one ``torch.Generator`` seeded with the workload's seed:
anchors U{0..V-1} [batch]; drafter logits; peak token ids U{0..V-1}
[batch][D]; peak heights; E; W. Target logits and the planted path use a second
generator seeded with ``seed + 1000`` so that they can be drawn after the tree
they are planted on is known.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np
import torch

__all__ = [
    "PCTreeWorkload", "CaddWorkload", "WORKLOADS", "CADDTREE", "FULL_ROUND",
    "drafter_inputs", "cadd_inputs", "target_logits", "plant_path",
    "random_tree", "bf16_bits", "PLANT_VALUE",
]

PLANT_VALUE = 20.0


@dataclass(frozen=True)
class PCTreeWorkload:
    name: str
    vocab: int
    block: int                 # B: anchor + B-1 drafted positions
    rank: int                  # r of the low-rank Markov stand-in E[p] . W
    k: int                     # local top-k per parent
    beam: int                  # per-depth beam width
    n_nodes: int               # N, verification budget, root included
    batch: int
    dtype: str                 # "f32" or "bf16" for logits and Markov params
    sigma: float               # std of the drafter logits
    peak: tuple                # (lo, hi) of the uniform peak height
    ew_std: float              # std of E and W
    seed: int

    @property
    def depth(self) -> int:
        return self.block - 1


@dataclass(frozen=True)
class CaddWorkload:
    name: str
    vocab: int
    block: int
    n_max: int                 # node cap, root included
    batch: int
    dtype: str
    sigma: float
    peak: tuple
    C_d: float
    a: float
    b: float
    c: float
    e: float
    ells: tuple
    seed: int

    @property
    def depth(self) -> int:
        return self.block - 1


WORKLOADS = {
    "tiny": PCTreeWorkload("tiny", 1000, 7, 16, 4, 4, 32, 1, "f32", 3.0, (2.0, 10.0), 0.1, 0),
    "qwen3_4b_scale": PCTreeWorkload("qwen3_4b_scale", 151936, 7, 256, 8, 16, 64, 1, "bf16",
                                     2.0, (2.0, 10.0), 0.05, 1),
    "long_block": PCTreeWorkload("long_block", 151936, 16, 256, 8, 32, 128, 32, "bf16",
                                 2.0, (0.0, 6.0), 0.05, 2),
}
CADDTREE = CaddWorkload("caddtree", 151936, 16, 512, 64, "bf16", 2.0, (0.0, 6.0),
                        1.0, 2.0, 1e-4, 5e-3, 1e-5, (512, 4096, 32768), 3)
FULL_ROUND = PCTreeWorkload("full_round", 151936, 16, 256, 8, 32, 256, 64, "bf16",
                            2.0, (0.0, 6.0), 0.05, 4)
FULL_ROUND_TARGET_SIGMA = 2.0
FULL_ROUND_PLANT_LEN = (0, 16)


def _tdtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 tensor as a numpy uint16 array (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def drafter_inputs(w: PCTreeWorkload, device="cpu", batch: Optional[int] = None,
                   seed: Optional[int] = None, markov: bool = True):
    """Drafter logits L [batch][D][V], anchors [batch], E [V][r], W [r][V].

    The peak is added in fp32 to the fp32 normal draw and the sum is rounded
    once to the storage type (round to nearest even for bf16).
    """
    batch = w.batch if batch is None else batch
    seed = w.seed if seed is None else seed
    g = torch.Generator(device=device).manual_seed(seed)
    V, D = w.vocab, w.depth
    anchor = torch.randint(0, V, (batch,), generator=g, device=device, dtype=torch.int64)
    normal = []
    for b in range(batch):
        normal.append(torch.randn((D, V), generator=g, device=device, dtype=torch.float32))
    peak_tok = torch.randint(0, V, (batch, D), generator=g, device=device, dtype=torch.int64)
    lo, hi = w.peak
    peak_h = torch.rand((batch, D), generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo
    L = torch.empty((batch, D, V), dtype=_tdtype(w.dtype), device=device)
    for b in range(batch):
        x = normal[b] * w.sigma
        x.scatter_add_(1, peak_tok[b][:, None], peak_h[b][:, None])
        L[b] = x.to(L.dtype)
        normal[b] = None
    out = {"L": L, "anchor": anchor.to(torch.int32), "peak_tok": peak_tok.to(torch.int32)}
    if markov:
        E = torch.randn((V, w.rank), generator=g, device=device, dtype=torch.float32) * w.ew_std
        W = torch.randn((w.rank, V), generator=g, device=device, dtype=torch.float32) * w.ew_std
        out["E"] = E.to(_tdtype(w.dtype))
        out["W"] = W.to(_tdtype(w.dtype))
    return out


def cadd_inputs(w: CaddWorkload, ell: int, device="cpu", batch: Optional[int] = None,
                seed: Optional[int] = None):
    """Per-position marginal logits [batch][D][V], anchors and context lengths."""
    pw = PCTreeWorkload(w.name, w.vocab, w.block, 1, 1, 1, 2, w.batch, w.dtype,
                        w.sigma, w.peak, 0.0, w.seed)
    d = drafter_inputs(pw, device=device, batch=batch, seed=seed, markov=False)
    b = d["L"].shape[0]
    d["ctx_len"] = torch.full((b,), int(ell), dtype=torch.int64, device=device)
    return d


def target_logits(batch: int, n_stride: int, vocab: int, sigma: float, seed: int,
                  device="cpu", dtype="bf16"):
    """Target-model logits [batch][n_stride][V] ~ N(0, sigma), drawn per request."""
    g = torch.Generator(device=device).manual_seed(seed)
    T = torch.empty((batch, n_stride, vocab), dtype=_tdtype(dtype), device=device)
    for b in range(batch):
        x = torch.randn((n_stride, vocab), generator=g, device=device, dtype=torch.float32)
        T[b] = (x * sigma).to(T.dtype)
    return T


def _children(parent_row: np.ndarray, count: int):
    ch = [[] for _ in range(count)]
    for i in range(1, count):
        ch[int(parent_row[i])].append(i)
    return ch


def plant_path(T: torch.Tensor, tok: np.ndarray, parent: np.ndarray, count: np.ndarray,
               seed: int, length_range=FULL_ROUND_PLANT_LEN, value=PLANT_VALUE):
    """Plant a target argmax along a random root path of each request's tree.

    For request b: draw a length U{lo..hi}; walk from the root picking a uniform
    child at each step, for that many steps or until a leaf; at every node on
    the walk but the last, write ``value`` at the next node's token; at the last
    node write ``value`` at a uniformly drawn token that is no child's token.
    Returns (lengths walked, node ids on each walk, end tokens) as numpy arrays
    padded with -1. T is modified in place (any device).
    """
    g = torch.Generator().manual_seed(seed)
    batch, n_stride, V = T.shape
    lo, hi = length_range
    walked = np.zeros(batch, np.int32)
    paths = np.full((batch, hi), -1, np.int32)
    ends = np.zeros(batch, np.int32)
    for b in range(batch):
        cnt = int(count[b])
        ch = _children(parent[b], cnt)
        want = int(torch.randint(lo, hi + 1, (1,), generator=g))
        u, steps = 0, 0
        while steps < want and ch[u]:
            pick = int(torch.randint(0, len(ch[u]), (1,), generator=g))
            c = ch[u][pick]
            T[b, u, int(tok[b, c])] = value
            paths[b, steps] = c
            u, steps = c, steps + 1
        child_toks = {int(tok[b, c]) for c in ch[u]}
        for _ in range(1000):
            t = int(torch.randint(0, V, (1,), generator=g))
            if t not in child_toks:
                break
        T[b, u, t] = value
        walked[b], ends[b] = steps, t
    return walked, paths, ends


def random_tree(batch: int, n_stride: int, vocab: int, max_depth: int, seed: int,
                counts: Optional[Sequence[int]] = None):
    """Random trees in the node-table layout: parent[i] < i, distinct sibling tokens.

    Returns numpy int32 arrays tok, parent, depth [batch][n_stride] and count
    [batch]; slots at or beyond count hold -1.
    """
    rng = np.random.default_rng(seed)
    tok = np.full((batch, n_stride), -1, np.int32)
    par = np.full((batch, n_stride), -1, np.int32)
    dep = np.full((batch, n_stride), -1, np.int32)
    cnt = np.zeros(batch, np.int32)
    for b in range(batch):
        n = int(counts[b]) if counts is not None else int(rng.integers(1, n_stride + 1))
        cnt[b] = n
        tok[b, 0], dep[b, 0] = rng.integers(0, vocab), 0
        sib = {0: set()}
        for i in range(1, n):
            while True:
                p = int(rng.integers(0, i))
                if dep[b, p] < max_depth and len(sib[p]) < vocab:
                    break
            while True:
                t = int(rng.integers(0, vocab))
                if t not in sib[p]:
                    break
            sib[p].add(t)
            sib[i] = set()
            tok[b, i], par[b, i], dep[b, i] = t, p, dep[b, p] + 1
    return tok, par, dep, cnt
