"""ctypes binding of libpctree.so (argument marshalling only).

Every step of the hot path runs in the library's CUDA kernels; this module only
checks shapes, allocates outputs and workspace with torch on the inputs' device,
and passes raw pointers plus the current CUDA stream. If the shared library is
missing it raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpctree.so")

PCT_OK, PCT_EINVAL, PCT_EWORKSPACE, PCT_ECUDA, PCT_EDEVICE, PCT_ETIMEOUT, PCT_EUNSUPPORTED = range(7)
PCT_F32, PCT_BF16 = 0, 1
DEV_BAD_PARENT, DEV_BAD_TOKEN, DEV_BAD_COUNT, DEV_DEPTH_OVERFLOW, DEV_BAD_COST, DEV_TIMEOUT = (
    1, 2, 4, 8, 16, 32)
_NAMES = {0: "PCT_OK", 1: "PCT_EINVAL", 2: "PCT_EWORKSPACE", 3: "PCT_ECUDA", 4: "PCT_EDEVICE",
          5: "PCT_ETIMEOUT", 6: "PCT_EUNSUPPORTED"}

EXPORTED = [
    "pct_tree_build_workspace", "pct_tree_build", "pct_score_parents_workspace",
    "pct_score_parents", "cadd_tree_grow_workspace", "cadd_tree_grow", "tree_ancestor_mask",
    "tree_verify_accept_workspace", "tree_verify_accept", "pct_trace_enable", "pct_trace_reset",
    "pct_trace_read", "pct_version", "tree_verify_accept_noalloc", "tree_verify_walk",
    "tree_accept_sim",
    "cadd_cost_fit", "pct_tree_build_seeded", "cadd_tree_grow_topk", "pct_markov_rank_pad",
    "pct_markov_transpose",
]


class PctError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what} returned {_NAMES.get(code, code)}")
        self.code = code


class BuildDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("depth", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("k", ctypes.c_int32), ("beam", ctypes.c_int32),
                ("n_nodes", ctypes.c_int32), ("logits_dtype", ctypes.c_int32),
                ("markov_dtype", ctypes.c_int32)]


class CaddDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("depth", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("n_max", ctypes.c_int32), ("logits_dtype", ctypes.c_int32),
                ("C_d", ctypes.c_float), ("a", ctypes.c_float), ("b", ctypes.c_float),
                ("c", ctypes.c_float), ("e", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libpctree.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m speculative_decoding_draft_07_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    bd, cd = ctypes.POINTER(BuildDesc), ctypes.POINTER(CaddDesc)
    sig = {
        "pct_tree_build_workspace": (sz, [bd]),
        "pct_tree_build": (i32, [bd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "pct_score_parents_workspace": (sz, [bd, i32]),
        "pct_score_parents": (i32, [bd, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "cadd_tree_grow_workspace": (sz, [cd]),
        "cadd_tree_grow": (i32, [cd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "tree_ancestor_mask": (i32, [i32, i32, vp, vp, vp, vp, vp]),
        "tree_verify_accept_workspace": (sz, [i32, i32]),
        "tree_verify_accept": (i32, [i32, i32, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp, vp,
                                     vp, vp, sz, vp]),
        "pct_trace_enable": (i32, [i32]),
        "pct_trace_reset": (i32, []),
        "pct_trace_read": (i32, [ctypes.c_char_p, i32, vp, vp, i32]),
        "pct_version": (ctypes.c_char_p, []),
        "tree_verify_accept_noalloc": (i32, [i32, i32, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp,
                                             vp, vp, vp]),
        "tree_verify_walk": (i32, [i32, i32, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]),
        "tree_accept_sim": (i32, [i32, i32, i32, vp, vp, vp, ctypes.c_int64, ctypes.c_uint64, vp,
                                  vp, vp]),
        "cadd_cost_fit": (i32, [ctypes.c_int64, vp, vp, vp, vp, vp, vp]),
        "pct_tree_build_seeded": (i32, [bd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        sz, vp]),
        "pct_markov_rank_pad": (i32, [i32]),
        "pct_markov_transpose": (i32, [i32, i32, vp, vp, vp]),
        "cadd_tree_grow_topk": (i32, [cd, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    _lib = L
    return L


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return PCT_BF16
    if t.dtype == torch.float32:
        return PCT_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _check(t: torch.Tensor, name: str, dev: torch.device, shape=None, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _workspace(nbytes: int, dev, ws: Optional[torch.Tensor]):
    if nbytes == 0:
        return None, 0
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace has {ws.numel() * ws.element_size()} bytes, needs {nbytes}")
        return ws, ws.numel() * ws.element_size()
    return torch.empty(nbytes, dtype=torch.uint8, device=dev), nbytes


def _raise(code: int, what: str):
    if code != PCT_OK:
        raise PctError(code, what)


@dataclass
class TreeOut:
    tok: torch.Tensor
    parent: torch.Tensor
    depth: torch.Tensor
    score: torch.Tensor
    count: torch.Tensor
    status: torch.Tensor
    phi: Optional[torch.Tensor] = None


def build_desc(batch, depth, vocab, rank, k, beam, n_nodes, logits_dtype, markov_dtype) -> BuildDesc:
    return BuildDesc(batch, depth, vocab, rank, k, beam, n_nodes, logits_dtype, markov_dtype)


def pct_tree_build_workspace(desc: BuildDesc) -> int:
    return int(lib().pct_tree_build_workspace(ctypes.byref(desc)))


def pct_tree_build(L: torch.Tensor, anchor: torch.Tensor, E: torch.Tensor, W: torch.Tensor,
                   k: int, beam: int, n_nodes: int, out: Optional[TreeOut] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None,
                   seeds: Optional[torch.Tensor] = None,
                   Wt: Optional[torch.Tensor] = None) -> TreeOut:
    """PCTree for a batch of requests. L [batch][D][V], anchor [batch] int32,
    E [V][r], W [r][V]; returns node tables [batch][N] in canonical BFS order.
    seeds [batch][D][k] int32 (optional): the columns that seed each row's top-k
    gate (pct_tree_build_seeded), e.g. cadd_tree_grow's top_tok for the same L;
    the result does not depend on them. Wt (optional, with seeds):
    markov_transpose(W), read for the seeds' W columns."""
    dev = L.device
    batch, D, V = L.shape
    r = E.shape[1]
    _check(L, "L", dev)
    _check(anchor, "anchor", dev, (batch,), torch.int32)
    _check(E, "E", dev, (V, r))
    _check(W, "W", dev, (r, V), E.dtype)
    desc = build_desc(batch, D, V, r, k, beam, n_nodes, _code(L), _code(E))
    if out is None:
        out = TreeOut(*(torch.empty((batch, n_nodes), dtype=torch.int32, device=dev) for _ in range(3)),
                      torch.empty((batch, n_nodes), dtype=torch.float32, device=dev),
                      torch.empty(batch, dtype=torch.int32, device=dev),
                      torch.empty(batch, dtype=torch.int32, device=dev))
    nbytes = pct_tree_build_workspace(desc)
    if nbytes == 0:
        _raise(PCT_EINVAL, "pct_tree_build_workspace")
    ws, wsb = _workspace(nbytes, dev, workspace)
    if seeds is not None:
        _check(seeds, "seeds", dev, (batch, D, k), torch.int32)
        if Wt is not None:
            _check(Wt, "Wt", dev, (V, int(lib().pct_markov_rank_pad(r))), torch.bfloat16)
        code = lib().pct_tree_build_seeded(ctypes.byref(desc), _p(L), _p(anchor), _p(E), _p(W),
                                           _p(Wt), _p(seeds), _p(out.tok), _p(out.parent),
                                           _p(out.depth), _p(out.score), _p(out.count),
                                           _p(out.status), _p(ws), wsb, _stream(stream))
        _raise(code, "pct_tree_build_seeded")
        return out
    code = lib().pct_tree_build(ctypes.byref(desc), _p(L), _p(anchor), _p(E), _p(W), _p(out.tok),
                                _p(out.parent), _p(out.depth), _p(out.score), _p(out.count),
                                _p(out.status), _p(ws), wsb, _stream(stream))
    _raise(code, "pct_tree_build")
    return out


def markov_transpose(W: torch.Tensor, stream=None) -> torch.Tensor:
    """Wt [V][r_pad] bf16: W [r][V] bf16 transposed, zero past r (once per model)."""
    dev = W.device
    r, V = W.shape
    _check(W, "W", dev, dtype=torch.bfloat16)
    r_pad = int(lib().pct_markov_rank_pad(r))
    if r_pad == 0:
        _raise(PCT_EINVAL, "pct_markov_rank_pad")
    Wt = torch.empty((V, r_pad), dtype=torch.bfloat16, device=dev)
    _raise(lib().pct_markov_transpose(V, r, _p(W), _p(Wt), _stream(stream)), "pct_markov_transpose")
    return Wt


def pct_score_parents(L_row: torch.Tensor, parent_tok: torch.Tensor, E: torch.Tensor,
                      W: torch.Tensor, k: int, stream=None):
    """One depth of batched parent scoring: returns (lse [b][p], top_tok [b][p][k],
    top_logpi [b][p][k], status [b])."""
    dev = L_row.device
    batch, V = L_row.shape
    n_par = parent_tok.shape[1]
    r = E.shape[1]
    _check(L_row, "L_row", dev)
    _check(parent_tok, "parent_tok", dev, (batch, n_par), torch.int32)
    _check(E, "E", dev, (V, r))
    _check(W, "W", dev, (r, V), E.dtype)
    desc = build_desc(batch, 1, V, r, k, 1, 1, _code(L_row), _code(E))
    nbytes = int(lib().pct_score_parents_workspace(ctypes.byref(desc), n_par))
    if nbytes == 0:
        _raise(PCT_EINVAL, "pct_score_parents_workspace")
    ws, wsb = _workspace(nbytes, dev, None)
    lse = torch.empty((batch, n_par), dtype=torch.float32, device=dev)
    tt = torch.empty((batch, n_par, k), dtype=torch.int32, device=dev)
    tl = torch.empty((batch, n_par, k), dtype=torch.float32, device=dev)
    st = torch.empty(batch, dtype=torch.int32, device=dev)
    code = lib().pct_score_parents(ctypes.byref(desc), n_par, _p(L_row), _p(parent_tok), _p(E),
                                   _p(W), _p(lse), _p(tt), _p(tl), _p(st), _p(ws), wsb,
                                   _stream(stream))
    _raise(code, "pct_score_parents")
    return lse, tt, tl, st


def cadd_desc(batch, depth, vocab, n_max, logits_dtype, C_d, a, b, c, e) -> CaddDesc:
    return CaddDesc(batch, depth, vocab, n_max, logits_dtype, C_d, a, b, c, e)


def cadd_tree_grow(L: torch.Tensor, anchor: torch.Tensor, ctx_len: torch.Tensor, n_max: int,
                   C_d: float, a: float, b: float, c: float, e: float,
                   out: Optional[TreeOut] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None, top_tok: Optional[torch.Tensor] = None) -> TreeOut:
    """CaDDTree for a batch of requests. L [batch][D][V] marginal logits,
    anchor [batch] int32, ctx_len [batch] int64; node tables [batch][n_max].
    top_tok [batch][D][top_k] int32 (optional, top_k 1..32): also written with
    each row's top_k tokens by logit (value desc, token asc), cadd_tree_grow_topk."""
    dev = L.device
    batch, D, V = L.shape
    _check(L, "L", dev)
    _check(anchor, "anchor", dev, (batch,), torch.int32)
    _check(ctx_len, "ctx_len", dev, (batch,), torch.int64)
    desc = cadd_desc(batch, D, V, n_max, _code(L), C_d, a, b, c, e)
    if out is None:
        out = TreeOut(*(torch.empty((batch, n_max), dtype=torch.int32, device=dev) for _ in range(3)),
                      torch.empty((batch, n_max), dtype=torch.float32, device=dev),
                      torch.empty(batch, dtype=torch.int32, device=dev),
                      torch.empty(batch, dtype=torch.int32, device=dev),
                      torch.empty(batch, dtype=torch.float32, device=dev))
    nbytes = int(lib().cadd_tree_grow_workspace(ctypes.byref(desc)))
    if nbytes == 0:
        _raise(PCT_EINVAL, "cadd_tree_grow_workspace")
    ws, wsb = _workspace(nbytes, dev, workspace)
    if top_tok is not None:
        if top_tok.dim() != 3:
            raise ValueError("top_tok must be [batch][D][top_k]")
        _check(top_tok, "top_tok", dev, (batch, D, top_tok.shape[2]), torch.int32)
        code = lib().cadd_tree_grow_topk(ctypes.byref(desc), _p(L), _p(anchor), _p(ctx_len),
                                         int(top_tok.shape[2]), _p(out.tok), _p(out.parent),
                                         _p(out.depth), _p(out.score), _p(out.count), _p(out.phi),
                                         _p(top_tok), _p(out.status), _p(ws), wsb, _stream(stream))
        _raise(code, "cadd_tree_grow_topk")
        return out
    code = lib().cadd_tree_grow(ctypes.byref(desc), _p(L), _p(anchor), _p(ctx_len), _p(out.tok),
                                _p(out.parent), _p(out.depth), _p(out.score), _p(out.count),
                                _p(out.phi), _p(out.status), _p(ws), wsb, _stream(stream))
    _raise(code, "cadd_tree_grow")
    return out


def tree_ancestor_mask(parent: torch.Tensor, count: torch.Tensor, mask: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, stream=None):
    """Self-plus-ancestor bitmask [batch][n_stride][ceil(n_stride/32)] (int32 view of uint32)."""
    dev = parent.device
    batch, n_stride = parent.shape
    _check(parent, "parent", dev, dtype=torch.int32)
    _check(count, "count", dev, (batch,), torch.int32)
    words = (n_stride + 31) // 32
    if mask is None:
        mask = torch.empty((batch, n_stride, words), dtype=torch.int32, device=dev)
    if status is None:
        status = torch.empty(batch, dtype=torch.int32, device=dev)
    code = lib().tree_ancestor_mask(batch, n_stride, _p(parent), _p(count), _p(mask), _p(status),
                                    _stream(stream))
    _raise(code, "tree_ancestor_mask")
    return mask, status


@dataclass
class VerifyOut:
    argmax: torch.Tensor
    accept_len: torch.Tensor
    accept_path: torch.Tensor
    correction: torch.Tensor
    status: torch.Tensor


def tree_verify_accept(tok: torch.Tensor, parent: torch.Tensor, count: torch.Tensor,
                       target: torch.Tensor, max_depth: int, out: Optional[VerifyOut] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> VerifyOut:
    """Greedy verification of node tables against target logits [batch][n_stride][V]."""
    dev = tok.device
    batch, n_stride = tok.shape
    V = target.shape[2]
    _check(tok, "tok", dev, dtype=torch.int32)
    _check(parent, "parent", dev, (batch, n_stride), torch.int32)
    _check(count, "count", dev, (batch,), torch.int32)
    _check(target, "target", dev, (batch, n_stride, V))
    if out is None:
        out = VerifyOut(torch.empty((batch, n_stride), dtype=torch.int32, device=dev),
                        torch.empty(batch, dtype=torch.int32, device=dev),
                        torch.empty((batch, max_depth), dtype=torch.int32, device=dev),
                        torch.empty(batch, dtype=torch.int32, device=dev),
                        torch.empty(batch, dtype=torch.int32, device=dev))
    nbytes = int(lib().tree_verify_accept_workspace(batch, n_stride))
    ws, wsb = _workspace(nbytes, dev, workspace)
    code = lib().tree_verify_accept(batch, n_stride, V, max_depth, _p(tok), _p(parent), _p(count),
                                    _p(target), _code(target), _p(out.argmax), _p(out.accept_len),
                                    _p(out.accept_path), _p(out.correction), _p(out.status),
                                    _p(ws), wsb, _stream(stream))
    _raise(code, "tree_verify_accept")
    return out


def tree_verify_walk(tok: torch.Tensor, parent: torch.Tensor, count: torch.Tensor,
                     target: torch.Tensor, max_depth: int, out: Optional[VerifyOut] = None,
                     stream=None) -> VerifyOut:
    """Greedy verification reading only the rows the walk reaches: the same
    accept_len, accept_path and correction as tree_verify_accept; argmax holds
    the walked rows' argmax and -1 elsewhere."""
    dev = tok.device
    batch, n_stride = tok.shape
    V = target.shape[2]
    _check(tok, "tok", dev, dtype=torch.int32)
    _check(parent, "parent", dev, (batch, n_stride), torch.int32)
    _check(count, "count", dev, (batch,), torch.int32)
    _check(target, "target", dev, (batch, n_stride, V))
    if out is None:
        out = VerifyOut(torch.empty((batch, n_stride), dtype=torch.int32, device=dev),
                        torch.empty(batch, dtype=torch.int32, device=dev),
                        torch.empty((batch, max_depth), dtype=torch.int32, device=dev),
                        torch.empty(batch, dtype=torch.int32, device=dev),
                        torch.empty(batch, dtype=torch.int32, device=dev))
    code = lib().tree_verify_walk(batch, n_stride, V, max_depth, _p(tok), _p(parent), _p(count),
                                  _p(target), _code(target), _p(out.argmax), _p(out.accept_len),
                                  _p(out.accept_path), _p(out.correction), _p(out.status),
                                  _stream(stream))
    _raise(code, "tree_verify_walk")
    return out


def tree_accept_sim(parent: torch.Tensor, count: torch.Tensor, p_child: torch.Tensor,
                    trials: int, seed: int, max_depth: int, stream=None):
    """Monte Carlo walks of greedy verification: (hist [batch][max_depth + 1]
    int64 walks per accepted length, status [batch])."""
    dev = parent.device
    batch, n_stride = parent.shape
    _check(parent, "parent", dev, dtype=torch.int32)
    _check(count, "count", dev, (batch,), torch.int32)
    _check(p_child, "p_child", dev, (batch, n_stride), torch.float32)
    hist = torch.empty((batch, max_depth + 1), dtype=torch.int64, device=dev)
    status = torch.empty(batch, dtype=torch.int32, device=dev)
    code = lib().tree_accept_sim(batch, n_stride, max_depth, _p(parent), _p(count), _p(p_child),
                                 int(trials), int(seed) & ((1 << 64) - 1), _p(hist), _p(status),
                                 _stream(stream))
    _raise(code, "tree_accept_sim")
    return hist, status


def cadd_cost_fit(n: torch.Tensor, ell: torch.Tensor, lat: torch.Tensor, stream=None):
    """Non-negative fit of C_v(n; l) = a + b l + c n + e n^2 to latency samples:
    (out float64 [5] = a, b, c, e, rms; status [1])."""
    dev = n.device
    m = n.numel()
    _check(n, "n", dev, (m,), torch.float32)
    _check(ell, "ell", dev, (m,), torch.float32)
    _check(lat, "lat", dev, (m,), torch.float32)
    out = torch.empty(5, dtype=torch.float64, device=dev)
    status = torch.empty(1, dtype=torch.int32, device=dev)
    code = lib().cadd_cost_fit(m, _p(n), _p(ell), _p(lat), _p(out), _p(status), _stream(stream))
    _raise(code, "cadd_cost_fit")
    return out, status


def trace_enable(on: bool = True) -> bool:
    return bool(lib().pct_trace_enable(1 if on else 0))


def trace_reset():
    lib().pct_trace_reset()


def trace_read(max_entries: int = 64) -> dict:
    """{kernel name: (launches, total ms)} for the launches recorded since the last reset."""
    stride = 64
    names = ctypes.create_string_buffer(stride * max_entries)
    launches = (ctypes.c_int64 * max_entries)()
    ms = (ctypes.c_double * max_entries)()
    n = lib().pct_trace_read(names, stride, ctypes.cast(launches, ctypes.c_void_p),
                             ctypes.cast(ms, ctypes.c_void_p), max_entries)
    if n < 0:
        raise PctError(PCT_ECUDA, "pct_trace_read")
    out = {}
    for i in range(n):
        nm = names.raw[i * stride:(i + 1) * stride].split(b"\0", 1)[0].decode()
        out[nm] = (int(launches[i]), float(ms[i]))
    return out


def version() -> str:
    return lib().pct_version().decode()
