"""Helpers shared by the GPU parity tests (comparison rules, host copies,
oracle runs over many requests, and the per-configuration parity report)."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle

SCORE_TOL = 1e-4      # absolute, path scores and log-probabilities
PHI_RTOL = 1e-4       # relative, Phi(T)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def f64(t) -> np.ndarray:
    return oracle.to_f64(t)


def compare_trees(gpu, ref, excluded=None, rows=None, label=""):
    """Bit-exact node tables and count on non-excluded requests; scores within SCORE_TOL.

    gpu: object with tok/parent/depth/score/count tensors; ref: oracle result.
    rows: which gpu rows correspond to ref rows (default: all, in order).
    Returns the number of compared requests.
    """
    tok, par, dep, sc, cnt = (host(gpu.tok), host(gpu.parent), host(gpu.depth),
                              host(gpu.score), host(gpu.count))
    n_ref = ref.tok.shape[0]
    rows = list(range(n_ref)) if rows is None else list(rows)
    excluded = ref.excluded if excluded is None else excluded
    compared = 0
    for j, b in enumerate(rows):
        if excluded[j]:
            continue
        n = int(ref.count[j])
        msg = f"{label} request {b}"
        assert int(cnt[b]) == n, f"{msg}: count {cnt[b]} != {n}"
        np.testing.assert_array_equal(tok[b], ref.tok[j], err_msg=msg + " tok")
        np.testing.assert_array_equal(par[b], ref.parent[j], err_msg=msg + " parent")
        np.testing.assert_array_equal(dep[b], ref.depth[j], err_msg=msg + " depth")
        np.testing.assert_allclose(sc[b, :n], ref.score[j, :n], rtol=0, atol=SCORE_TOL,
                                   err_msg=msg + " score")
        assert np.isneginf(sc[b, n:]).all(), msg + " padding score"
        compared += 1
    return compared


def check_tree_invariants(gpu, anchor, n_nodes, label=""):
    """Properties of any valid output: root, canonical order, parent < child, scores."""
    tok, par, dep, sc, cnt = (host(gpu.tok), host(gpu.parent), host(gpu.depth),
                              host(gpu.score), host(gpu.count))
    anchor = np.asarray(anchor)
    for b in range(tok.shape[0]):
        n = int(cnt[b])
        assert 1 <= n <= n_nodes, label
        assert tok[b, 0] == anchor[b] and par[b, 0] == -1 and dep[b, 0] == 0 and sc[b, 0] == 0
        p = par[b, 1:n]
        assert (p >= 0).all() and (p < np.arange(1, n)).all(), f"{label} parent order {b}"
        assert (dep[b, 1:n] == dep[b, p] + 1).all()
        assert (sc[b, 1:n] <= sc[b, p] + 1e-6).all()
        keys = list(zip(dep[b, 1:n], p, tok[b, 1:n]))
        assert keys == sorted(keys) and len(set(keys)) == len(keys), f"{label} canonical {b}"
        assert (tok[b, n:] == -1).all() and (par[b, n:] == -1).all() and (dep[b, n:] == -1).all()


# ---------------------------------------------------------------------------
# oracle over many requests: one request per task, in threads (numpy's sorts,
# matrix products and elementwise loops release the interpreter lock)
def host_threads() -> int:
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return max(1, int(n or 1))


def oracle_map(fn, items):
    items = list(items)
    with ThreadPoolExecutor(max_workers=min(len(items), host_threads())) as ex:
        return list(ex.map(fn, items))


def gpu_paths(gpu, b) -> set:
    """Token paths below the root of request b's tree in a GPU result."""
    tok, par, n = host(gpu.tok)[b], host(gpu.parent)[b], int(host(gpu.count)[b])
    paths, out = {0: ()}, set()
    for i in range(1, n):
        p = int(par[i])
        if p < 0 or p >= i:
            break                      # malformed table: leave it to the comparison
        paths[i] = paths[p] + (int(tok[i]),)
        out.add(paths[i])
    return out


# ---------------------------------------------------------------------------
# parity report, printed at the end of the pytest run (tests/conftest.py)
REPORT: dict = {}


def report(label, requests, exact, resolved, excluded):
    REPORT[label] = (requests, exact, resolved, excluded)


def compare_all(gpu, refs, rebuild, rows, label, max_unresolved=1, phi=False):
    """Every request of ``rows`` against the oracle, element by element.

    refs[j] is the oracle's result for gpu row rows[j] (a one-request result).
    A request with no near tie at a selection boundary must match bit-exactly.
    A request with one (two candidates closer than the tolerance, so that either
    order is correct) is compared bit-exactly against rebuild(j, paths): the
    oracle's tree with its near ties resolved toward the GPU's nodes ``paths``.
    If even that differs the request counts as excluded; at most
    ``max_unresolved`` may. Returns (exact, resolved, excluded) and records them
    in the parity report under ``label``.
    """
    exact = resolved = excluded = 0
    for j, b in enumerate(rows):
        ref = refs[j]
        if not ref.excluded[0]:
            compare_trees(gpu, ref, excluded=[False], rows=[b], label=label)
            if phi:
                np.testing.assert_allclose(host(gpu.phi)[b], ref.phi[0], rtol=PHI_RTOL, atol=1e-7)
            exact += 1
            continue
        alt = rebuild(j, gpu_paths(gpu, b))
        try:
            compare_trees(gpu, alt, excluded=[False], rows=[b], label=label + " (near tie)")
            if phi:
                np.testing.assert_allclose(host(gpu.phi)[b], alt.phi[0], rtol=PHI_RTOL, atol=1e-7)
            resolved += 1
        except AssertionError:
            excluded += 1
    report(label, len(rows), exact, resolved, excluded)
    assert excluded <= max_unresolved, f"{label}: {excluded} requests unresolved of {len(rows)}"
    return exact, resolved, excluded
