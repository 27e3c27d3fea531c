"""GPU parity: greedy tree verification and the ancestor mask against the oracle.

DSpark explainer (xiaohu-jiedu), one round from drafting to confirmation:
accept the longest matching root path, then the target's own token.
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


def _to_dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).to(DEV) for a in arrs]


@pytest.mark.parametrize("dtype,V", [("bf16", 1000), ("bf16", 1003), ("bf16", 64),
                                     ("f32", 777), ("f32", 1024)])
def test_verify_matches_oracle(dtype, V):
    batch, n_stride, D = 6, 70, 9
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, V, D, seed=V)
    T = workloads.target_logits(batch, n_stride, V, 2.0, seed=V + 1, dtype=dtype)
    walked, paths, ends = workloads.plant_path(T, tok, par, cnt, seed=V + 2, length_range=(0, 12))
    # exact ties in a planted row: the lower token must win
    T[0, 0, :] = -5.0
    T[0, 0, 3] = T[0, 0, 7] = 9.0
    # an all -inf row
    T[1, 1, :] = float("-inf")
    ref = oracle.tree_verify_accept(tok, par, cnt, T, max_depth=D)
    dtok, dpar, dcnt = _to_dev(tok, par, cnt)
    out = pct.tree_verify_accept(dtok, dpar, dcnt, T.to(DEV), max_depth=D)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(out.argmax), ref.argmax)
    np.testing.assert_array_equal(host(out.accept_len), ref.accept_len)
    np.testing.assert_array_equal(host(out.accept_path), ref.accept_path)
    np.testing.assert_array_equal(host(out.correction), ref.correction)
    np.testing.assert_array_equal(host(out.status), ref.status)
    assert host(out.argmax)[0, 0] == 3


def test_verify_repeated_calls_are_identical():
    batch, n_stride, V, D = 4, 40, 2048, 6
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, V, D, seed=5)
    T = workloads.target_logits(batch, n_stride, V, 2.0, seed=6).to(DEV)
    dtok, dpar, dcnt = _to_dev(tok, par, cnt)
    first = pct.tree_verify_accept(dtok, dpar, dcnt, T, max_depth=D)
    a0 = [host(x).copy() for x in (first.argmax, first.accept_len, first.accept_path, first.correction)]
    for _ in range(10):
        o = pct.tree_verify_accept(dtok, dpar, dcnt, T, max_depth=D)
        for x, y in zip(a0, (o.argmax, o.accept_len, o.accept_path, o.correction)):
            np.testing.assert_array_equal(x, host(y))


def test_verify_depth_overflow_and_bad_inputs_set_status():
    V = 128
    tok = np.array([[0, 1, 2, 3], [0, 1, 2, -1]], np.int32)
    par = np.array([[-1, 0, 1, 2], [-1, 0, 5, -1]], np.int32)    # request 1: parent 5 > 2
    cnt = np.array([4, 3], np.int32)
    T = torch.zeros((2, 4, V), dtype=torch.bfloat16)
    T[0, 0, 1] = T[0, 1, 2] = T[0, 2, 3] = T[0, 3, 9] = 1.0
    ref = oracle.tree_verify_accept(tok, par, cnt, T, max_depth=2)
    dtok, dpar, dcnt = _to_dev(tok, par, cnt)
    out = pct.tree_verify_accept(dtok, dpar, dcnt, T.to(DEV), max_depth=2)
    st = host(out.status)
    assert st[0] & pct.DEV_DEPTH_OVERFLOW and ref.status[0] != 0
    assert host(out.accept_len)[0] == 2
    assert st[1] & pct.DEV_BAD_PARENT
    # a count outside [1, n_stride]
    cnt2 = np.array([4, 9], np.int32)
    out = pct.tree_verify_accept(dtok, dpar, _to_dev(cnt2)[0], T.to(DEV), max_depth=4)
    assert host(out.status)[1] & pct.DEV_BAD_COUNT


@pytest.mark.parametrize("n_stride", [1, 31, 32, 33, 256, 1000])
def test_mask_matches_oracle(n_stride):
    batch, D = 5, 15
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, 5000, D, seed=n_stride + 3)
    ref = oracle.tree_ancestor_mask(par, cnt, n_stride)
    dpar, dcnt = _to_dev(par, cnt)
    mask, status = pct.tree_ancestor_mask(dpar, dcnt)
    got = host(mask).view(np.uint32)
    np.testing.assert_array_equal(got, ref)
    assert (host(status) == 0).all()


def test_mask_flags_bad_parent():
    par = np.array([[-1, 0, 3, 1]], np.int32)   # node 2 points forward
    cnt = np.array([4], np.int32)
    dpar, dcnt = _to_dev(par, cnt)
    mask, status = pct.tree_ancestor_mask(dpar, dcnt)
    assert host(status)[0] & pct.DEV_BAD_PARENT


@pytest.mark.slow
def test_verify_full_size_planted_paths():
    """Full-round verification shape: 64 requests x 256 nodes x V = 151936 bf16 (4.98 GB)."""
    w = workloads.FULL_ROUND
    batch, n_stride, V, D = w.batch, w.n_nodes, w.vocab, w.depth
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, V, D, seed=41,
                                               counts=[n_stride] * batch)
    T = workloads.target_logits(batch, n_stride, V, 2.0, seed=w.seed + 1000, device=DEV)
    walked, paths, ends = workloads.plant_path(T, tok, par, cnt, seed=w.seed + 1001)
    dtok, dpar, dcnt = _to_dev(tok, par, cnt)
    out = pct.tree_verify_accept(dtok, dpar, dcnt, T, max_depth=D)
    torch.cuda.synchronize()
    # every request: the planted walk is recovered exactly
    np.testing.assert_array_equal(host(out.accept_len), walked)
    np.testing.assert_array_equal(host(out.correction), ends)
    ap = host(out.accept_path)
    for b in range(batch):
        assert list(ap[b, : walked[b]]) == list(paths[b, : walked[b]])
    # two requests: every row's argmax against the oracle
    sample = [0, batch - 1]
    ref = oracle.tree_verify_accept(tok[sample], par[sample], cnt[sample], T[sample], max_depth=D)
    np.testing.assert_array_equal(host(out.argmax)[sample], ref.argmax)
    np.testing.assert_array_equal(host(out.accept_len)[sample], ref.accept_len)
    del T
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# Lazy walk: argmax only of the rows the walk reaches (DSpark explainer: the
# comparison runs from the head and stops at the first miss).
def _walk_vs_oracle(tok, par, cnt, T, D, label=""):
    ref = oracle.tree_verify_accept(tok, par, cnt, T, max_depth=D)
    dtok, dpar, dcnt = _to_dev(tok, par, cnt)
    out = pct.tree_verify_walk(dtok, dpar, dcnt, T.to(DEV), max_depth=D)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(out.accept_len), ref.accept_len, err_msg=label)
    np.testing.assert_array_equal(host(out.accept_path), ref.accept_path, err_msg=label)
    np.testing.assert_array_equal(host(out.correction), ref.correction, err_msg=label)
    am = host(out.argmax)
    for b in range(tok.shape[0]):
        walked = [0] + [int(x) for x in ref.accept_path[b, : ref.accept_len[b]]] \
            if int(cnt[b]) >= 1 else []
        want = np.full(tok.shape[1], -1, np.int32)
        want[walked] = ref.argmax[b, walked]
        np.testing.assert_array_equal(am[b], want, err_msg=f"{label} request {b} argmax")
    return out, ref


@pytest.mark.parametrize("dtype,V", [("bf16", 1000), ("bf16", 1003), ("bf16", 64),
                                     ("bf16", 8), ("f32", 777), ("f32", 1024), ("f32", 5)])
def test_walk_matches_oracle(dtype, V):
    batch, n_stride, D = 6, 70, 9
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, V, D, seed=V + 50)
    T = workloads.target_logits(batch, n_stride, V, 2.0, seed=V + 51, dtype=dtype)
    workloads.plant_path(T, tok, par, cnt, seed=V + 52, length_range=(0, 12))
    T[0, 0, :] = -5.0                    # exact ties at the root: the lower token wins
    T[0, 0, 3 % V] = T[0, 0, (V - 1)] = 9.0
    T[1, 0, :] = float("-inf")           # an all -inf root row: token 0
    out, ref = _walk_vs_oracle(tok, par, cnt, T, D, f"{dtype} V={V}")
    assert (host(out.status) == 0).all()


def test_walk_ties_across_the_eight_parts():
    """Equal maxima in different eighths of the row: the lowest token wins."""
    V, D = 8192, 4
    tok = np.array([[0, 5, 1000, 7000, -1]], np.int32)
    par = np.array([[-1, 0, 0, 0, -1]], np.int32)
    cnt = np.array([4], np.int32)
    T = torch.zeros((1, 5, V), dtype=torch.bfloat16)
    T[0, 0, [7000, 1000, 5000]] = 3.0    # parts 6, 0 and 4: token 1000 wins
    out, ref = _walk_vs_oracle(tok, par, cnt, T, D, "ties")
    assert host(out.accept_path)[0, 0] == 2 and host(out.accept_len)[0] == 1


def test_walk_status_like_full_verification():
    V = 128
    tok = np.array([[0, 1, 2, 3], [0, 1, 2, -1]], np.int32)
    par = np.array([[-1, 0, 1, 2], [-1, 0, 5, -1]], np.int32)
    cnt = np.array([4, 3], np.int32)
    T = torch.zeros((2, 4, V), dtype=torch.bfloat16)
    T[0, 0, 1] = T[0, 1, 2] = T[0, 2, 3] = T[0, 3, 9] = 1.0
    dtok, dpar, dcnt = _to_dev(tok, par, cnt)
    for D, cn in ((2, cnt), (4, np.array([4, 9], np.int32)), (4, np.array([0, 3], np.int32))):
        dc = _to_dev(cn)[0]
        full = pct.tree_verify_accept(dtok, dpar, dc, T.to(DEV), max_depth=D)
        walk = pct.tree_verify_walk(dtok, dpar, dc, T.to(DEV), max_depth=D)
        torch.cuda.synchronize()
        for f in ("status", "accept_len", "accept_path", "correction"):
            np.testing.assert_array_equal(host(getattr(walk, f)), host(getattr(full, f)),
                                          err_msg=f"max_depth {D} counts {cn}: {f}")


def test_walk_repeated_calls_are_identical():
    batch, n_stride, V, D = 4, 40, 2048, 6
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, V, D, seed=15)
    T = workloads.target_logits(batch, n_stride, V, 2.0, seed=16)
    workloads.plant_path(T, tok, par, cnt, seed=17, length_range=(2, 6))
    T = T.to(DEV)
    dtok, dpar, dcnt = _to_dev(tok, par, cnt)
    first = pct.tree_verify_walk(dtok, dpar, dcnt, T, max_depth=D)
    a0 = [host(x).copy() for x in (first.argmax, first.accept_len, first.accept_path,
                                   first.correction)]
    for _ in range(10):
        o = pct.tree_verify_walk(dtok, dpar, dcnt, T, max_depth=D)
        for x, y in zip(a0, (o.argmax, o.accept_len, o.accept_path, o.correction)):
            np.testing.assert_array_equal(x, host(y))
