"""Pins of the verification and mask oracles (CPU only)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_round_four_plus_one():
    """The explainer's round: 4 drafted tokens accepted + 1 target correction = 5 tokens."""
    g = json.load(open(os.path.join(GOLDEN, "worked_round.json")))
    chain = g["drafted_chain"]
    n = len(chain) + 1
    tok = np.array([[g["anchor"]] + chain], np.int32)
    par = np.array([[-1] + list(range(n - 1))], np.int32)
    T = np.zeros((1, n, g["vocab"]))
    for i, t in enumerate(g["target_argmax_per_node"]):
        T[0, i, t] = 5.0
    r = oracle.tree_verify_accept(tok, par, [n], T, max_depth=len(chain))
    exp = g["expected"]
    assert r.accept_len[0] == exp["accepted"]
    assert r.correction[0] == exp["correction"]
    assert r.accept_len[0] + 1 == exp["tokens_gained"]
    assert list(r.accept_path[0, : exp["accepted"]]) == exp["accepted_nodes"]
    assert (r.accept_path[0, exp["accepted"]:] == -1).all()


@pytest.mark.parametrize("seed", range(4))
def test_planted_paths_are_recovered(seed):
    batch, n_stride, V, D = 6, 48, 300, 7
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, V, D, seed=seed)
    T = workloads.target_logits(batch, n_stride, V, 2.0, seed=seed)
    walked, paths, ends = workloads.plant_path(T, tok, par, cnt, seed=seed, length_range=(0, 16))
    r = oracle.tree_verify_accept(tok, par, cnt, T, max_depth=D)
    np.testing.assert_array_equal(r.accept_len, walked)
    np.testing.assert_array_equal(r.correction, ends)
    for b in range(batch):
        assert list(r.accept_path[b, : walked[b]]) == list(paths[b, : walked[b]])
    assert (r.argmax[np.arange(n_stride)[None, :] >= cnt[:, None]] == -1).all()


def test_argmax_ties_go_to_lower_token_and_bf16_is_compared_exactly():
    T = torch.zeros((1, 2, 40), dtype=torch.bfloat16)
    T[0, 0, 9] = T[0, 0, 31] = 3.0
    T[0, 1, 5] = 1.0078125            # next bf16 above 1.0
    T[0, 1, 4] = 1.0
    r = oracle.tree_verify_accept(np.array([[0, 9]]), np.array([[-1, 0]]), [2], T, max_depth=1)
    assert list(r.argmax[0]) == [9, 5]
    assert r.accept_len[0] == 1 and r.correction[0] == 5


def test_walk_longer_than_max_depth_sets_status():
    tok = np.array([[0, 1, 2]])
    par = np.array([[-1, 0, 1]])
    T = np.zeros((1, 3, 4))
    T[0, 0, 1] = T[0, 1, 2] = T[0, 2, 3] = 1.0
    r = oracle.tree_verify_accept(tok, par, [3], T, max_depth=1)
    assert r.status[0] != 0 and r.accept_len[0] == 1
    r = oracle.tree_verify_accept(tok, par, [3], T, max_depth=2)
    assert r.status[0] == 0 and r.accept_len[0] == 2 and r.correction[0] == 3


def _closure_bits(par, n, n_stride):
    """Self + ancestors via boolean powers of the child->parent adjacency matrix."""
    A = np.zeros((n_stride, n_stride), np.int64)
    for i in range(1, n):
        A[i, par[i]] = 1
    R = np.eye(n_stride, dtype=np.int64)
    R[n:, :] = 0
    P = R.copy()
    for _ in range(n):
        P = np.minimum(P @ A, 1)
        R = np.minimum(R + P, 1)
    words = (n_stride + 31) // 32
    out = np.zeros((n_stride, words), np.uint32)
    for i in range(n):
        for j in np.nonzero(R[i])[0]:
            out[i, j // 32] |= np.uint32(1 << (j % 32))
    return out


@pytest.mark.parametrize("n_stride", [1, 31, 32, 33, 70, 256])
def test_mask_is_transitive_closure(n_stride):
    batch, D = 3, 9
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, 500, D, seed=n_stride)
    m = oracle.tree_ancestor_mask(par, cnt, n_stride)
    assert m.shape == (batch, n_stride, (n_stride + 31) // 32)
    for b in range(batch):
        np.testing.assert_array_equal(m[b], _closure_bits(par[b], cnt[b], n_stride))
        for i in range(cnt[b]):
            bits = sum(bin(int(w)).count("1") for w in m[b, i])
            assert bits == dep[b, i] + 1
            assert (m[b, i, i // 32] >> (i % 32)) & 1
            if i:
                p = par[b, i]
                assert ((m[b, i] & m[b, p]) == m[b, p]).all()
        assert (m[b, cnt[b]:] == 0).all()
