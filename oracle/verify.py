"""Tree verification oracle (test infrastructure only).

Source: DSpark explainer (xiaohu-jiedu), section on one round from drafting to
confirmation: the drafted tokens are checked from the head; every consecutive
match is kept, checking stops at the first miss, and at that point the target
supplies its own token, so a round that matched four drafts yields five tokens
for one verification. The PCTree article adds that the whole tree is verified in
one target forward and that decoding is greedy.

Readings taken: greedy verification on a tree. am[u] is the argmax of the
target logits of node u (ties toward the lower token id, compared on the raw
values). From the root, move to the child whose token equals am[u]; stop when
no child matches. The correction token is am at the last accepted node (when
every drafted level matched, that is the target's next token after the leaf).

The ancestor mask has bit j of row i set when j = i or j is an ancestor of i;
uint32 words, least significant bit first, ceil(n_stride / 32) words per row;
rows at or past ``count`` are zero.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .numerics import to_f64


@dataclass
class VerifyResult:
    argmax: np.ndarray        # [batch][n_stride] int32, -1 past count
    accept_len: np.ndarray    # [batch]
    accept_path: np.ndarray   # [batch][max_depth] accepted node ids, -1 padded
    correction: np.ndarray    # [batch]
    status: np.ndarray        # [batch], nonzero when a walk would exceed max_depth


def tree_verify_accept(tok, parent, count, target, max_depth: int) -> VerifyResult:
    """Greedy tree verification.

    target: per-request rows of target logits, indexable as target[b][i] and
    decodable by ``to_f64`` (fp32 / bf16 tensors or numpy arrays); rows are
    decoded one at a time so full-size inputs need not be widened at once.
    """
    tok = np.asarray(tok)
    parent = np.asarray(parent)
    count = np.asarray(count)
    batch, n_stride = tok.shape
    am = np.full((batch, n_stride), -1, np.int32)
    alen = np.zeros(batch, np.int32)
    path = np.full((batch, max_depth), -1, np.int32)
    corr = np.zeros(batch, np.int32)
    status = np.zeros(batch, np.int32)
    for b in range(batch):
        n = int(count[b])
        for i in range(n):
            row = to_f64(target[b][i])
            am[b, i] = int(np.argmax(row))          # first maximum: lowest token id
        u, acc = 0, []
        while True:
            nxt = [c for c in range(1, n) if parent[b, c] == u and tok[b, c] == am[b, u]]
            if not nxt:
                break
            if len(acc) == max_depth:
                status[b] = 1
                break
            u = min(nxt)
            acc.append(u)
        alen[b] = len(acc)
        path[b, : len(acc)] = acc
        corr[b] = am[b, u]
    return VerifyResult(am, alen, path, corr, status)


def tree_ancestor_mask(parent, count, n_stride: int) -> np.ndarray:
    """Self-plus-ancestor bitmask [batch][n_stride][ceil(n_stride/32)] uint32."""
    parent = np.asarray(parent)
    count = np.asarray(count)
    batch = parent.shape[0]
    words = (n_stride + 31) // 32
    mask = np.zeros((batch, n_stride, words), np.uint32)
    for b in range(batch):
        for i in range(int(count[b])):
            j = i
            while j != -1:
                mask[b, i, j // 32] |= np.uint32(1) << np.uint32(j % 32)
                j = int(parent[b, j])
    return mask
