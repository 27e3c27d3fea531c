"""Acceptance simulation oracle: Monte Carlo walks of greedy verification (test infrastructure only).

Source: DSpark explainer (xiaohu-jiedu), one round from drafting to
confirmation: the drafts are checked from the head, every consecutive match is
kept and the first miss ends the round, which then yields the matches plus one
token of the target's own. On a tree the round starts at the root; at a node u
the target's token for the next position is drawn, and the round moves to the
child of u that carries it, or ends if no child does. PCTree article (qiita),
numbers table: tau, the tokens accepted per round, is the headline measure.

What a walk needs at node u is only which child the draw hits, or that it hits
none: with p(c) = P(target's token = token of child c | the target agreed up to
u), one uniform draw x and the children of u in index order, the walk moves to
the first child c whose running sum p(c_1) + ... + p(c) exceeds x, and stops if
none does. When the target is the drafter itself, p(c) = exp(s(c) - s(u)) and
the expected number of accepted drafts is Phi(T), the sum of exp(s) over the
non-root nodes ("Cost-Aware Diffusion Draft Trees for Speculative Decoding",
gist.science summary, "Method: CaDDTree"). The tests pin this routine to that
identity and its random numbers to the published known answers of the
generator.

Random numbers: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
numbers: as easy as 1, 2, 3", SC 2011): a 128-bit counter and a 64-bit key,
ten rounds of two 32 x 32 -> 64-bit multiplications with the round key bumped
by the Weyl constants between rounds. Draw j of trial t of request b uses the
counter (t, b, j, 0) and the key (seed mod 2^32, seed div 2^32); the uniform is
the first output word's top 24 bits times 2^-24 (exact in float32). The running
sums are float32, added in child index order, and compared as float32, so that
a float32 implementation takes every decision the same way.
"""
from __future__ import annotations

import numpy as np

M0, M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
W0, W1 = np.uint32(0x9E3779B9), np.uint32(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Philox4x32-10 on arrays: ctr (..., 4) uint32, key (..., 2) uint32 -> (..., 4) uint32."""
    c = [np.asarray(ctr[..., i], dtype=np.uint32) for i in range(4)]
    k0 = np.asarray(key[..., 0], dtype=np.uint32)
    k1 = np.asarray(key[..., 1], dtype=np.uint32)
    for rnd in range(10):
        if rnd > 0:
            k0 = ((k0.astype(np.uint64) + np.uint64(W0)) & MASK32).astype(np.uint32)
            k1 = ((k1.astype(np.uint64) + np.uint64(W1)) & MASK32).astype(np.uint32)
        p0 = c[0].astype(np.uint64) * M0          # 32 x 32 -> 64 bits
        p1 = c[2].astype(np.uint64) * M1
        hi0, lo0 = (p0 >> np.uint64(32)).astype(np.uint32), (p0 & MASK32).astype(np.uint32)
        hi1, lo1 = (p1 >> np.uint64(32)).astype(np.uint32), (p1 & MASK32).astype(np.uint32)
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return np.stack(c, axis=-1)


def uniform24(word):
    """float32 uniform in [0, 1) from the top 24 bits of a uint32 word."""
    return (np.asarray(word, dtype=np.uint32) >> np.uint32(8)).astype(np.float32) * \
        np.float32(1.0 / 16777216.0)


def accept_sim(parent, count, p_child, trials: int, seed: int, max_depth: int):
    """Histogram [batch][max_depth + 1] of accepted drafts over `trials` walks per request.

    parent, p_child: [batch][n_stride] (p_child[c] as above, float32); count:
    [batch]. A walk also stops after max_depth accepted drafts.
    """
    parent = np.asarray(parent)
    count = np.asarray(count)
    p_child = np.asarray(p_child, dtype=np.float32)
    batch = parent.shape[0]
    hist = np.zeros((batch, max_depth + 1), np.int64)
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], np.uint32)
    t = np.arange(trials, dtype=np.uint32)
    for b in range(batch):
        n = int(count[b])
        kids = [[] for _ in range(n)]
        for c in range(1, n):
            kids[int(parent[b, c])].append(c)
        node = np.zeros(trials, np.int64)
        alive = np.ones(trials, bool)
        acc = np.zeros(trials, np.int64)
        for j in range(max_depth):
            if not alive.any():
                break
            ctr = np.stack([t, np.full(trials, b, np.uint32), np.full(trials, j, np.uint32),
                            np.zeros(trials, np.uint32)], axis=-1)
            x = uniform24(philox4x32_10(ctr, np.broadcast_to(key, (trials, 2)))[:, 0])
            nxt = np.full(trials, -1, np.int64)
            for i in np.nonzero(alive)[0]:
                cum = np.float32(0.0)
                for c in kids[int(node[i])]:
                    cum = np.float32(cum + p_child[b, c])
                    if x[i] < cum:
                        nxt[i] = c
                        break
            moved = alive & (nxt >= 0)
            node = np.where(moved, nxt, node)
            acc += moved
            alive = moved
        hist[b] = np.bincount(acc, minlength=max_depth + 1)[: max_depth + 1]
    return hist
