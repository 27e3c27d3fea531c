"""The roofline numerators of bench.py against the closed forms of the hot path.

For the full round (64 requests, V = 151936, D = 15, r = 256, k = 8, beam 32,
N = 256), the parent rows per depth are 64, 512 and then 2048 for the
remaining 13 depths. Each row costs 2 r V flops in the Markov contraction.
Verify reads every node row of bf16 target logits once, and the CaDDTree row
pass reads every marginal row once. No GPU needed.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_frontier_rows_per_depth():
    F = bench.frontier_sizes()
    assert F == [1, 8, 32] + [32] * 13
    rows = [64 * f for f in F[:15]]
    assert rows[:3] == [64, 512, 2048] and sum(rows) == 27200


def test_algorithmic_work_matches_closed_forms():
    w = bench.algorithmic_work()
    V, r = 151936, 256
    pair = 2.0 * r * V * (512 + 13 * 2048)
    single = 2.0 * r * V * 64
    assert w["pct_score_pair"]["flop"] == pair
    assert w["pct_score_umma"]["flop"] == single
    assert abs((pair + single) / 1e12 - 2.116) < 1e-3            # 2.116 TFLOP per round
    assert w["verify_argmax_walk"]["bytes"] == 64 * 256 * V * 2  # 4.979 GB
    assert abs(w["verify_argmax_walk"]["bytes"] / 1e9 - 4.979) < 1e-3
    assert w["cadd_rowpass"]["bytes"] == 64 * 15 * V * 2         # 291.7 MB
    assert abs(w["cadd_rowpass"]["bytes"] / 1e6 - 291.7) < 0.05
    # seeds from given columns: k rows of W's transpose (r bf16 values) read
    # and copied per logits row
    assert w["seed_columns"]["bytes"] == 64 * 15 * 8 * r * 2 * 2   # 7.9 MB


def test_pair_kernel_row_split():
    """Depths with more than 128 parent rows go to the CTA-pair scorer: all but depth 1."""
    rows = [64 * f for f in bench.frontier_sizes()[:15]]
    assert [m >= bench.PAIR_ROWS_MIN for m in rows] == [False] + [True] * 14
