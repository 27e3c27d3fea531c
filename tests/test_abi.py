"""C-ABI checks that need no GPU: the library loads, exports what the header
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

import speculative_decoding_draft_07_b200 as pct

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "pctree.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    L = pct.lib()
    names = _declared()
    assert "pct_tree_build" in names and "tree_verify_accept" in names
    for n in names:
        assert hasattr(L, n), n
    assert sorted(names) == sorted(pct.EXPORTED)
    assert "sm_100a" in pct.version()


def _desc(**kw):
    base = dict(batch=2, depth=3, vocab=1024, rank=64, k=4, beam=8, n_nodes=16,
                logits_dtype=pct.PCT_BF16, markov_dtype=pct.PCT_BF16)
    base.update(kw)
    return pct.build_desc(**base)


@pytest.mark.parametrize("bad", [dict(batch=0), dict(depth=0), dict(depth=65), dict(k=0), dict(k=17),
                                 dict(vocab=3, k=4), dict(rank=0), dict(rank=257), dict(beam=0),
                                 dict(beam=257), dict(beam=128, k=16), dict(n_nodes=0),
                                 dict(n_nodes=4097), dict(depth=64, beam=65),
                                 dict(logits_dtype=7), dict(markov_dtype=-1)])
def test_build_rejects_bad_descriptors(bad):
    d = _desc(**bad)
    assert pct.lib().pct_tree_build_workspace(ctypes.byref(d)) == 0
    dummy = ctypes.c_void_p(256)
    args = [dummy] * 10
    rc = pct.lib().pct_tree_build(ctypes.byref(d), *args, dummy, 1 << 30, None)
    assert rc == pct.PCT_EINVAL


def test_bf16_markov_needs_vocab_multiple_of_8():
    d = _desc(vocab=1001)
    dummy = ctypes.c_void_p(256)
    rc = pct.lib().pct_tree_build(ctypes.byref(d), *([dummy] * 10), dummy, 1 << 30, None)
    assert rc == pct.PCT_EUNSUPPORTED
    d = _desc(vocab=1001, markov_dtype=pct.PCT_F32, logits_dtype=pct.PCT_F32)
    assert pct.lib().pct_tree_build_workspace(ctypes.byref(d)) > 0


def test_vocab_above_2_pow_22_unsupported():
    d = _desc(vocab=(1 << 22) + 8)
    dummy = ctypes.c_void_p(256)
    rc = pct.lib().pct_tree_build(ctypes.byref(d), *([dummy] * 10), dummy, 1 << 30, None)
    assert rc == pct.PCT_EUNSUPPORTED


def test_null_pointers_rejected_before_device_check():
    d = _desc()
    rc = pct.lib().pct_tree_build(ctypes.byref(d), *([None] * 10), None, 0, None)
    assert rc == pct.PCT_EINVAL


def test_workspace_grows_with_problem():
    small = pct.lib().pct_tree_build_workspace(ctypes.byref(_desc()))
    big = pct.lib().pct_tree_build_workspace(ctypes.byref(_desc(batch=64, depth=15, beam=32, vocab=151936, rank=256, k=8, n_nodes=256)))
    assert 0 < small < big
    c = pct.cadd_desc(64, 15, 151936, 512, pct.PCT_BF16, 1.0, 2.0, 1e-4, 5e-3, 1e-5)
    assert pct.lib().cadd_tree_grow_workspace(ctypes.byref(c)) >= 64 * 15 * 511 * 8
    assert pct.lib().tree_verify_accept_workspace(64, 256) >= 64 * 4


def test_cadd_workspace_holds_the_segment_buffers():
    """bf16 rows with V % 8 == 0 take the segmented row pass: V / 8 16-byte groups per
    row cut into ceil(groups / 1280) segments, each with a partial (max, sum) and a
    tight threshold, and two bitmaps of one bit per group (rows padded to whole
    32-byte sectors); fp32 rows (single-block row pass) need none of it."""
    def ws(dtype, V):
        c = pct.cadd_desc(64, 15, V, 512, dtype, 1.0, 2.0, 1e-4, 5e-3, 1e-5)
        return pct.lib().cadd_tree_grow_workspace(ctypes.byref(c))
    rows, V = 64 * 15, 151936
    S = -(-(V // 8) // 1280)
    assert S == 15
    words = -(-(V // 8) // 32)
    words += -words % 8
    assert words == 600
    bf, f32 = ws(pct.PCT_BF16, V), ws(pct.PCT_F32, V)
    assert bf - f32 >= rows * S * (8 + 4) + rows * 4 + 2 * rows * words * 4
    assert ws(pct.PCT_BF16, V + 4) == ws(pct.PCT_F32, V + 4)     # V % 8 != 0: no segments


@pytest.mark.parametrize("bad", [dict(n_max=0), dict(n_max=1025), dict(depth=64), dict(c=-1e-3),
                                 dict(e=-1e-6), dict(C_d=float("nan")), dict(logits_dtype=3)])
def test_cadd_rejects_bad_descriptors(bad):
    base = dict(batch=4, depth=15, vocab=1000, n_max=64, logits_dtype=pct.PCT_BF16, C_d=1.0,
                a=2.0, b=1e-4, c=5e-3, e=1e-5)
    base.update(bad)
    c = pct.cadd_desc(**base)
    assert pct.lib().cadd_tree_grow_workspace(ctypes.byref(c)) == 0
    dummy = ctypes.c_void_p(256)
    rc = pct.lib().cadd_tree_grow(ctypes.byref(c), *([dummy] * 10), dummy, 1 << 30, None)
    assert rc == pct.PCT_EINVAL


def test_one_pass_entry_points_reject_bad_arguments():
    """pct_tree_build_seeded without seeds or with a misaligned Wt, pct_markov_transpose
    with a bad shape, cadd_tree_grow_topk with top_k outside 1..32 or no output:
    PCT_EINVAL on the host, before the device is looked at."""
    L = pct.lib()
    dummy = ctypes.c_void_p(256)
    d = _desc()
    rc = L.pct_tree_build_seeded(ctypes.byref(d), dummy, dummy, dummy, dummy, None, None,
                                 *([dummy] * 6), dummy, 1 << 30, None)
    assert rc == pct.PCT_EINVAL
    # Wt needs bf16 Markov parameters and 16-byte alignment
    rc = L.pct_tree_build_seeded(ctypes.byref(d), dummy, dummy, dummy, dummy,
                                 ctypes.c_void_p(264), dummy, *([dummy] * 6), dummy, 1 << 30, None)
    assert rc == pct.PCT_EINVAL
    assert L.pct_markov_rank_pad(1) == 64 and L.pct_markov_rank_pad(256) == 256
    assert L.pct_markov_rank_pad(0) == 0 and L.pct_markov_rank_pad(257) == 0
    assert L.pct_markov_transpose(1004, 64, dummy, dummy, None) == pct.PCT_EINVAL   # V % 8
    assert L.pct_markov_transpose(1024, 0, dummy, dummy, None) == pct.PCT_EINVAL
    assert L.pct_markov_transpose(1024, 64, None, dummy, None) == pct.PCT_EINVAL
    c = pct.cadd_desc(batch=4, depth=15, vocab=1000, n_max=64, logits_dtype=pct.PCT_BF16,
                      C_d=1.0, a=2.0, b=1e-4, c=5e-3, e=1e-5)
    for k, out in ((0, dummy), (33, dummy), (-1, dummy), (8, None)):
        rc = L.cadd_tree_grow_topk(ctypes.byref(c), dummy, dummy, dummy, k, *([dummy] * 6), out,
                                   dummy, dummy, 1 << 30, None)
        assert rc == pct.PCT_EINVAL, k


def test_verify_and_mask_reject_bad_shapes():
    L = pct.lib()
    dummy = ctypes.c_void_p(256)
    assert L.tree_ancestor_mask(0, 16, dummy, dummy, dummy, dummy, None) == pct.PCT_EINVAL
    assert L.tree_ancestor_mask(2, 4097, dummy, dummy, dummy, dummy, None) == pct.PCT_EINVAL
    assert L.tree_verify_accept_workspace(2, 0) == 0
    rc = L.tree_verify_accept(2, 16, 1000, 0, dummy, dummy, dummy, dummy, pct.PCT_BF16, dummy,
                              dummy, dummy, dummy, dummy, dummy, 1 << 20, None)
    assert rc == pct.PCT_EINVAL
    rc = L.tree_verify_accept(2, 16, 1000, 4, dummy, dummy, dummy, dummy, 5, dummy,
                              dummy, dummy, dummy, dummy, dummy, 1 << 20, None)
    assert rc == pct.PCT_EINVAL


def test_trace_api_roundtrip_without_launches():
    prev = pct.trace_enable(True)
    pct.trace_reset()
    assert pct.trace_read() == {}
    pct.trace_enable(prev)


def test_binding_refuses_cpu_tensors():
    import torch
    L = torch.zeros((1, 2, 64), dtype=torch.bfloat16)
    with pytest.raises((ValueError, pct.PctError)):
        pct.pct_tree_build(L, torch.zeros(1, dtype=torch.int64), torch.zeros((64, 16), dtype=torch.bfloat16),
                           torch.zeros((16, 64), dtype=torch.bfloat16), 2, 2, 4)
