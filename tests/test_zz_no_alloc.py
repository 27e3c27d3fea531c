"""Allocation-free verification entry point (tree_verify_accept_noalloc).

Some callers cannot allocate device memory: a component inside a serving
runtime that reserves all device memory up front and hands its parts only their
input and output buffers, or code on a latency-critical path where a cudaMalloc
(which may synchronise the device) is not acceptable. For them the library
offers a variant of tree_verify_accept that takes no workspace: its scratch (one
arrival counter per request) lives in a static device array inside the library.

This test calls the variant through the C ABI twice in a row and checks that
both calls give exactly the results of the workspace entry point (verification
outputs are integers, so the comparison is exact). It sits in a file of its own
that pytest collects last and depends on no other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import speculative_decoding_draft_07_b200 as pct
import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(tok, par, cnt, T, max_depth, outs):
    batch, n_stride = tok.shape
    code = pct.PCT_BF16 if T.dtype == torch.bfloat16 else pct.PCT_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return pct.lib().tree_verify_accept_noalloc(
        batch, n_stride, T.shape[2], max_depth, _ptr(tok), _ptr(par), _ptr(cnt), _ptr(T), code,
        _ptr(outs["argmax"]), _ptr(outs["accept_len"]), _ptr(outs["accept_path"]),
        _ptr(outs["correction"]), _ptr(outs["status"]), stream)


def _case(batch, n_stride, V, D, seed, dtype="bf16", counts=None):
    tok, par, dep, cnt = workloads.random_tree(batch, n_stride, V, D, seed=seed, counts=counts)
    T = workloads.target_logits(batch, n_stride, V, 2.0, seed=seed + 1, dtype=dtype)
    workloads.plant_path(T, tok, par, cnt, seed=seed + 2, length_range=(0, 10))
    dtok, dpar, dcnt = (torch.from_numpy(x).to(DEV) for x in (tok, par, cnt))
    return dtok, dpar, dcnt, T.to(DEV)


def _check_against_workspace_entry_point(dtok, dpar, dcnt, T, D, calls=2, label=""):
    """Calls the allocation-free entry point `calls` times in a row; every call
    must give exactly the workspace entry point's outputs, status included."""
    ref = pct.tree_verify_accept(dtok, dpar, dcnt, T, max_depth=D)
    torch.cuda.synchronize()
    want = {"argmax": ref.argmax, "accept_len": ref.accept_len, "accept_path": ref.accept_path,
            "correction": ref.correction, "status": ref.status}
    for call in range(calls):
        outs = {k: torch.full_like(v, -7) for k, v in want.items()}
        rc = _noalloc(dtok, dpar, dcnt, T, D, outs)
        assert rc == pct.PCT_OK, f"{label} call {call} returned {rc}"
        torch.cuda.synchronize()
        for k, v in want.items():
            np.testing.assert_array_equal(outs[k].cpu().numpy(), v.cpu().numpy(),
                                          err_msg=f"{label} call {call}: {k}")
    return want


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    dtok, dpar, dcnt, T = _case(7, 90, 3000, 8, seed=77)
    _check_against_workspace_entry_point(dtok, dpar, dcnt, T, 8, label="bf16 V=3000")


@pytest.mark.parametrize("dtype,V", [("f32", 3001), ("f32", 2048), ("bf16", 1999)])
def test_noalloc_other_row_layouts(dtype, V):
    """fp32 rows and rows whose length is not a multiple of the 16-byte vector
    take the other forms of the row scan."""
    dtok, dpar, dcnt, T = _case(5, 40, V, 6, seed=V, dtype=dtype)
    _check_against_workspace_entry_point(dtok, dpar, dcnt, T, 6, label=f"{dtype} V={V}")


def test_noalloc_call_after_flagged_errors():
    """A call whose requests carry bad counts and bad parents (the kernel flags
    them in the status words) followed by a clean call: the shared counters and
    the status words start afresh, so the clean call matches too."""
    dtok, dpar, dcnt, T = _case(6, 50, 2048, 6, seed=5, counts=[50, 20, 33, 12, 40, 1])
    bad_cnt = dcnt.clone()
    bad_cnt[1] = 51                 # above n_stride
    bad_cnt[3] = 0                  # below 1
    bad_par = dpar.clone()
    bad_par[4, 7] = 9               # not an earlier node (request 4 has 40 nodes)
    want = _check_against_workspace_entry_point(dtok, bad_par, bad_cnt, T, 6, calls=1,
                                                label="flagged")
    st = want["status"].cpu().numpy()
    assert st[1] & pct.DEV_BAD_COUNT and st[3] & pct.DEV_BAD_COUNT and st[4] & pct.DEV_BAD_PARENT
    want = _check_against_workspace_entry_point(dtok, dpar, dcnt, T, 6, calls=1, label="clean")
    assert (want["status"].cpu().numpy() == 0).all()


def test_noalloc_rejects_batch_above_its_limit():
    dummy = torch.zeros(16, dtype=torch.int32, device=DEV)
    outs = {k: dummy for k in ("argmax", "accept_len", "accept_path", "correction", "status")}
    T = torch.zeros((1, 1, 16), dtype=torch.bfloat16, device=DEV)
    L = pct.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = _ptr(dummy)
    rc = L.tree_verify_accept_noalloc(4097, 1, 16, 1, p, p, p, _ptr(T), pct.PCT_BF16, p, p, p, p, p,
                                      stream)
    assert rc == pct.PCT_EUNSUPPORTED
