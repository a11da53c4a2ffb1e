"""The allocation-free fused scan + commit against the context entry point.

stree_tree_scan_commit_noalloc serves callers that may not allocate device
memory where they run the scan (a runtime that owns all device memory through
its own pool, a process at its memory cap, a loop where an allocator call would
synchronise).  It takes its scratch from the library's fixed device array, so
its results must match stree_tree_scan_commit, which uses a context's workspace,
and the fp64 oracle.  Two calls in a row check that leftovers in the shared
array never leak into the next result.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_commit, oracle_tree_scan

from gpu_util import TOL, assert_close, f64, upload_layer, upload_tree

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_packed_tree_b200 import stree
    return stree


def _with_ctx(st, d, tr):
    ctx = st.stree_ctx_create()
    y = torch.empty_like(d["x"])
    h_new = torch.empty_like(d["h0"])
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                              tr["path"], tr["path_len"], y, h_new)
    st.stree_sync_check(ctx)
    st.stree_ctx_destroy(ctx)
    return y, h_new


@pytest.mark.parametrize("name,batch", [("tiny", None), ("m2_2p7b", None), ("hyb8b", None), ("serve64", 4),
                                        ("wide256_chain", 2)])
def test_noalloc_matches_context_entry_point_twice(st, name, batch):
    w = wl.make_workload(name, batch=batch, layers=1)
    d, tr = upload_layer(w), upload_tree(w)
    y_ref, h_ref = _with_ctx(st, d, tr)
    err = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        y = torch.full_like(d["x"], float("nan"))
        h_new = torch.full_like(d["h0"], float("nan"))
        st.stree_tree_scan_commit_noalloc(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                                          tr["path"], tr["path_len"], y, h_new, err_out=err)
        torch.cuda.synchronize()
        assert err.tolist() == [0, 0, 0, 0]
        assert_close(f64(y), f64(y_ref), w.dtype, f"{name} y")
        assert_close(f64(h_new), f64(h_ref), w.dtype, f"{name} h_new")
    # And against the oracle, so that a layout fault of the scratch shared by
    # both calls cannot pass unseen.
    f = w.f64(0)
    y_or = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent, nthreads=8)
    h_or = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, w.path, w.path_len, nthreads=8)[0]
    assert_close(f64(y), y_or, w.dtype, f"{name} y against the oracle")
    assert_close(f64(h_new), h_or, w.dtype, f"{name} h_new against the oracle")


def test_noalloc_batch_zero_is_a_no_op_like_the_context_call(st):
    x = torch.empty((0, 5, 2, 8), device="cuda")
    dt = torch.empty((0, 5, 2), device="cuda")
    B = torch.empty((0, 5, 1, 8), device="cuda")
    h0 = torch.empty((0, 2, 8, 8), device="cuda")
    A = torch.ones(2, device="cuda")
    parent = torch.empty((0, 5), dtype=torch.int32, device="cuda")
    path = torch.empty((0, 0), dtype=torch.int32, device="cuda")        # maxlen 0
    plen = torch.empty((0,), dtype=torch.int32, device="cuda")
    ctx = st.stree_ctx_create()
    st.stree_tree_scan_commit(ctx, x, dt, A, B, B, A, h0, parent, path, plen, torch.empty_like(x),
                              torch.empty_like(h0))
    st.stree_tree_scan_commit_noalloc(x, dt, A, B, B, A, h0, parent, path, plen, torch.empty_like(x),
                                      torch.empty_like(h0))


def test_noalloc_reports_a_bad_path_in_its_error_word(st):
    w = wl.custom_workload([[-1, 0, 0, 1]], nheads=2, headdim=8, dstate=8, seed=2,
                           path=[[0, 2, 3, -1]], path_len=[3])
    d, tr = upload_layer(w), upload_tree(w)
    err = torch.zeros((4,), dtype=torch.int32, device="cuda")
    y = torch.empty_like(d["x"])
    h_new = torch.full_like(d["h0"], 7.0)
    st.stree_tree_scan_commit_noalloc(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                                      tr["path"], tr["path_len"], y, h_new, err_out=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 4
    assert torch.all(h_new == 7.0)


def test_noalloc_rejects_sizes_beyond_its_scratch(st):
    # 65536 sequences of 256 nodes need far more than the 8 MiB of tree scratch.
    x = torch.zeros((16,), device="cuda")
    fn = st._lib.stree_tree_scan_commit_noalloc
    p = x.data_ptr()
    args = [p] * 8 + [256, 1 << 16, 8, 64, 128, 1, 1] + [p, p, 256, p, p, None, None]
    assert fn(*args) == 2
