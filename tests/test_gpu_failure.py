"""Failure detection of the tensor-core kernel, exercised without a GPU fault.

Every wait inside the tensor-core kernel is bounded.  The context's test hook
withholds one hand-off between two warp roles (the first tile's coefficients;
no copy or MMA depends on it), so the epilogue's bounded wait runs out: the call
must return, report STREE_ERR_TIMEOUT in the error word, leave the outputs of
the abandoned tiles untouched, and the next call on the same context must be
exact again.
"""
import pytest
import torch

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_commit, oracle_tree_scan

from gpu_util import assert_close, f64, upload_layer, upload_tree

pytestmark = pytest.mark.gpu

STREE_ERR_TIMEOUT = 7


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_packed_tree_b200 import stree
    return stree


@pytest.mark.parametrize("name,batch", [("m2_2p7b", None), ("serve64", 4)])
def test_bounded_wait_runs_out_and_the_context_recovers(st, name, batch):
    w = wl.make_workload(name, batch=batch, layers=1)
    ctx = st.stree_ctx_create()
    st.stree_ctx_set_kernel(ctx, "tc")
    d, tr = upload_layer(w), upload_tree(w)

    st.stree_ctx_set_wait_limit(ctx, 2_000_000)          # 2 ms
    st.stree_ctx_set_test_fault(ctx, 1)
    y = torch.full_like(d["x"], 7.0)
    h_new = torch.full_like(d["h0"], 7.0)
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                              tr["path"], tr["path_len"], y, h_new)
    status, info = st.stree_sync_check(ctx, raise_on_error=False)
    assert status == STREE_ERR_TIMEOUT, info
    # Every CTA gave up at its first tile: nothing was stored.
    assert torch.all(y == 7.0) and torch.all(h_new == 7.0)

    st.stree_ctx_set_test_fault(ctx, 0)
    st.stree_ctx_set_wait_limit(ctx, 0)
    y2 = torch.empty_like(d["x"])
    h2 = torch.empty_like(d["h0"])
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                              tr["path"], tr["path_len"], y2, h2)
    st.stree_sync_check(ctx)
    f = w.f64(0)
    y_ref = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent, nthreads=8)
    h_ref = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, w.path, w.path_len, nthreads=8)[0]
    assert_close(f64(y2), y_ref, w.dtype, "y after the timeout")
    assert_close(f64(h2), h_ref, w.dtype, "h_new after the timeout")


def test_test_hook_rejects_unknown_values(st):
    ctx = st.stree_ctx_create()
    with pytest.raises(st.StreeError) as e:
        st.stree_ctx_set_test_fault(ctx, 2)
    assert e.value.status == 1
