"""The unrolled-tree baseline (stree_unrolled_scan) against the oracle.

Each root-to-leaf path is scanned as its own sequence, so position k of a path
must carry the oracle's y of the node there (a node's output depends only on its
root path), and each path's final state must equal the oracle's commit of that
path.  Tolerances are the scan's: 1e-4 (fp32) or 2e-2 (bf16) of max|ref|.
"""
import numpy as np
import pytest
import torch

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_commit, oracle_tree_scan

from gpu_util import assert_close, f64, i32, upload_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_packed_tree_b200 import stree
    return stree


def _run(st, w, d, paths, plen):
    b, n_paths, depth = paths.shape
    y = torch.full((b, n_paths, depth, w.nheads, w.headdim), float("nan"), dtype=d["x"].dtype, device="cuda")
    h = torch.full((b, n_paths, w.nheads, w.headdim, w.dstate), float("nan"), device="cuda")
    err = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    st.stree_unrolled_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], i32(paths), i32(plen), y, h,
                           err_out=err)
    torch.cuda.synchronize()
    return y, h, err


@pytest.mark.parametrize("name,batch", [("tiny", None), ("m2_2p7b", None), ("m2_2p7b_16", None), ("hyb8b", 2),
                                        ("serve64", 2), ("wide256", 1)])
def test_unrolled_matches_oracle_node_outputs_and_path_states(st, name, batch):
    w = wl.make_workload(name, batch=batch, layers=1)
    d = upload_layer(w)
    paths, plen = wl.unroll_paths(w.parent)
    y, h, err = _run(st, w, d, paths, plen)
    assert err.tolist() == [0, 0, 0, 0]
    f = w.f64(0)
    y_node = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent, nthreads=8)
    yg, yr, hs, hr = [], [], [], []
    for k in range(paths.shape[1]):
        h_ref = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, np.ascontiguousarray(paths[:, k]),
                              np.ascontiguousarray(plen[:, k]), nthreads=8)[0]
        hs.append(f64(h[:, k]))
        hr.append(h_ref)
        for b in range(w.batch):
            for q in range(plen[b, k]):
                yg.append(f64(y[b, k, q]))
                yr.append(y_node[b, paths[b, k, q]])
    assert_close(np.stack(yg), np.stack(yr), w.dtype, f"{name} unrolled y")
    assert_close(np.stack(hs), np.stack(hr), w.dtype, f"{name} path states")


def test_unrolled_empty_and_invalid_paths(st):
    w = wl.custom_workload([[-1, 0, 0, 1], [-1, 0, 1, 2]], nheads=2, headdim=16, dstate=16, seed=4)
    d = upload_layer(w)
    paths = np.array([[[0, 1, 3], [0, 2, -1]], [[0, 1, 2], [0, 7, -1]]], np.int32)   # node 7 does not exist
    plen = np.array([[3, 0], [3, 2]], np.int32)
    y, h, err = _run(st, w, d, paths, plen)
    assert int(err[0]) == 4 and int(err[1]) == 1
    assert torch.equal(h[0, 1], d["h0"][0])                       # empty path keeps h0
    assert torch.isnan(y[0, 1]).all()                             # ... and writes no y
    assert torch.isnan(h[1, 1]).all() and torch.isnan(y[1, 1]).all()   # invalid path untouched
    assert torch.isfinite(h[1, 0]).all() and torch.isfinite(y[1, 0]).all()
