"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Bars: tree masks, depths and resolved paths bit-exact; y and h_new within
max|err| <= 1e-4 max|ref| (fp32 inputs) or 2e-2 max|ref| (bf16 inputs, fp32
accumulation); zero NaN/Inf.  Small workloads are compared element by element;
the full-size workloads, in the launch configuration the benchmark times, are
compared on sampled (sequence, head) units that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_build_tree, oracle_commit, oracle_tree_scan

from gpu_util import TOL, assert_close, f64, i32, to_dev, upload_layer, upload_tree

pytestmark = pytest.mark.gpu

KERNELS = ["simt", "tc", "small"]


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_packed_tree_b200 import stree
    return stree


def _ctx(st, kernel):
    ctx = st.stree_ctx_create()
    st.stree_ctx_set_kernel(ctx, kernel)
    return ctx


def _run_fused(st, ctx, w, layer, d, tr):
    y = torch.empty_like(d["x"])
    h_new = torch.empty_like(d["h0"])
    try:
        st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"],
                                  tr["parent"], tr["path"], tr["path_len"], y, h_new)
    except st.StreeError as e:
        if e.status == 2:
            pytest.skip("shape not supported by this kernel")
        raise
    st.stree_sync_check(ctx)
    return y, h_new


def _oracle(w, layer=0):
    f = w.f64(layer)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent, nthreads=8)
    h, ok, leaf = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, w.path, w.path_len, nthreads=8)
    return y, h


SMALL = [("tiny", None, None), ("m2_2p7b", None, None), ("m2_2p7b_16", None, None),
         ("hyb8b", None, None), ("serve64", 3, 1), ("wide256", 2, 1), ("wide256_chain", 1, 1)]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name,batch,layers", SMALL)
def test_fused_scan_commit_matches_oracle(st, kernel, name, batch, layers):
    w = wl.make_workload(name, batch=batch, layers=layers)
    ctx = _ctx(st, kernel)
    d, tr = upload_layer(w), upload_tree(w)
    y, h_new = _run_fused(st, ctx, w, 0, d, tr)
    y_ref, h_ref = _oracle(w)
    assert_close(f64(y), y_ref, w.dtype, f"{name} y")
    assert_close(f64(h_new), h_ref, w.dtype, f"{name} h_new")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name", ["tiny", "hyb8b"])
def test_separate_scan_then_commit(st, kernel, name):
    w = wl.make_workload(name)
    ctx = _ctx(st, kernel)
    d, tr = upload_layer(w), upload_tree(w)
    y = torch.empty_like(d["x"])
    h_new = torch.empty_like(d["h0"])
    try:
        st.stree_tree_scan(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"], y)
    except st.StreeError as e:
        if e.status == 2:
            pytest.skip("shape not supported by this kernel")
        raise
    st.stree_commit(ctx, tr["path"], tr["path_len"], h_new)
    st.stree_sync_check(ctx)
    y_ref, h_ref = _oracle(w)
    assert_close(f64(y), y_ref, w.dtype, "y")
    assert_close(f64(h_new), h_ref, w.dtype, "h_new")


@pytest.mark.parametrize("name", ["tiny", "m2_2p7b", "hyb8b", "serve64", "wide256", "wide256_chain"])
def test_tree_masks_and_paths_bit_exact(st, name):
    w = wl.make_workload(name, layers=1)
    ctx = st.stree_ctx_create()
    tr = upload_tree(w)
    b, T = w.parent.shape
    W = (T + 31) // 32
    anc = torch.zeros((b, T, W), dtype=torch.int32, device="cuda")
    depth = torch.zeros((b, T), dtype=torch.int32, device="cuda")
    st.stree_build_tree(ctx, tr["parent"], anc, depth)
    leaf = torch.zeros((b,), dtype=torch.int32, device="cuda")
    st.stree_resolve_path(ctx, tr["path"], tr["path_len"], leaf)
    st.stree_sync_check(ctx)
    anc_ref, depth_ref, ok = oracle_build_tree(w.parent)
    assert np.array_equal(anc.cpu().numpy().view(np.uint32), anc_ref)
    assert np.array_equal(depth.cpu().numpy(), depth_ref)
    expect_leaf = np.asarray([w.path[i, w.path_len[i] - 1] if w.path_len[i] else -1 for i in range(b)])
    assert np.array_equal(leaf.cpu().numpy(), expect_leaf)


def _unit_f64(w, layer, b, h):
    """fp64 inputs of one (sequence, head) unit, as a one-head, one-group problem."""
    L = w.layers[layer]
    g = h // (w.nheads // w.ngroups)
    io = w.dtype
    return dict(
        x=wl.stored_to_f64(L.x[b:b + 1, :, h:h + 1], io), dt=wl.stored_to_f64(L.dt[b:b + 1, :, h:h + 1], io),
        A=L.A[h:h + 1].astype(np.float64), D=L.D[h:h + 1].astype(np.float64),
        B=wl.stored_to_f64(L.B[b:b + 1, :, g:g + 1], io), C=wl.stored_to_f64(L.C[b:b + 1, :, g:g + 1], io),
        h0=L.h0[b:b + 1, h:h + 1].astype(np.float64))


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name", ["m2_2p7b", "hyb8b", "serve64", "wide256", "wide256_chain"])
def test_full_size_sampled_units(st, kernel, name):
    """Full sizes (all layers), one fused call per layer as the benchmark runs them."""
    w = wl.make_workload(name)
    ctx = _ctx(st, kernel)
    tr = upload_tree(w)
    rng = np.random.default_rng(77)
    st.stree_build_tree(ctx, tr["parent"])
    for layer in range(w.nlayers):
        d = upload_layer(w, layer)
        y = torch.empty_like(d["x"])
        h_new = torch.empty_like(d["h0"])
        try:
            st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], None,
                                      tr["path"], tr["path_len"], y, h_new)
        except st.StreeError as e:
            if e.status == 2:
                pytest.skip("shape not supported by this kernel")
            raise
        st.stree_sync_check(ctx)
        assert torch.isfinite(y.float()).all() and torch.isfinite(h_new).all()
        units = [(int(rng.integers(w.batch)), int(rng.integers(w.nheads))) for _ in range(6)]
        units += [(0, 0), (w.batch - 1, w.nheads - 1)]
        ys, yr, hs, hr = [], [], [], []
        for (b, h) in units:
            u = _unit_f64(w, layer, b, h)
            par = w.parent[b:b + 1]
            yr.append(oracle_tree_scan(u["x"], u["dt"], u["A"], u["B"], u["C"], u["D"], u["h0"], par))
            hr.append(oracle_commit(u["x"], u["dt"], u["A"], u["B"], u["h0"], par,
                                    w.path[b:b + 1], w.path_len[b:b + 1])[0])
            ys.append(f64(y[b:b + 1, :, h:h + 1]))
            hs.append(f64(h_new[b:b + 1, h:h + 1]))
        assert_close(np.stack(ys), np.stack(yr), w.dtype, f"{name} layer {layer} y")
        assert_close(np.stack(hs), np.stack(hr), w.dtype, f"{name} layer {layer} h_new")


# ----------------------------------------------------------------------------- edge cases


EDGE = [
    # (parent rows, H, P, N, G, dtype)
    ([[-1]], 2, 8, 8, 1, "f32"),                                              # one node
    ([[-1, 0]], 1, 8, 16, 1, "f32"),                                          # one edge
    ([wl.chain_tree(33).tolist()], 2, 16, 24, 1, "f32"),                      # ragged T, deep
    ([wl.random_tree(np.random.default_rng(1), 100, max_depth=12).tolist()] * 2, 4, 40, 32, 2, "f32"),
    ([wl.random_tree(np.random.default_rng(2), 256, max_depth=20).tolist()], 2, 8, 256, 1, "f32"),  # max T, max N
    ([wl.random_tree(np.random.default_rng(3), 70, max_depth=9).tolist()], 3, 256, 8, 1, "f32"),   # max P
    ([wl.random_tree(np.random.default_rng(4), 45, max_depth=6).tolist()] * 3, 8, 64, 128, 4, "bf16"),
    ([wl.random_tree(np.random.default_rng(5), 130, max_depth=15).tolist()], 4, 128, 128, 1, "bf16"),
]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("case", range(len(EDGE)))
def test_edge_shapes(st, kernel, case):
    parent, H, P, N, G, dtype = EDGE[case]
    w = wl.custom_workload(parent, nheads=H, headdim=P, dstate=N, ngroups=G, dtype=dtype, seed=case,
                           h0_std=1.0 if dtype == "f32" else 0.1)
    ctx = _ctx(st, kernel)
    d, tr = upload_layer(w), upload_tree(w)
    y, h_new = _run_fused(st, ctx, w, 0, d, tr)
    y_ref, h_ref = _oracle(w)
    assert_close(f64(y), y_ref, dtype, "y")
    assert_close(f64(h_new), h_ref, dtype, "h_new")


def test_batch_zero_is_a_no_op(st):
    ctx = st.stree_ctx_create()
    x = torch.empty((0, 5, 2, 8), device="cuda")
    dt = torch.empty((0, 5, 2), device="cuda")
    B = torch.empty((0, 5, 1, 8), device="cuda")
    h0 = torch.empty((0, 2, 8, 8), device="cuda")
    A = torch.ones(2, device="cuda")
    parent = torch.empty((0, 5), dtype=torch.int32, device="cuda")
    path = torch.empty((0, 5), dtype=torch.int32, device="cuda")
    plen = torch.empty((0,), dtype=torch.int32, device="cuda")
    st.stree_tree_scan_commit(ctx, x, dt, A, B, B, A, h0, parent, path, plen, torch.empty_like(x), torch.empty_like(h0))
    assert st.stree_sync_check(ctx)[0] == 0


def test_empty_path_and_in_place_commit(st):
    w = wl.make_workload("hyb8b")
    w.path_len[1] = 0
    w.path[1] = -1
    ctx = st.stree_ctx_create()
    d, tr = upload_layer(w), upload_tree(w)
    h0_orig = d["h0"].clone()
    y = torch.empty_like(d["x"])
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                              tr["path"], tr["path_len"], y, d["h0"])      # h_new aliases h0
    st.stree_sync_check(ctx)
    y_ref, h_ref = _oracle(w)
    assert_close(f64(y), y_ref, w.dtype, "y")
    assert_close(f64(d["h0"]), h_ref, w.dtype, "h_new in place")
    assert torch.equal(d["h0"][1], h0_orig[1])                           # empty path keeps h0 exactly


def test_identical_siblings_bitwise_equal(st):
    parent = np.asarray([[-1, 0, 0, 1, 2]], np.int32)
    w = wl.custom_workload(parent, nheads=4, headdim=64, dstate=128, dtype="bf16", seed=3, h0_std=0.1)
    L = w.layers[0]
    for arr in (L.x, L.dt, L.B, L.C):
        arr[:, 2] = arr[:, 1]
        arr[:, 4] = arr[:, 3]
    ctx = st.stree_ctx_create()
    d, tr = upload_layer(w), upload_tree(w)
    y, _ = _run_fused(st, ctx, w, 0, d, tr)
    assert torch.equal(y[:, 1], y[:, 2]) and torch.equal(y[:, 3], y[:, 4])


@pytest.mark.parametrize("bad", [[0, 0, 1, 1], [-1, 2, 0, 1], [-1, 0, -1, 1], [-1, 0, 9, 1]])
def test_invalid_tree_latches_error_and_skips(st, bad):
    w = wl.custom_workload([[-1, 0, 0, 1], [-1, 0, 0, 1]], nheads=2, headdim=8, dstate=8, seed=1)
    w.parent[1] = bad
    ctx = st.stree_ctx_create()
    d, tr = upload_layer(w), upload_tree(w)
    y = torch.full_like(d["x"], 7.0)
    h_new = torch.full_like(d["h0"], 7.0)
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                              tr["path"], tr["path_len"], y, h_new)
    status, info = st.stree_sync_check(ctx, raise_on_error=False)
    assert status == 3 and info[1] == 1
    assert torch.all(y[1] == 7.0) and torch.all(h_new[1] == 7.0)      # skipped
    assert torch.isfinite(y[0]).all() and not torch.all(y[0] == 7.0)


@pytest.mark.parametrize("kernel", ["tc", "small"])
@pytest.mark.parametrize("rebuild", [True, False], ids=["parent", "ctx_tree"])
@pytest.mark.parametrize("bad", [[-1, 0, 0, 0, 1, 1, 2, 2, 3, 3, 4, 5, 6, 7, 15],
                                 [0, 0, 0, 0, 1, 1, 2, 2, 3, 3, 4, 5, 6, 7, 8],
                                 [-1, 0, 0, 0, 1, 1, 2, 2, 3, 3, 4, 5, 6, 13, 8]])
def test_invalid_tree_skips_only_that_sequence(st, kernel, rebuild, bad):
    """Tensor-core and small-batch kernels (bf16, dstate 128) with an invalid middle
    sequence: its masks built in-kernel from parent[] (parent passed; the kernel
    reports the tree) or read from the context's tree (built and reported by an
    earlier call).  The kernel writes neither y nor h_new of that sequence and the
    others stay exact."""
    par = list(wl.M2_PARENT_15)
    w = wl.custom_workload([par, par, par], nheads=4, headdim=64, dstate=128, dtype="bf16", seed=5, h0_std=0.1)
    w.parent[1] = bad
    ctx = _ctx(st, kernel)
    d, tr = upload_layer(w), upload_tree(w)
    y = torch.full_like(d["x"], 7.0)
    h_new = torch.full_like(d["h0"], 7.0)
    if not rebuild:
        st.stree_build_tree(ctx, tr["parent"])
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"],
                              tr["parent"] if rebuild else None, tr["path"], tr["path_len"], y, h_new)
    status, info = st.stree_sync_check(ctx, raise_on_error=False)
    assert status == 3 and info[1] == 1
    assert torch.all(y[1] == 7.0) and torch.all(h_new[1] == 7.0)
    f = w.f64(0)
    keep = [0, 2]
    sel = {k: (f[k][keep] if k in ("x", "dt", "B", "C", "h0") else f[k]) for k in f}
    yr = oracle_tree_scan(sel["x"], sel["dt"], sel["A"], sel["B"], sel["C"], sel["D"], sel["h0"], w.parent[keep])
    hr = oracle_commit(sel["x"], sel["dt"], sel["A"], sel["B"], sel["h0"], w.parent[keep], w.path[keep],
                       w.path_len[keep])[0]
    assert_close(f64(y[keep]), yr, "bf16", "y of the valid sequences")
    assert_close(f64(h_new[keep]), hr, "bf16", "h_new of the valid sequences")


@pytest.mark.parametrize("path,plen", [([1, 3, -1, -1], 2), ([0, 2, 3, -1], 3), ([0, 1, 3, 3], 5),
                                       ([0, 1, 3, 9], 4), ([0, 0, -1, -1], 2), ([0, 1, 3, -1], -1)])
def test_invalid_path_latches_error(st, path, plen):
    w = wl.custom_workload([[-1, 0, 0, 1]], nheads=2, headdim=8, dstate=8, seed=2,
                           path=[path], path_len=[plen])
    ctx = st.stree_ctx_create()
    d, tr = upload_layer(w), upload_tree(w)
    y = torch.empty_like(d["x"])
    h_new = torch.full_like(d["h0"], 7.0)
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                              tr["path"], tr["path_len"], y, h_new)
    status, info = st.stree_sync_check(ctx, raise_on_error=False)
    assert status == 4
    assert torch.all(h_new == 7.0)
    leaf = torch.zeros(1, dtype=torch.int32, device="cuda")
    st.stree_resolve_path(ctx, tr["path"], tr["path_len"], leaf)
    st.stree_sync_check(ctx, raise_on_error=False)
    assert int(leaf[0]) == -2


def test_host_argument_checks(st):
    ctx = st.stree_ctx_create()
    x = torch.zeros((1, 4, 2, 12), device="cuda")               # headdim 12: not a multiple of 8
    dt = torch.zeros((1, 4, 2), device="cuda")
    B = torch.zeros((1, 4, 1, 16), device="cuda")
    h0 = torch.zeros((1, 2, 12, 16), device="cuda")
    A = torch.zeros(2, device="cuda")
    parent = i32([[-1, 0, 0, 1]])
    with pytest.raises(st.StreeError) as e:
        st.stree_tree_scan(ctx, x, dt, A, B, B, A, h0, parent, torch.empty_like(x))
    assert e.value.status == 2
    x2 = torch.zeros((1, 4, 2, 16), device="cuda")
    h02 = torch.zeros((1, 2, 16, 16), device="cuda")
    with pytest.raises(st.StreeError) as e:                      # parent=None before any tree
        st.stree_tree_scan(ctx, x2, dt, A, B, B, A, h02, None, torch.empty_like(x2))
    assert e.value.status == 8
    with pytest.raises(st.StreeError) as e:                      # commit before any scan
        st.stree_commit(ctx, i32([[0]]), i32([1]), torch.empty_like(h02))
    assert e.value.status == 8
    big = i32([[-1] + list(range(256))])                         # 257 nodes
    with pytest.raises(st.StreeError) as e:
        st.stree_build_tree(ctx, big)
    assert e.value.status == 2


@pytest.mark.parametrize("kernel", ["tc", "small"])
@pytest.mark.parametrize("path,plen", [([1, 3, -1, -1], 2), ([0, 2, 3, -1], 3), ([0, 1, 3, 3], 5),
                                       ([0, 1, 4, 9], 4), ([0, 0, -1, -1], 2), ([0, 1, 3, -1], -1)])
def test_invalid_path_on_the_fused_kernels(st, kernel, path, plen):
    """An invalid accepted path on the tensor-core and small-batch kernels: the
    error is latched, h_new of that sequence stays untouched, y is still exact."""
    par = [-1, 0, 0, 1, 1, 2]
    w = wl.custom_workload([par, par], nheads=2, headdim=64, dstate=128, dtype="bf16", seed=9, h0_std=0.1,
                           path=[[0, 1, 3, -1], path], path_len=[3, plen])
    ctx = _ctx(st, kernel)
    d, tr = upload_layer(w), upload_tree(w)
    y = torch.empty_like(d["x"])
    h_new = torch.full_like(d["h0"], 7.0)
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                              tr["path"], tr["path_len"], y, h_new)
    status, info = st.stree_sync_check(ctx, raise_on_error=False)
    assert status == 4 and info[1] == 1
    assert torch.all(h_new[1] == 7.0)
    f = w.f64(0)
    assert_close(f64(y), oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent),
                 "bf16", "y")
    h_ref = oracle_commit(f["x"][:1], f["dt"][:1], f["A"], f["B"][:1], f["h0"][:1], w.parent[:1], w.path[:1],
                          w.path_len[:1])[0]
    assert_close(f64(h_new[:1]), h_ref, "bf16", "h_new of the valid sequence")


@pytest.mark.parametrize("kernel", ["tc", "small"])
def test_fused_call_leaves_the_tree_in_the_context(st, kernel):
    """With parent[] the fused kernels rebuild the tree themselves (no builder launch)
    and leave it in the context: the path resolver and a later parent=NULL layer use it."""
    w = wl.make_workload("hyb8b" if kernel == "small" else "serve64", batch=3, layers=2)
    ctx = _ctx(st, kernel)
    tr = upload_tree(w)
    n0 = st.stree_ctx_launch_count(ctx)
    outs = []
    for layer in range(2):
        d = upload_layer(w, layer)
        y = torch.empty_like(d["x"])
        h_new = torch.empty_like(d["h0"])
        st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"],
                                  tr["parent"] if layer == 0 else None, tr["path"], tr["path_len"], y, h_new)
        outs.append((y, h_new))
    assert st.stree_ctx_launch_count(ctx) - n0 == 2                     # one kernel per layer
    leaf = torch.zeros((w.batch,), dtype=torch.int32, device="cuda")
    st.stree_resolve_path(ctx, tr["path"], tr["path_len"], leaf)
    st.stree_sync_check(ctx)
    expect_leaf = [w.path[i, w.path_len[i] - 1] if w.path_len[i] else -1 for i in range(w.batch)]
    assert leaf.tolist() == expect_leaf
    for layer, (y, h_new) in enumerate(outs):
        yr, hr = _oracle(w, layer)
        assert_close(f64(y), yr, w.dtype, f"layer {layer} y")
        assert_close(f64(h_new), hr, w.dtype, f"layer {layer} h_new")


@pytest.mark.parametrize("name,batch", [("tiny", None), ("m2_2p7b", None), ("serve64", 4), ("wide256", 2),
                                        ("wide256_chain", 2)])
def test_commit_alone_matches_oracle(st, name, batch):
    """stree_commit (the streaming replay kernel) after a scan: every element of h_new,
    including paths longer than one staging chunk (the chain) and an empty path."""
    w = wl.make_workload(name, batch=batch, layers=1)
    if w.batch > 1:
        w.path_len[1] = 0
        w.path[1] = -1
    ctx = st.stree_ctx_create()
    d, tr = upload_layer(w), upload_tree(w)
    y = torch.empty_like(d["x"])
    st.stree_tree_scan(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"], y)
    h_new = torch.empty_like(d["h0"])
    st.stree_commit(ctx, tr["path"], tr["path_len"], h_new)
    st.stree_sync_check(ctx)
    f = w.f64(0)
    h_ref = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, w.path, w.path_len, nthreads=8)[0]
    assert_close(f64(h_new), h_ref, w.dtype, f"{name} h_new")
    if w.batch > 1:
        assert torch.equal(h_new[1], d["h0"][1])                         # empty path keeps h0 exactly
    st.stree_commit(ctx, tr["path"], tr["path_len"], d["h0"])            # in place
    st.stree_sync_check(ctx)
    assert_close(f64(d["h0"]), h_ref, w.dtype, f"{name} h_new in place")


def test_commit_alone_reports_a_bad_path(st):
    w = wl.custom_workload([[-1, 0, 0, 1], [-1, 0, 0, 1]], nheads=2, headdim=8, dstate=8, seed=2,
                           path=[[0, 1, 3, -1], [0, 2, 3, -1]], path_len=[3, 3])
    ctx = st.stree_ctx_create()
    d, tr = upload_layer(w), upload_tree(w)
    st.stree_tree_scan(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"],
                       torch.empty_like(d["x"]))
    h_new = torch.full_like(d["h0"], 7.0)
    st.stree_commit(ctx, tr["path"], tr["path_len"], h_new)
    status, info = st.stree_sync_check(ctx, raise_on_error=False)
    assert status == 4 and info[1] == 1 and info[2] == 1
    assert torch.all(h_new[1] == 7.0) and not torch.all(h_new[0] == 7.0)
