"""The gated delta rule over the packed tree (stree_gdn_tree_scan_commit) against
the fp64 oracle: every node's output and the committed state, element by element,
at the tolerances of the scan (1e-4 max|ref| for fp32 inputs, 2e-2 for bf16);
invalid trees and paths, the empty path, the in-place commit and the call
without a commit; the erase strength apart from the write strength (random, and
zero: gated linear attention).  bf16 with d_v = 128 and up to 64 nodes runs the
tensor-core kernel, every other shape the CUDA-core one; both are covered."""
import numpy as np
import pytest
import torch

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_gdn_commit, oracle_gdn_tree

from gpu_util import assert_close, f64, i32, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_packed_tree_b200 import stree
    return stree


def _upload(g):
    d = {k: to_dev(getattr(g, k), g.dtype) for k in ("q", "k", "v")}
    d.update({k: to_dev(getattr(g, k), "f32") for k in ("alpha", "beta", "S0")})
    d.update({"parent": i32(g.parent), "path": i32(g.path), "path_len": i32(g.path_len)})
    return d


def _run(st, g, d, commit=True, S_new=None, erase=None):
    o = torch.full_like(d["v"], 7.0)
    if commit and S_new is None:
        S_new = torch.full_like(d["S0"], 7.0)
    err = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    st.stree_gdn_tree_scan_commit(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], d["parent"], o,
                                  d["path"] if commit else None, d["path_len"] if commit else None,
                                  S_new if commit else None, err_out=err,
                                  erase=None if erase is None else to_dev(erase, "f32"))
    torch.cuda.synchronize()
    return o, S_new, err.tolist()


def _oracle(g, erase=None):
    f = g.f64()
    o = oracle_gdn_tree(f["q"], f["k"], f["v"], f["alpha"], f["beta"], f["S0"], g.parent, erase=erase)
    S = oracle_gdn_commit(f["k"], f["v"], f["alpha"], f["beta"], f["S0"], g.parent, g.path, g.path_len,
                          erase=erase)
    return o, S


CASES = [
    # (tree workload, batch, value heads, key heads, dv, dtype)
    ("m2_2p7b", None, 32, 16, 128, "bf16"),
    ("m2_2p7b", None, 4, 4, 64, "f32"),
    ("hyb8b", None, 8, 2, 128, "bf16"),
    ("serve64", 3, 4, 1, 96, "f32"),
    ("serve64", 2, 8, 4, 128, "bf16"),
]


@pytest.mark.parametrize("name,batch,hv,hk,dv,dtype", CASES)
def test_gdn_matches_oracle(st, name, batch, hv, hk, dv, dtype):
    w = wl.make_workload(name, batch=batch, layers=1)
    g = wl.gdn_inputs(w.parent, w.path, w.path_len, heads_v=hv, heads_k=hk, dv=dv, dtype=dtype, seed=41)
    d = _upload(g)
    o, S_new, err = _run(st, g, d)
    assert err == [0, 0, 0, 0]
    o_ref, S_ref = _oracle(g)
    assert_close(f64(o), o_ref, dtype, f"{name} o")
    assert_close(f64(S_new), S_ref, dtype, f"{name} S_new")


@pytest.mark.parametrize("name,batch,hv,hk,dv,dtype,kind", [
    ("serve64", 3, 4, 2, 64, "f32", "random"),
    ("hyb8b", None, 8, 2, 128, "bf16", "random"),
    ("m2_2p7b", None, 4, 4, 128, "f32", "zero"),
    ("serve64", 2, 8, 4, 96, "bf16", "zero"),
])
def test_gdn_decoupled_erase_matches_oracle(st, name, batch, hv, hk, dv, dtype, kind):
    w = wl.make_workload(name, batch=batch, layers=1)
    g = wl.gdn_inputs(w.parent, w.path, w.path_len, heads_v=hv, heads_k=hk, dv=dv, dtype=dtype, seed=43)
    er = (np.random.default_rng(44).uniform(0.0, 1.0, size=g.beta.shape) if kind == "random"
          else np.zeros(g.beta.shape)).astype(np.float32)
    d = _upload(g)
    o, S_new, err = _run(st, g, d, erase=er)
    assert err == [0, 0, 0, 0]
    o_ref, S_ref = _oracle(g, erase=er.astype(np.float64))
    assert_close(f64(o), o_ref, dtype, f"{name} o ({kind} erase)")
    assert_close(f64(S_new), S_ref, dtype, f"{name} S_new ({kind} erase)")


# (dv, dtype): the CUDA-core kernel, and the tensor-core kernel (bf16, d_v = 128).
KERNEL_SHAPES = [(32, "f32"), (128, "bf16")]


@pytest.mark.parametrize("dv,dtype", KERNEL_SHAPES)
def test_gdn_chain_of_64_and_empty_path_in_place(st, dv, dtype):
    parent = np.stack([wl.chain_tree(64), wl.random_tree(np.random.default_rng(3), 64, max_depth=8)])
    path = np.full((2, 64), -1, np.int32)
    path[0, :40] = np.arange(40)
    plen = np.asarray([40, 0], np.int32)
    g = wl.gdn_inputs(parent, path, plen, heads_v=2, heads_k=1, dv=dv, dtype=dtype, seed=5)
    d = _upload(g)
    S0 = d["S0"].clone()
    o, _, err = _run(st, g, d, S_new=d["S0"])                        # commit in place over S0
    assert err == [0, 0, 0, 0]
    o_ref, S_ref = _oracle(g)
    assert_close(f64(o), o_ref, dtype, "o")
    assert_close(f64(d["S0"]), S_ref, dtype, "S_new in place")
    assert torch.equal(d["S0"][1], S0[1])                            # empty path keeps S0 exactly


def test_gdn_without_commit(st):
    w = wl.make_workload("m2_2p7b")
    g = wl.gdn_inputs(w.parent, w.path, w.path_len, heads_v=4, heads_k=2, dtype="bf16", seed=6)
    d = _upload(g)
    o, _, err = _run(st, g, d, commit=False)
    assert err == [0, 0, 0, 0]
    assert_close(f64(o), _oracle(g)[0], "bf16", "o")


@pytest.mark.parametrize("dv,dtype", KERNEL_SHAPES)
def test_gdn_bad_tree_and_bad_path(st, dv, dtype):
    par = [-1, 0, 0, 1, 1, 2]
    parent = np.asarray([par, par, par], np.int32)
    parent[1, 4] = 5                                                 # not topological
    path = np.asarray([[0, 1, 3, -1], [0, 1, -1, -1], [0, 2, 4, -1]], np.int32)   # 4 is not under 2
    plen = np.asarray([3, 2, 3], np.int32)
    g = wl.gdn_inputs(parent, path, plen, heads_v=2, heads_k=1, dv=dv, dtype=dtype, seed=7)
    d = _upload(g)
    o, S_new, err = _run(st, g, d)
    assert err[0] in (3, 4)
    assert torch.all(o[1] == 7.0) and torch.all(S_new[1] == 7.0)    # bad tree: untouched
    assert torch.all(S_new[2] == 7.0)                                # bad path: S_new untouched
    keep = [0]
    f = g.f64()
    o_ref = oracle_gdn_tree(*(f[k][keep] for k in ("q", "k", "v", "alpha", "beta", "S0")), parent[keep])
    assert_close(f64(o[keep]), o_ref, dtype, "o of the valid sequence")
    S_ref = oracle_gdn_commit(*(f[k][keep] for k in ("k", "v", "alpha", "beta", "S0")), parent[keep], path[keep],
                              plen[keep])
    assert_close(f64(S_new[keep]), S_ref, dtype, "S_new of the valid sequence")
    o_ref2 = oracle_gdn_tree(*(f[k][[2]] for k in ("q", "k", "v", "alpha", "beta", "S0")), parent[[2]])
    assert_close(f64(o[[2]]), o_ref2, dtype, "o of the sequence with the bad path")


@pytest.mark.parametrize("T", [1, 2, 16, 17, 32, 33, 47, 63])
def test_gdn_tensor_core_node_counts(st, T):
    # The tensor-core kernel keeps 16, 32 or 64 nodes in registers and solves the
    # second 32-node block after one product: node counts at and across those edges,
    # a random tree and a chain, the random tree's path to its last node, the chain's
    # whole length; a random erase strength for odd counts.
    rng = np.random.default_rng(300 + T)
    parent = np.stack([wl.random_tree(rng, T, max_depth=8), wl.chain_tree(T)]).astype(np.int32)
    path = np.full((2, T), -1, np.int32)
    p0 = wl.root_path_nodes(parent[0], T - 1)
    path[0, :len(p0)] = p0
    path[1, :T] = np.arange(T)
    plen = np.asarray([len(p0), T], np.int32)
    g = wl.gdn_inputs(parent, path, plen, heads_v=4, heads_k=2, dv=128, dtype="bf16", seed=50 + T)
    er = np.random.default_rng(60 + T).uniform(0.0, 1.0, size=g.beta.shape).astype(np.float32) if T % 2 else None
    d = _upload(g)
    o, S_new, err = _run(st, g, d, erase=er)
    assert err == [0, 0, 0, 0]
    o_ref, S_ref = _oracle(g, erase=None if er is None else er.astype(np.float64))
    assert_close(f64(o), o_ref, "bf16", f"T={T} o")
    assert_close(f64(S_new), S_ref, "bf16", f"T={T} S_new")
