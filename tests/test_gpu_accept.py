"""Greedy tree verification (stree_accept_greedy) against the oracle, bit-exact:
predictions, accepted paths, lengths and bonus tokens are integers, and both sides
take the argmax in the logits' own precision.  The accepted path then drives the
fused commit, which must equal the oracle's commit of that path."""
import json
import os

import numpy as np
import pytest
import torch

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_accept_greedy, oracle_commit

from gpu_util import assert_close, f64, i32, upload_layer, upload_tree

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_packed_tree_b200 import stree
    return stree


def _logits_tensor(logits, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(logits).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(logits, dtype=np.float32)).cuda()


def _run(st, lg, tokens, parent, maxlen):
    b, T = tokens.shape
    pred = torch.full((b, T), -7, dtype=torch.int32, device="cuda")
    path = torch.full((b, maxlen), -7, dtype=torch.int32, device="cuda")
    plen = torch.full((b,), -7, dtype=torch.int32, device="cuda")
    bonus = torch.full((b,), -7, dtype=torch.int32, device="cuda")
    err = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    st.stree_accept_greedy(lg, i32(tokens), i32(parent), pred, path, plen, bonus, err_out=err)
    torch.cuda.synchronize()
    return pred.cpu().numpy(), path.cpu().numpy(), plen.cpu().numpy(), bonus.cpu().numpy(), err.tolist()


def test_accept_golden_cases(st):
    with open(os.path.join(os.path.dirname(__file__), "golden", "accept_greedy.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        lg = _logits_tensor(np.asarray(c["logits"], np.float32)[None], "f32")
        pred, path, plen, bonus, err = _run(st, lg, np.asarray([c["tokens"]], np.int32),
                                            np.asarray([c["parent"]], np.int32), c["maxlen"])
        n = c["path_len"]
        assert err == [0, 0, 0, 0], c["name"]
        assert int(plen[0]) == n and path[0, :n].tolist() == c["path"] and (path[0, n:] == -1).all(), c["name"]
        assert int(bonus[0]) == c["bonus"], c["name"]


@pytest.mark.parametrize("name,batch,vocab,dtype", [("m2_2p7b", None, 50280, "bf16"), ("hyb8b", None, 1001, "bf16"),
                                                    ("serve64", 8, 4096, "f32"), ("wide256", 4, 777, "f32"),
                                                    ("wide256_chain", 1, 96, "bf16")])
def test_accept_matches_oracle_on_planted_trees(st, name, batch, vocab, dtype):
    w = wl.make_workload(name, batch=batch, layers=1)
    logits, tokens, planted = wl.acceptance_inputs(w.parent, vocab, seed=5, dtype=dtype)
    lg_ref = wl.stored_to_f64(logits, dtype)
    maxlen = w.n_nodes
    want = oracle_accept_greedy(lg_ref, tokens, w.parent, maxlen)
    got = _run(st, _logits_tensor(logits, dtype), tokens, w.parent, maxlen)
    assert got[4] == [0, 0, 0, 0]
    for g, r, what in zip(got[:4], want, ("pred", "path", "path_len", "bonus")):
        assert np.array_equal(g, r), what
    for s, nodes in enumerate(planted):                      # the planted path is accepted
        assert got[1][s, :got[2][s]].tolist() == nodes


def test_accept_invalid_tree(st):
    parent = np.array([[-1, 0, 0, 1], [-1, 0, 3, 1]], np.int32)        # node 2's parent comes later
    tokens = np.zeros((2, 4), np.int32)
    lg = _logits_tensor(np.zeros((2, 4, 16), np.float32), "f32")
    pred, path, plen, bonus, err = _run(st, lg, tokens, parent, 4)
    assert err[0] == 3 and err[1] == 1
    assert plen[1] == 0 and bonus[1] == -1 and (path[1] == -1).all()
    assert plen[0] >= 1


def test_accepted_path_drives_the_commit(st):
    """Verify -> accept -> commit: the path chosen by the acceptance kernel goes
    straight into the fused scan + commit."""
    w = wl.make_workload("serve64", batch=4, layers=1)
    logits, tokens, _ = wl.acceptance_inputs(w.parent, 512, seed=9, dtype="bf16")
    maxlen = w.n_nodes
    b, T = tokens.shape
    pred = torch.empty((b, T), dtype=torch.int32, device="cuda")
    path = torch.empty((b, maxlen), dtype=torch.int32, device="cuda")
    plen = torch.empty((b,), dtype=torch.int32, device="cuda")
    bonus = torch.empty((b,), dtype=torch.int32, device="cuda")
    d, tr = upload_layer(w), upload_tree(w)
    st.stree_accept_greedy(_logits_tensor(logits, "bf16"), i32(tokens), tr["parent"], pred, path, plen, bonus)
    ctx = st.stree_ctx_create()
    y = torch.empty_like(d["x"])
    h_new = torch.empty_like(d["h0"])
    st.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], tr["parent"], path, plen,
                              y, h_new)
    st.stree_sync_check(ctx)
    f = w.f64(0)
    h_ref = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, path.cpu().numpy(),
                          plen.cpu().numpy(), nthreads=8)[0]
    assert_close(f64(h_new), h_ref, w.dtype, "commit of the accepted path")
    st.stree_ctx_destroy(ctx)
