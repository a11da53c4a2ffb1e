"""Tree-masked attention (stree_tree_attention) against the fp64 oracle, element
by element at the bf16 tolerance (2e-2 max|ref|): trees of the workloads with
ragged context lengths (including none), grouped heads of several sizes, the
128-node chain, cache positions past the valid length holding NaN (never read),
and an invalid tree; each case both split over CTAs (partials in a workspace,
merged by a second launch) and unsplit (no workspace)."""
import numpy as np
import pytest
import torch

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_tree_attention

from gpu_util import assert_close, f64, i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_packed_tree_b200 import stree
    return stree


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _workspace(st, a, split, short=0):
    if not split:
        return None
    b, T, hq, _ = a["q"].shape
    n = st.stree_tree_attention_workspace_size(T, b, a["k_ctx"].shape[1], hq, a["k_ctx"].shape[2])
    return torch.full((max(n - short, 0),), 0xFF, dtype=torch.uint8, device="cuda")   # NaN-filled partials


def _run(st, a, split=True, short=0):
    q = _bf16(a["q"])
    o = torch.full_like(q, 7.0)
    err = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    st.stree_tree_attention(q, _bf16(a["k_ctx"]), _bf16(a["v_ctx"]), _bf16(a["k_tree"]), _bf16(a["v_tree"]),
                            i32(a["ctx_len"]), i32(a["parent"]), o, a["scale"], err,
                            workspace=_workspace(st, a, split, short))
    torch.cuda.synchronize()
    return o, err.tolist()


def _oracle(a, keep=None):
    sel = slice(None) if keep is None else keep
    f = {k: wl.bf16_to_f64(a[k])[sel] for k in ("q", "k_ctx", "v_ctx", "k_tree", "v_tree")}
    return oracle_tree_attention(f["q"], f["k_ctx"], f["v_ctx"], f["k_tree"], f["v_tree"], a["parent"][sel],
                                 a["scale"], ctx_len=a["ctx_len"][sel])


CASES = [
    # (tree workload, batch, context capacity, context lengths, query heads, key/value heads)
    ("hyb8b", None, 1024, [1024, 1, 0, 130, 1000, 257, 128, 999], 32, 8),
    ("serve64", 3, 640, [640, 300, 129], 32, 8),
    ("m2_2p7b", None, 384, [383], 32, 4),
    ("hyb8b", 2, 256, [256, 100], 8, 8),
    ("wide256_chain", 1, 256, [200], 16, 16),
    ("wide256", 2, 512, [512, 300], 32, 8),
    ("hyb8b", 1, 4096, [4096], 32, 8),                 # 33 key blocks over many splits
    ("serve64", 2, 2048, [2047, 129], 64, 8),          # two query tiles per head group
]


@pytest.mark.parametrize("split", [True, False], ids=["split", "unsplit"])
@pytest.mark.parametrize("name,batch,cap,lens,hq,hkv", CASES)
def test_tree_attention_matches_oracle(st, name, batch, cap, lens, hq, hkv, split):
    w = wl.make_workload(name, batch=batch, layers=1)
    a = wl.attention_inputs(w.parent, cap, lens, heads_q=hq, heads_kv=hkv, seed=61)
    o, err = _run(st, a, split)
    assert err == [0, 0, 0, 0]
    assert_close(f64(o), _oracle(a), "bf16", f"{name} o")


def test_tree_attention_workspace_sizes(st):
    # A long context over few tiles splits; many tiles over a short context do not.
    assert st.stree_tree_attention_workspace_size(26, 1, 4096, 32, 8) > 0
    assert st.stree_tree_attention_workspace_size(64, 64, 1024, 32, 8) == 0
    assert st.stree_tree_attention_workspace_size(26, 0, 4096, 32, 8) == 0
    with pytest.raises(st.StreeError):
        st.stree_tree_attention_workspace_size(26, 1, 4096, 32, 8, head_dim=64)


def test_tree_attention_workspace_too_small_runs_unsplit(st):
    w = wl.make_workload("hyb8b", batch=2, layers=1)
    a = wl.attention_inputs(w.parent, 2048, [2048, 700], heads_q=32, heads_kv=8, seed=64)
    o_split, err = _run(st, a, split=True)
    assert err == [0, 0, 0, 0]
    o_short, err = _run(st, a, split=True, short=16)
    assert err == [0, 0, 0, 0]
    o_none, err = _run(st, a, split=False)
    assert err == [0, 0, 0, 0]
    assert torch.equal(o_short, o_none)                # the short workspace is not used
    ref = _oracle(a)
    assert_close(f64(o_split), ref, "bf16", "split o")
    assert_close(f64(o_none), ref, "bf16", "unsplit o")


def test_tree_attention_without_context(st):
    w = wl.make_workload("m2_2p7b")
    a = wl.attention_inputs(w.parent, 0, [0], heads_q=8, heads_kv=2, seed=62)
    q = _bf16(a["q"])
    o = torch.full_like(q, 7.0)
    err = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    empty = torch.empty((1, 0, 2, 128), dtype=torch.bfloat16, device="cuda")
    st.stree_tree_attention(q, empty, empty, _bf16(a["k_tree"]), _bf16(a["v_tree"]), i32(a["ctx_len"]),
                            i32(a["parent"]), o, a["scale"], err, workspace=_workspace(st, a, True))
    torch.cuda.synchronize()
    assert err.tolist() == [0, 0, 0, 0]
    assert_close(f64(o), _oracle(a), "bf16", "o")


@pytest.mark.parametrize("split", [True, False], ids=["split", "unsplit"])
def test_tree_attention_invalid_tree(st, split):
    par = [-1, 0, 0, 1, 1, 2]
    parent = np.asarray([par, par], np.int32)
    parent[1, 3] = 4
    a = wl.attention_inputs(parent, 1024, [1024, 50], heads_q=4, heads_kv=1, seed=63)
    o, err = _run(st, a, split)
    assert err[0] == 3 and err[1] == 1
    assert torch.all(o[1] == 7.0)
    assert_close(f64(o[:1]), _oracle(a, keep=[0]), "bf16", "o of the valid sequence")
