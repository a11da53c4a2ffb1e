"""Pins of the fp64 CPU oracle against facts that do not come from the oracle itself.

The pages print no worked example, so the oracle is pinned by: two hand-worked
cases (tests/golden/), closed forms (geometric series on a constant chain, dt = 0,
C = 0), structural invariants of a tree scan (chain = sequential scan, each leaf's
path = the unrolled path, identical siblings, relabelling), a second formulation
(the packed closed form, oracle/packed.py) and brute force on the tree masks.
A mutation test plants plausible mistakes in a copy of the C oracle and checks
that the pins catch each one.
"""
import ctypes
import json
import os
import subprocess

import numpy as np
import pytest

from hybrid_packed_tree_b200 import workloads as wl
from oracle import oracle_build_tree, oracle_commit, oracle_tree_scan
from oracle.packed import ancestor_matrix, packed_commit, packed_scan

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _scalar_case():
    g = _load("scalar_tree.json")
    T = len(g["parent"])
    x = np.asarray(g["x"]).reshape(1, T, 1, 1)
    dt = np.asarray(g["dt"]).reshape(1, T, 1)
    A = np.asarray([g["A"]])
    B = np.asarray(g["B"]).reshape(1, T, 1, 1)
    C = np.asarray(g["C"]).reshape(1, T, 1, 1)
    D = np.asarray([g["D"]])
    h0 = np.asarray([g["h0"]]).reshape(1, 1, 1, 1)
    parent = np.asarray([g["parent"]], np.int32)
    return g, (x, dt, A, B, C, D, h0, parent)


# ----------------------------------------------------------------------------- golden


def test_golden_scalar_tree_outputs():
    g, (x, dt, A, B, C, D, h0, parent) = _scalar_case()
    y = oracle_tree_scan(x, dt, A, B, C, D, h0, parent)
    np.testing.assert_allclose(y.reshape(-1), g["y"], rtol=0, atol=1e-12)


def test_golden_scalar_tree_masks():
    g, (*_, parent) = _scalar_case()
    anc, depth, ok = oracle_build_tree(parent)
    assert ok.tolist() == [1]
    assert anc[0, :, 0].tolist() == g["anc_bits"]
    assert depth[0].tolist() == g["depth"]


def test_golden_scalar_tree_commits():
    g, (x, dt, A, B, C, D, h0, parent) = _scalar_case()
    for c in g["commits"]:
        path = np.full((1, 4), -1, np.int32)
        path[0, :len(c["path"])] = c["path"]
        h_new, ok, leaf = oracle_commit(x, dt, A, B, h0, parent, path, [len(c["path"])])
        assert ok[0] == 1
        assert leaf[0] == (c["path"][-1] if c["path"] else -1)
        assert abs(h_new.reshape(-1)[0] - c["h_new"]) < 1e-12


def test_golden_matrix_chain():
    g = _load("matrix_chain.json")
    x = np.asarray(g["x"]).reshape(1, 2, 1, 2)
    dt = np.asarray(g["dt"]).reshape(1, 2, 1)
    B = np.asarray(g["B"]).reshape(1, 2, 1, 3)
    C = np.asarray(g["C"]).reshape(1, 2, 1, 3)
    h0 = np.asarray(g["h0"]).reshape(1, 1, 2, 3)
    A, D = np.asarray([g["A"]]), np.asarray([g["D"]])
    parent = np.asarray([g["parent"]], np.int32)
    y = oracle_tree_scan(x, dt, A, B, C, D, h0, parent)
    np.testing.assert_allclose(y.reshape(2, 2), g["y"], rtol=0, atol=1e-12)
    h_new, ok, _ = oracle_commit(x, dt, A, B, h0, parent, [[0, 1]], [2])
    np.testing.assert_allclose(h_new.reshape(2, 3), g["h_new_full_path"], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- closed forms


def test_constant_chain_geometric_closed_form():
    """Constant dt, x, B on a chain: s_k = a^(k+1) h0 + dt (1-a^(k+1))/(1-a) outer(x,B)."""
    rng = np.random.default_rng(5)
    T, P, N = 9, 3, 5
    a_log = -0.37
    dtv = 0.8
    A = np.asarray([a_log / dtv])
    x1, B1 = rng.normal(size=P), rng.normal(size=N)
    C = rng.normal(size=(1, T, 1, N))
    D = np.asarray([0.3])
    h0 = rng.normal(size=(1, 1, P, N))
    x = np.broadcast_to(x1, (1, T, 1, P)).copy()
    B = np.broadcast_to(B1, (1, T, 1, N)).copy()
    dt = np.full((1, T, 1), dtv)
    parent = wl.chain_tree(T)[None]
    y = oracle_tree_scan(x, dt, A, B, C, D, h0, parent)
    a = np.exp(a_log)
    for k in range(T):
        s = a ** (k + 1) * h0[0, 0] + dtv * (1 - a ** (k + 1)) / (1 - a) * np.outer(x1, B1)
        np.testing.assert_allclose(y[0, k, 0], s @ C[0, k, 0] + D[0] * x1, rtol=1e-12, atol=1e-12)
    h_new, _, _ = oracle_commit(x, dt, A, B, h0, parent, [list(range(T))], [T])
    s = a ** T * h0[0, 0] + dtv * (1 - a ** T) / (1 - a) * np.outer(x1, B1)
    np.testing.assert_allclose(h_new[0, 0], s, rtol=1e-12, atol=1e-12)


def _rand_case(seed=0, parent=None, H=3, P=4, N=6, G=1, dtype="f32"):
    if parent is None:
        parent = [-1, 0, 0, 1, 1, 2, 3, 3, 6, 4]
    w = wl.custom_workload(parent, nheads=H, headdim=P, dstate=N, ngroups=G, dtype=dtype, seed=seed)
    f = w.f64(0)
    return w, f


def test_dt_zero_gives_root_readout():
    """dt = 0: no decay and no input, every node reads the cached state: y = h0 C_i + D x_i."""
    w, f = _rand_case(1)
    dt = np.zeros_like(f["dt"])
    y = oracle_tree_scan(f["x"], dt, f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    ref = np.einsum("bhpn,btn->bthp", f["h0"], f["C"][:, :, 0, :]) + f["D"][None, None, :, None] * f["x"]
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


def test_c_zero_gives_skip_only():
    w, f = _rand_case(2)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], np.zeros_like(f["C"]), f["D"], f["h0"], w.parent)
    np.testing.assert_allclose(y, f["D"][None, None, :, None] * f["x"], rtol=0, atol=0)


# ----------------------------------------------------------------------------- invariants


def _seq_scan(x, dt, A, B, C, D, h0):
    """Textbook sequential selective scan over a time axis (one sequence, one head)."""
    s = h0.copy()
    ys = []
    for t in range(x.shape[0]):
        s = np.exp(dt[t] * A) * s + dt[t] * np.outer(x[t], B[t])
        ys.append(s @ C[t] + D * x[t])
    return np.asarray(ys), s


def test_chain_tree_equals_sequential_scan():
    T = 12
    w, f = _rand_case(3, parent=wl.chain_tree(T), H=2, P=3, N=4)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    for h in range(2):
        ys, s_end = _seq_scan(f["x"][0, :, h], f["dt"][0, :, h], f["A"][h], f["B"][0, :, 0],
                              f["C"][0, :, 0], f["D"][h], f["h0"][0, h])
        np.testing.assert_allclose(y[0, :, h], ys, rtol=1e-12, atol=1e-12)
    h_new, _, _ = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent,
                                [list(range(T))], [T])
    np.testing.assert_allclose(h_new[0, 1], s_end, rtol=1e-12, atol=1e-12)


def test_each_leaf_path_equals_unrolled_sequence():
    rng = np.random.default_rng(4)
    parent = wl.random_tree(rng, 20, max_depth=6)
    w, f = _rand_case(4, parent=parent, H=2, P=3, N=5)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    for leaf in wl.leaves(parent):
        nodes = wl.root_path_nodes(parent, int(leaf))
        sub = {k: (v[:, nodes] if k in ("x", "dt", "B", "C") else v) for k, v in f.items()}
        yc = oracle_tree_scan(sub["x"], sub["dt"], sub["A"], sub["B"], sub["C"], sub["D"], sub["h0"],
                              wl.chain_tree(len(nodes))[None])
        np.testing.assert_allclose(y[:, nodes], yc, rtol=1e-13, atol=1e-13)


def test_identical_siblings_identical_outputs():
    parent = np.asarray([-1, 0, 0, 1, 2], np.int32)      # 1 and 2 are siblings, 3 and 4 their kids
    w, f = _rand_case(5, parent=parent, H=2, P=3, N=4)
    for k in ("x", "dt", "B", "C"):
        f[k][:, 2] = f[k][:, 1]
        f[k][:, 4] = f[k][:, 3]
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], parent[None])
    assert np.array_equal(y[:, 1], y[:, 2]) and np.array_equal(y[:, 3], y[:, 4])
    assert not np.allclose(y[:, 1], y[:, 0])


def test_topological_relabel_permutes_outputs():
    rng = np.random.default_rng(6)
    parent = wl.random_tree(rng, 16, max_depth=5)
    w, f = _rand_case(6, parent=parent, H=2, P=3, N=4)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    # Another topological order: depth-first, children in decreasing label order.
    children = [[] for _ in range(16)]
    for i, p in enumerate(parent):
        if p >= 0:
            children[p].append(i)
    order, stack = [], [0]
    while stack:
        n = stack.pop()
        order.append(n)
        stack.extend(sorted(children[n]))
    new_of = np.empty(16, int)
    new_of[order] = np.arange(16)
    par2 = np.asarray([-1 if parent[o] < 0 else new_of[parent[o]] for o in order], np.int32)
    g = {k: (v[:, order] if k in ("x", "dt", "B", "C") else v) for k, v in f.items()}
    y2 = oracle_tree_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["h0"], par2[None])
    np.testing.assert_allclose(y2, y[:, order], rtol=1e-13, atol=1e-13)


def test_group_mapping_matches_per_group_calls():
    """Heads h use group h // (H/G): a G=2 call equals two G=1 calls on the head halves."""
    w, f = _rand_case(7, H=4, P=3, N=4, G=2)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    for g in range(2):
        hs = slice(2 * g, 2 * g + 2)
        yg = oracle_tree_scan(f["x"][:, :, hs], f["dt"][:, :, hs], f["A"][hs], f["B"][:, :, g:g + 1],
                              f["C"][:, :, g:g + 1], f["D"][hs], f["h0"][:, hs], w.parent)
        np.testing.assert_allclose(y[:, :, hs], yg, rtol=0, atol=0)


@pytest.mark.parametrize("seed,T,H,P,N,G", [(8, 10, 3, 4, 6, 1), (9, 26, 4, 5, 7, 2), (10, 40, 2, 3, 3, 1)])
def test_packed_closed_form_equals_walk(seed, T, H, P, N, G):
    rng = np.random.default_rng(seed)
    parents = np.stack([wl.random_tree(rng, T, max_depth=7), wl.random_tree(rng, T, max_depth=3)])
    w, f = _rand_case(seed, parent=parents, H=H, P=P, N=N, G=G)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    yp = packed_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    np.testing.assert_allclose(y, yp, rtol=1e-12, atol=1e-12)
    h_new, ok, _ = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, w.path, w.path_len)
    hp = packed_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, w.path, w.path_len)
    np.testing.assert_allclose(h_new, hp, rtol=1e-12, atol=1e-12)


def test_commit_state_reads_out_the_leaf_output():
    """The replayed state at the path's end reproduces the scan's output there: y_leaf = h_new C_leaf + D x_leaf."""
    rng = np.random.default_rng(11)
    parent = wl.random_tree(rng, 18, max_depth=6)
    w, f = _rand_case(11, parent=parent, H=2, P=3, N=4)
    y = oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent)
    for node in range(18):
        nodes = wl.root_path_nodes(parent, node)
        h_new, ok, leaf = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent,
                                        [nodes + [-1] * (18 - len(nodes))], [len(nodes)])
        assert leaf[0] == node
        ro = np.einsum("hpn,n->hp", h_new[0], f["C"][0, node, 0]) + f["D"][:, None] * f["x"][0, node]
        np.testing.assert_allclose(ro, y[0, node], rtol=1e-12, atol=1e-12)


def test_commit_empty_path_keeps_state_and_allows_alias():
    w, f = _rand_case(12)
    h_new, ok, leaf = oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, [[-1] * 10], [0])
    assert ok[0] == 1 and leaf[0] == -1
    assert np.array_equal(h_new, f["h0"])


# ----------------------------------------------------------------------------- masks / validation


def test_masks_equal_recursive_definition():
    """anc(i) = anc(parent(i)) + {i}, depth(i) = depth(parent(i)) + 1, built independently."""
    rng = np.random.default_rng(13)
    for T in (1, 2, 31, 32, 33, 64, 100, 128, 200, 256):
        parent = wl.random_tree(rng, T, max_depth=T) if T > 1 else np.asarray([-1], np.int32)
        anc, depth, ok = oracle_build_tree(parent[None])
        assert ok[0] == 1
        W = (T + 31) // 32
        ref = np.zeros((T, W), np.uint32)
        dref = np.zeros(T, np.int32)
        for i in range(T):
            if parent[i] >= 0:
                ref[i] = ref[parent[i]]
                dref[i] = dref[parent[i]] + 1
            ref[i, i // 32] |= np.uint32(1 << (i % 32))
        assert np.array_equal(anc[0], ref) and np.array_equal(depth[0], dref)
        assert np.array_equal(ancestor_matrix(parent), np.unpackbits(
            ref.view(np.uint8), bitorder="little").reshape(T, W * 32)[:, :T].astype(bool))


@pytest.mark.parametrize("parent", [
    [0, 0, 1],          # root is not marked -1
    [-1, 2, 0],         # parent after the child
    [-1, 1],            # self loop
    [-1, 0, -1],        # two roots
    [-1, 0, 7],         # out of range
    [-1, -5, 0],        # negative, not -1
])
def test_invalid_trees_rejected(parent):
    anc, depth, ok = oracle_build_tree(np.asarray([parent], np.int32))
    assert ok[0] == 0
    w, f = _rand_case(14, parent=[-1, 0, 1], H=1, P=2, N=2)
    with pytest.raises(ValueError):
        oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], np.asarray([parent], np.int32))


@pytest.mark.parametrize("path,plen", [
    ([1, 3, -1, -1], 2),   # does not start at the root
    ([0, 2, 3, -1], 3),    # 3's parent is 1, not 2
    ([0, 1, 3, 3], 5),     # longer than maxlen
    ([0, 1, 3, 9], 4),     # out of range
    ([0, 0, -1, -1], 2),   # repeats the root
])
def test_invalid_paths_rejected(path, plen):
    g, (x, dt, A, B, C, D, h0, parent) = _scalar_case()
    h_new, ok, leaf = oracle_commit(x, dt, A, B, h0, parent, [path], [plen], allow_invalid=True)
    assert ok[0] == 0 and leaf[0] == -1


def test_workload_trees_match_their_descriptions():
    w = wl.make_workload("hyb8b")
    for row in w.parent:
        d = wl.node_depths(row)
        assert d.max() == 5
        assert np.bincount(row[1:], minlength=26).max() <= 4
    w = wl.make_workload("wide256", batch=16)
    for row in w.parent:
        d = wl.node_depths(row)
        assert d.max() <= 10 and np.bincount(d).max() <= 16
    w = wl.make_workload("serve64", batch=16, layers=1)
    for b, row in enumerate(w.parent):
        assert wl.node_depths(row).max() <= 8
        assert 1 <= w.path_len[b] <= 8
    for name in wl.SPECS:
        w = wl.make_workload(name, batch=min(wl.SPECS[name][1], 4), layers=1)
        anc, depth, ok = oracle_build_tree(w.parent)
        assert ok.all()
        if name == "m2_2p7b":
            assert w.n_nodes == 15


# ----------------------------------------------------------------------------- mutation check


_MUTANTS = {
    "decay sign flipped": ("double decay = exp(dt * A);", "double decay = exp(-dt * A);"),
    "skip term dropped": ("yi[p] = acc + D[h] * xi[p];", "yi[p] = acc;"),
    "input not scaled by dt": ("+ dt * x[p] * B[n];", "+ x[p] * B[n];"),
    "readout uses parent's C": ("const double *Ci = Cm + (((size_t)b * T + i) * G + g) * N;",
                                "const double *Ci = Cm + (((size_t)b * T + (i ? par[i] : 0)) * G + g) * N;"),
    "path walk skips the node itself": ("for (int k = node; k != -1; k = par[k]) path[len++] = k;",
                                        "for (int k = par[node]; k != -1; k = par[k]) path[len++] = k;"),
    "outer product transposed": ("+ dt * x[p] * B[n];", "+ dt * x[n % P] * B[p % N];"),
}


@pytest.mark.parametrize("mutant", sorted(_MUTANTS))
def test_pins_catch_planted_mistakes(mutant, tmp_path):
    src = open(os.path.join(os.path.dirname(__file__), "..", "oracle", "stree_oracle.c")).read()
    old, new = _MUTANTS[mutant]
    assert old in src
    cfile = tmp_path / "mut.c"
    cfile.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(cfile), "-lm"], check=True)
    lib = ctypes.CDLL(str(so))
    dp, ip = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int32)
    lib.oracle_tree_scan.argtypes = [dp] * 7 + [ip] + [ctypes.c_int] * 6 + [dp, ctypes.c_int]

    def run(x, dt, A, B, C, D, h0, parent):
        arrs = [np.ascontiguousarray(v, np.float64) for v in (x, dt, A, B, C, D, h0)]
        par = np.ascontiguousarray(parent, np.int32)
        b, T, H, P = arrs[0].shape
        G, N = arrs[3].shape[2], arrs[3].shape[3]
        y = np.zeros((b, T, H, P))
        lib.oracle_tree_scan(*[a.ctypes.data_as(dp) for a in arrs], par.ctypes.data_as(ip),
                             T, b, H, P, N, G, y.ctypes.data_as(dp), 1)
        return y

    caught = []
    g, case = _scalar_case()
    caught.append(not np.allclose(run(*case).reshape(-1), g["y"], atol=1e-12))
    m = _load("matrix_chain.json")
    mc = (np.asarray(m["x"]).reshape(1, 2, 1, 2), np.asarray(m["dt"]).reshape(1, 2, 1),
          np.asarray([m["A"]]), np.asarray(m["B"]).reshape(1, 2, 1, 3),
          np.asarray(m["C"]).reshape(1, 2, 1, 3), np.asarray([m["D"]]),
          np.asarray(m["h0"]).reshape(1, 1, 2, 3), np.asarray([m["parent"]], np.int32))
    caught.append(not np.allclose(run(*mc).reshape(2, 2), m["y"], atol=1e-12))
    assert any(caught), f"no pin caught the planted mistake: {mutant}"


def test_unroll_paths_lists_every_root_to_leaf_chain():
    """Host-side unrolling used by the unrolled baseline: one path per leaf, each a
    chain from the root (parent[path[k]] == path[k-1]) ending at that leaf."""
    rng = np.random.default_rng(11)
    parents = np.stack([wl.random_tree(rng, 40, max_depth=6) for _ in range(3)])
    paths, plen = wl.unroll_paths(parents)
    for b in range(3):
        lv = set(int(l) for l in wl.leaves(parents[b]))
        got = set()
        for k in range(paths.shape[1]):
            n = int(plen[b, k])
            if n == 0:
                continue
            nodes = paths[b, k, :n]
            assert nodes[0] == 0 and parents[b][nodes[0]] == -1
            assert all(parents[b][nodes[q]] == nodes[q - 1] for q in range(1, n))
            got.add(int(nodes[-1]))
        assert got == lv and sum(plen[b] > 0) == len(lv)


# ------------------------------------------------------------------ greedy acceptance


def test_accept_greedy_golden_cases():
    """Hand-worked cases (tests/golden/accept_greedy.json): ties, equal sibling
    tokens, no match, a full chain and the maxlen cut."""
    from oracle import oracle_accept_greedy
    with open(os.path.join(os.path.dirname(__file__), "golden", "accept_greedy.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        lg = np.asarray(c["logits"], np.float64)[None]
        pred, path, plen, bonus = oracle_accept_greedy(lg, np.asarray(c["tokens"])[None],
                                                       np.asarray(c["parent"])[None], c["maxlen"])
        n = c["path_len"]
        assert int(plen[0]) == n, c["name"]
        assert path[0, :n].tolist() == c["path"], c["name"]
        assert (path[0, n:] == -1).all(), c["name"]
        assert int(bonus[0]) == c["bonus"], c["name"]


def test_accept_greedy_follows_a_planted_path():
    """Random trees with distinct sibling tokens and logits whose maximum after
    every node of a chosen root-to-leaf path is the next node's token: exactly
    that path is accepted, and the bonus is the token planted after the leaf."""
    from oracle import oracle_accept_greedy
    rng = np.random.default_rng(21)
    b, T, V = 5, 30, 97
    parents = np.stack([wl.random_tree(rng, T, max_depth=6) for _ in range(b)])
    tokens = np.zeros((b, T), np.int64)
    logits = rng.normal(size=(b, T, V))
    want_paths, want_bonus = [], []
    for s in range(b):
        for u in range(T):                        # distinct tokens among each node's children
            kids = [c for c in range(T) if parents[s, c] == u]
            tokens[s, kids] = rng.choice(V, size=len(kids), replace=False)
        leaf = int(rng.choice(wl.leaves(parents[s])))
        nodes = wl.root_path_nodes(parents[s], leaf)
        for u, v in zip(nodes[:-1], nodes[1:]):
            logits[s, u, tokens[s, v]] = logits[s, u].max() + 1.0
        bonus_tok = int(rng.integers(V))
        logits[s, leaf, bonus_tok] = logits[s, leaf].max() + 1.0
        want_paths.append(nodes)
        want_bonus.append(bonus_tok)
    pred, path, plen, bonus = oracle_accept_greedy(logits, tokens, parents, T)
    for s in range(b):
        assert path[s, :plen[s]].tolist() == want_paths[s]
        assert int(bonus[s]) == want_bonus[s]


# ------------------------------------------------------------------ sampling acceptance


def test_accept_sampling_golden_cases():
    """Hand-worked cases (tests/golden/accept_sampling.json): acceptance with
    probability p/q, the residual after a rejection, a second sibling accepted
    against the residual, bonus tokens by inverse CDF."""
    from oracle import oracle_accept_sampling
    with open(os.path.join(os.path.dirname(__file__), "golden", "accept_sampling.json")) as f:
        doc = json.load(f)
    for c in doc["cases"]:
        path, plen, bonus = oracle_accept_sampling(
            np.asarray(c["target_logits"])[None], np.asarray(c["draft_logits"])[None], np.asarray(c["tokens"])[None],
            np.asarray(c["parent"])[None], doc["temperature"], np.asarray(c["u_accept"])[None],
            np.asarray([c["u_bonus"]]), c["maxlen"])
        n = c["path_len"]
        assert int(plen[0]) == n and path[0, :n].tolist() == c["path"], c["name"]
        assert int(bonus[0]) == c["bonus"], c["name"]


def test_accept_sampling_at_vanishing_temperature_is_greedy():
    """As the temperature goes to 0 both distributions become one-hot on their
    argmax: a child is accepted exactly when its token is the target's argmax,
    and the bonus is that argmax -- the greedy rule."""
    from oracle import oracle_accept_greedy, oracle_accept_sampling
    w = wl.make_workload("serve64", batch=6, layers=1)
    logits, tokens, _ = wl.acceptance_inputs(w.parent, 64, seed=13, dtype="f32")
    rng = np.random.default_rng(14)
    draft = rng.normal(size=logits.shape)
    ua = rng.uniform(size=tokens.shape)
    ub = rng.uniform(size=w.batch) * 0.999
    g_pred, g_path, g_len, g_bonus = oracle_accept_greedy(logits, tokens, w.parent, w.n_nodes)
    s_path, s_len, s_bonus = oracle_accept_sampling(logits, draft, tokens, w.parent, 1e-4, ua, ub, w.n_nodes)
    assert np.array_equal(g_path, s_path) and np.array_equal(g_len, s_len) and np.array_equal(g_bonus, s_bonus)


def test_accept_sampling_first_token_follows_the_target_distribution():
    """Losslessness: with the root's children drawn independently from the draft
    distribution q, the first token emitted (the accepted child's token, else the
    bonus) is distributed as the target's p, whatever q is (Monte Carlo, 5 sigma)."""
    from oracle import oracle_accept_sampling
    rng = np.random.default_rng(15)
    V, k, n = 5, 3, 30000
    p = np.array([0.35, 0.05, 0.25, 0.15, 0.20])
    q = np.array([0.10, 0.40, 0.10, 0.30, 0.10])
    tl = np.zeros((n, k + 1, V))
    tl[:, 0] = np.log(p)
    dl = np.zeros((n, k + 1, V))
    dl[:, 0] = np.log(q)
    tokens = np.zeros((n, k + 1), np.int64)
    tokens[:, 1:] = rng.choice(V, size=(n, k), p=q)
    parent = np.tile(np.array([-1] + [0] * k), (n, 1))
    path, plen, bonus = oracle_accept_sampling(tl, dl, tokens, parent, 1.0, rng.uniform(size=(n, k + 1)),
                                               rng.uniform(size=n), k + 1)
    first = np.where(plen >= 2, tokens[np.arange(n), np.maximum(path[:, 1], 0)], bonus)
    freq = np.bincount(first, minlength=V) / n
    assert np.all(np.abs(freq - p) < 5 * np.sqrt(p * (1 - p) / n)), (freq, p)


def test_accept_pins_catch_planted_mistakes():
    """Copies of the verification oracles with one planted mistake each must fail
    the pins above: last-index ties, the largest matching child, no maxlen cut, no
    residual after a rejection, a bonus from the undisturbed target distribution."""
    import oracle.accept as acc
    src = open(acc.__file__).read()
    mutants = {
        "ties to the larger id": ("pred = np.argmax(logits, axis=-1).astype(np.int64)",
                                  "pred = (logits.shape[-1] - 1 - np.argmax(logits[..., ::-1], axis=-1)).astype(np.int64)"),
        "largest matching child": ("for c in range(T):                       # children in increasing index order",
                                   "for c in reversed(range(T)):             # children in decreasing index order"),
        "no maxlen cut": ("        while len(nodes) < maxlen:\n", "        while True:\n"),
        "no residual": ("                    r = np.maximum(p - q, 0.0)\n                    if r.sum() > 0.0:\n                        p = r / r.sum()\n",
                        "                    pass\n"),
        "bonus from the target": ("        cdf = np.cumsum(p)\n", "        cdf = np.cumsum(_softmax(tl[s, cur] / temperature))\n"),
    }
    checks = [test_accept_greedy_golden_cases, test_accept_greedy_follows_a_planted_path,
              test_accept_sampling_golden_cases, test_accept_sampling_at_vanishing_temperature_is_greedy,
              test_accept_sampling_first_token_follows_the_target_distribution]
    import oracle
    for name, (old, new) in mutants.items():
        assert src.count(old) == 1, name
        ns = {"__name__": "mutant"}
        exec(compile(src.replace(old, new), "mutant", "exec"), ns)
        saved = (oracle.oracle_accept_greedy, oracle.oracle_accept_sampling)
        oracle.oracle_accept_greedy, oracle.oracle_accept_sampling = ns["oracle_accept_greedy"], ns["oracle_accept_sampling"]
        try:
            caught = False
            for chk in checks:
                try:
                    chk()
                except (AssertionError, IndexError, ValueError):
                    caught = True
                    break
            assert caught, f"mutant '{name}' passed every pin"
        finally:
            oracle.oracle_accept_greedy, oracle.oracle_accept_sampling = saved
