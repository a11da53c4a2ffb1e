"""Pins of the gated-delta-rule tree oracle (oracle/gdn.py) against facts that do
not come from the oracle itself: a hand-worked case with a non-square state, the
pure-decay closed form at beta = 0, the delta rule's write property (with alpha
= beta = 1 and a unit key, the new state maps that key exactly to its value),
exact recall along a path of orthonormal keys, each leaf against its path
decoded alone, identical siblings, the commit against the leaf's state, the
packed triangular-solve formulation, and a mutation check.  With the erase
strength given apart from the write strength: a hand-worked decoupled case, and
zero erase against the closed form of gated linear attention (every node's output
a decayed sum over its root path, written out directly).
"""
import json
import os

import numpy as np

from hybrid_packed_tree_b200 import workloads as wl
from oracle.gdn import oracle_gdn_commit, oracle_gdn_tree, packed_gdn

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLD, "gdn_tree.json")) as f:
        g = json.load(f)
    T = len(g["parent"])
    q = np.asarray(g["q"]).reshape(1, T, 1, 2)
    k = np.asarray(g["k"]).reshape(1, T, 1, 2)
    v = np.asarray(g["v"]).reshape(1, T, 1, 1)
    a = np.asarray(g["alpha"]).reshape(1, T, 1)
    be = np.asarray(g["beta"]).reshape(1, T, 1)
    S0 = np.asarray(g["S0"]).reshape(1, 1, 1, 2)
    return g, (q, k, v, a, be, S0, np.asarray([g["parent"]]))


def _rand(seed, parent, Hv=2, Hk=1, dk=6, dv=5, unit=True):
    rng = np.random.default_rng(seed)
    parent = np.asarray(parent)
    b, T = parent.shape
    q = rng.normal(size=(b, T, Hk, dk))
    k = rng.normal(size=(b, T, Hk, dk))
    if unit:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(b, T, Hv, dv))
    a = np.exp(-rng.uniform(0.01, 0.5, size=(b, T, Hv)))
    be = rng.uniform(0.05, 0.95, size=(b, T, Hv))
    S0 = rng.normal(size=(b, Hv, dv, dk))
    return q, k, v, a, be, S0


def test_golden_hand_worked_tree():
    g, (q, k, v, a, be, S0, parent) = _golden()
    o = oracle_gdn_tree(q, k, v, a, be, S0, parent)
    np.testing.assert_allclose(o.reshape(-1), g["o"], rtol=0, atol=1e-12)
    for i in range(3):
        path = np.asarray([[0] if i == 0 else [0, i]])
        S = oracle_gdn_commit(k, v, a, be, S0, parent, path, np.asarray([path.shape[1]]))
        np.testing.assert_allclose(S.reshape(-1), g["S"][i], rtol=0, atol=1e-12)


def test_beta_zero_is_pure_decay():
    parent = wl.random_tree(np.random.default_rng(1), 12, max_depth=4)[None]
    q, k, v, a, be, S0 = _rand(2, parent)
    o = oracle_gdn_tree(q, k, v, a, np.zeros_like(be), S0, parent)
    for i in range(12):
        path = []
        j = i
        while j >= 0:
            path.append(j)
            j = int(parent[0, j])
        for h in range(2):
            gam = np.prod(a[0, path, h])
            np.testing.assert_allclose(o[0, i, h], gam * S0[0, h] @ q[0, i, 0], rtol=1e-12, atol=1e-12)


def test_unit_write_maps_the_key_to_its_value():
    """alpha = beta = 1, |k| = 1: S' k = S k - (S k) + v = v, whatever S was."""
    parent = wl.random_tree(np.random.default_rng(3), 10, max_depth=5)[None]
    q, k, v, a, be, S0 = _rand(4, parent)
    o = oracle_gdn_tree(k, k, v, np.ones_like(a), np.ones_like(be), S0, parent)     # q = k
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o[0, :, 1], v[0, :, 1], rtol=1e-12, atol=1e-12)


def test_orthonormal_keys_recall_every_value_on_the_path():
    """With alpha = beta = 1 and orthonormal keys along a chain, the state at the end
    maps each key of the chain to its own value."""
    T, d = 5, 8
    rng = np.random.default_rng(5)
    basis, _ = np.linalg.qr(rng.normal(size=(d, d)))
    k = basis[:, :T].T.reshape(1, T, 1, d)
    v = rng.normal(size=(1, T, 1, 3))
    S0 = rng.normal(size=(1, 1, 3, d))
    parent = wl.chain_tree(T)[None]
    S = oracle_gdn_commit(k, v, np.ones((1, T, 1)), np.ones((1, T, 1)), S0, parent,
                          np.arange(T)[None], np.asarray([T]))
    for j in range(T):
        np.testing.assert_allclose(S[0, 0] @ k[0, j, 0], v[0, j, 0], rtol=1e-12, atol=1e-12)


def test_each_node_equals_its_path_decoded_alone():
    parent = wl.random_tree(np.random.default_rng(6), 16, max_depth=5)
    q, k, v, a, be, S0 = _rand(7, parent[None])
    o = oracle_gdn_tree(q, k, v, a, be, S0, parent[None])
    for i in range(16):
        path = []
        j = i
        while j >= 0:
            path.insert(0, j)
            j = int(parent[j])
        n = len(path)
        oc = oracle_gdn_tree(q[:, path], k[:, path], v[:, path], a[:, path], be[:, path], S0, wl.chain_tree(n)[None])
        np.testing.assert_allclose(o[0, i], oc[0, n - 1], rtol=1e-12, atol=1e-12)


def test_identical_siblings_and_commit_at_the_leaf():
    parent = np.asarray([[-1, 0, 0, 1, 2]])
    q, k, v, a, be, S0 = _rand(8, parent)
    for arr in (q, k, v, a, be):
        arr[:, 2] = arr[:, 1]
        arr[:, 4] = arr[:, 3]
    o = oracle_gdn_tree(q, k, v, a, be, S0, parent)
    np.testing.assert_array_equal(o[:, 1], o[:, 2])
    np.testing.assert_array_equal(o[:, 3], o[:, 4])
    # The read-out of the committed state at the leaf is the leaf's output.
    S = oracle_gdn_commit(k, v, a, be, S0, parent, np.asarray([[0, 1, 3]]), np.asarray([3]))
    for h in range(2):
        np.testing.assert_allclose(S[0, h] @ q[0, 3, 0], o[0, 3, h], rtol=1e-12, atol=1e-12)


def test_golden_decoupled_erase_and_write():
    with open(os.path.join(GOLD, "gdn_decoupled.json")) as f:
        g = json.load(f)
    T = len(g["parent"])
    q = np.asarray(g["q"]).reshape(1, T, 1, 2)
    k = np.asarray(g["k"]).reshape(1, T, 1, 2)
    v = np.asarray(g["v"]).reshape(1, T, 1, 1)
    a, be, er = (np.asarray(g[n]).reshape(1, T, 1) for n in ("alpha", "beta", "erase"))
    S0 = np.asarray(g["S0"]).reshape(1, 1, 1, 2)
    parent = np.asarray([g["parent"]])
    o = oracle_gdn_tree(q, k, v, a, be, S0, parent, erase=er)
    np.testing.assert_allclose(o.reshape(-1), g["o"], rtol=0, atol=1e-12)
    for i in range(3):
        path = np.asarray([[0] if i == 0 else [0, i]])
        S = oracle_gdn_commit(k, v, a, be, S0, parent, path, np.asarray([path.shape[1]]), erase=er)
        np.testing.assert_allclose(S.reshape(-1), g["S"][i], rtol=0, atol=1e-12)


def test_zero_erase_is_gated_linear_attention():
    """a = 0: o_i = gamma_i S0 q_i + sum_{j in anc(i)} (gamma_i / gamma_j) beta_j (k_j . q_i) v_j,
    with gamma the product of alpha over the root path (the closed form, summed here
    directly instead of walking the recurrence)."""
    parent = wl.random_tree(np.random.default_rng(11), 14, max_depth=5)[None]
    q, k, v, a, be, S0 = _rand(12, parent, Hv=4, Hk=2, unit=False)
    o = oracle_gdn_tree(q, k, v, a, be, S0, parent, erase=np.zeros_like(be))
    for i in range(14):
        path = []
        j = i
        while j >= 0:
            path.insert(0, j)
            j = int(parent[0, j])
        for h in range(4):
            g = h // 2
            gam = np.cumprod(a[0, path, h])                # gamma of each path node
            ref = gam[-1] * (S0[0, h] @ q[0, i, g])
            for t, j in enumerate(path):
                ref = ref + gam[-1] / gam[t] * be[0, j, h] * (k[0, j, g] @ q[0, i, g]) * v[0, j, h]
            np.testing.assert_allclose(o[0, i, h], ref, rtol=1e-12, atol=1e-12)


def test_packed_triangular_solve_equals_the_walk():
    for seed, T, depth in ((9, 20, 6), (10, 40, 12)):
        parent = np.stack([wl.random_tree(np.random.default_rng(seed + s), T, max_depth=depth) for s in range(2)])
        q, k, v, a, be, S0 = _rand(seed, parent, Hv=4, Hk=2)
        path = np.full((2, T), -1)
        plen = np.zeros(2, int)
        for s in range(2):
            leaf = int(wl.leaves(parent[s])[0])
            nodes = wl.root_path_nodes(parent[s], leaf)
            path[s, :len(nodes)] = nodes
            plen[s] = len(nodes)
        er = np.random.default_rng(seed + 7).uniform(0.0, 1.0, size=be.shape)
        for erase in (None, er):
            o = oracle_gdn_tree(q, k, v, a, be, S0, parent, erase=erase)
            S = oracle_gdn_commit(k, v, a, be, S0, parent, path, plen, erase=erase)
            o2, S2 = packed_gdn(q, k, v, a, be, S0, parent, path, plen, erase=erase)
            np.testing.assert_allclose(o2, o, rtol=1e-10, atol=1e-10)
            np.testing.assert_allclose(S2, S, rtol=1e-10, atol=1e-10)


def test_gdn_pins_catch_planted_mistakes():
    import oracle.gdn as gd
    src = open(gd.__file__).read()
    step = "    return a * (S - er * np.outer(S @ kj, kj)) + be * np.outer(vj, kj)\n"
    assert src.count(step) == 1
    mutants = {
        "gate after the write": (step, "    return a * (S - er * np.outer(S @ kj, kj) + be * np.outer(vj, kj))\n"),
        "no beta on the write": (step, "    return a * (S - er * np.outer(S @ kj, kj)) + np.outer(vj, kj)\n"),
        "no erase (plain linear attention)": (step, "    return a * S + be * np.outer(vj, kj)\n"),
        "write strength erases": (step, "    return a * (S - be * np.outer(S @ kj, kj)) + be * np.outer(vj, kj)\n"),
        "erase strength writes": (step, "    return a * (S - er * np.outer(S @ kj, kj)) + er * np.outer(vj, kj)\n"),
        "heads round robin": ("                g = h // grp\n                S = S0[s, h].copy()\n                for j in path:",
                              "                g = h % Hk\n                S = S0[s, h].copy()\n                for j in path:"),
        "root skipped": ("    return out[::-1]\n", "    return out[::-1][1:]\n"),
    }
    checks = [test_golden_hand_worked_tree, test_beta_zero_is_pure_decay, test_unit_write_maps_the_key_to_its_value,
              test_orthonormal_keys_recall_every_value_on_the_path, test_each_node_equals_its_path_decoded_alone,
              test_identical_siblings_and_commit_at_the_leaf, test_golden_decoupled_erase_and_write,
              test_zero_erase_is_gated_linear_attention, test_packed_triangular_solve_equals_the_walk]
    g = globals()
    for name, (old, new) in mutants.items():
        assert src.count(old) >= 1, name
        ns = {"__name__": "mutant"}
        exec(compile(src.replace(old, new), "mutant", "exec"), ns)
        saved = {n: g[n] for n in ("oracle_gdn_tree", "oracle_gdn_commit")}
        g["oracle_gdn_tree"], g["oracle_gdn_commit"] = ns["oracle_gdn_tree"], ns["oracle_gdn_commit"]
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
            g.update(saved)
