"""Pins of the tree-masked attention oracle (oracle/attention.py) against facts
that do not come from the oracle itself: a hand-worked case, causal attention on
a chain (a masked-matrix formulation), each node against its own path decoded as
a sequence, identical siblings, the uniform-score closed form, invariance of
softmax to a shift shared by all keys, grouped heads against repeated heads, and
a mutation check that plants plausible mistakes in a copy of the oracle.
"""
import json
import os

import numpy as np
import pytest
from scipy.special import softmax

from hybrid_packed_tree_b200 import workloads as wl
from oracle.attention import oracle_tree_attention, root_path

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, b, T, S, Hq, Hkv, d):
    return (rng.normal(size=(b, T, Hq, d)), rng.normal(size=(b, S, Hkv, d)), rng.normal(size=(b, S, Hkv, d)),
            rng.normal(size=(b, T, Hkv, d)), rng.normal(size=(b, T, Hkv, d)))


def test_golden_hand_worked_case():
    with open(os.path.join(GOLD, "tree_attention.json")) as f:
        g = json.load(f)
    T = len(g["parent"])
    o = oracle_tree_attention(np.asarray(g["q"]).reshape(1, T, 1, 2), np.asarray(g["k_ctx"]).reshape(1, -1, 1, 2),
                              np.asarray(g["v_ctx"]).reshape(1, -1, 1, 2), np.asarray(g["k_tree"]).reshape(1, T, 1, 2),
                              np.asarray(g["v_tree"]).reshape(1, T, 1, 2), np.asarray([g["parent"]]), g["scale"],
                              ctx_len=np.asarray([g["ctx_len"]]))
    np.testing.assert_allclose(o.reshape(T, 2), np.asarray(g["o"]), rtol=0, atol=1e-12)


def test_chain_is_causal_attention():
    """On a chain, node i sees the context and nodes 0..i: causal attention,
    computed here as one masked score matrix."""
    rng = np.random.default_rng(1)
    T, S, d = 9, 5, 8
    q, kc, vc, kt, vt = _rand(rng, 1, T, S, 1, 1, d)
    o = oracle_tree_attention(q, kc, vc, kt, vt, wl.chain_tree(T)[None], 0.3)
    K = np.concatenate([kc[0, :, 0], kt[0, :, 0]])
    V = np.concatenate([vc[0, :, 0], vt[0, :, 0]])
    scores = 0.3 * q[0, :, 0] @ K.T
    mask = np.arange(S + T)[None, :] <= (S + np.arange(T))[:, None]
    ref = softmax(np.where(mask, scores, -np.inf), axis=1) @ V
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=1e-12, atol=1e-12)


def test_each_node_equals_its_path_decoded_alone():
    rng = np.random.default_rng(2)
    parent = wl.random_tree(np.random.default_rng(3), 20, max_depth=5)
    T, S, d = 20, 7, 4
    q, kc, vc, kt, vt = _rand(rng, 1, T, S, 2, 1, d)
    o = oracle_tree_attention(q, kc, vc, kt, vt, parent[None], 0.5)
    for i in range(T):
        path = root_path(parent, i)
        n = len(path)
        oi = oracle_tree_attention(q[:, path], kc, vc, kt[:, path], vt[:, path], wl.chain_tree(n)[None], 0.5)
        np.testing.assert_allclose(o[0, i], oi[0, n - 1], rtol=1e-12, atol=1e-12)


def test_identical_siblings_give_identical_outputs():
    rng = np.random.default_rng(4)
    parent = np.asarray([[-1, 0, 0, 1, 2]])
    q, kc, vc, kt, vt = _rand(rng, 1, 5, 3, 2, 2, 4)
    for a in (q, kt, vt):
        a[:, 2] = a[:, 1]
        a[:, 4] = a[:, 3]
    o = oracle_tree_attention(q, kc, vc, kt, vt, parent, 1.0)
    np.testing.assert_array_equal(o[:, 1], o[:, 2])
    np.testing.assert_array_equal(o[:, 3], o[:, 4])


def test_zero_query_is_the_mean_of_visible_values():
    rng = np.random.default_rng(5)
    parent = np.asarray([[-1, 0, 1, 0, 3]])
    _, kc, vc, kt, vt = _rand(rng, 1, 5, 6, 1, 1, 3)
    q = np.zeros((1, 5, 1, 3))
    o = oracle_tree_attention(q, kc, vc, kt, vt, parent, 1.0, ctx_len=np.asarray([4]))
    for i in range(5):
        vis = np.concatenate([vc[0, :4, 0], vt[0, root_path(parent[0], i), 0]])
        np.testing.assert_allclose(o[0, i, 0], vis.mean(axis=0), rtol=1e-12, atol=1e-12)


def test_shift_shared_by_all_keys_changes_nothing():
    rng = np.random.default_rng(6)
    parent = wl.random_tree(np.random.default_rng(7), 12, max_depth=4)[None]
    q, kc, vc, kt, vt = _rand(rng, 1, 12, 5, 2, 1, 4)
    c = rng.normal(size=4)
    o1 = oracle_tree_attention(q, kc, vc, kt, vt, parent, 0.7)
    o2 = oracle_tree_attention(q, kc + c, vc, kt + c, vt, parent, 0.7)
    np.testing.assert_allclose(o1, o2, rtol=1e-10, atol=1e-10)


def test_grouped_heads_equal_repeated_heads():
    rng = np.random.default_rng(8)
    parent = np.asarray([wl.random_tree(np.random.default_rng(9), 10, max_depth=4)] * 2)
    q, kc, vc, kt, vt = _rand(rng, 2, 10, 4, 8, 2, 4)
    o = oracle_tree_attention(q, kc, vc, kt, vt, parent, 0.25, ctx_len=np.asarray([4, 2]))
    rep = [np.repeat(a, 4, axis=2) for a in (kc, vc, kt, vt)]
    o_mha = oracle_tree_attention(q, *rep, parent, 0.25, ctx_len=np.asarray([4, 2]))
    np.testing.assert_allclose(o, o_mha, rtol=1e-12, atol=1e-12)


def test_attention_pins_catch_planted_mistakes():
    """Copies of the oracle with one planted mistake each must fail a pin above."""
    import oracle.attention as att
    src = open(att.__file__).read()
    mutants = {
        "path without the node itself": ("    out = []\n    j = int(i)\n", "    out = []\n    j = int(parent_row[i])\n"),
        "siblings visible": ("            path = root_path(parent[s], i)\n", "            path = list(range(i + 1))\n"),
        "heads mapped round robin": ("                g = h // group\n", "                g = h % Hkv\n"),
        "scale dropped": ("                scores = scale * (keys @ q[s, i, h])\n",
                          "                scores = keys @ q[s, i, h]\n"),
        "context length ignored": ("        L = int(ctx_len[s])\n", "        L = S\n"),
    }
    checks = [test_golden_hand_worked_case, test_chain_is_causal_attention, test_each_node_equals_its_path_decoded_alone,
              test_identical_siblings_give_identical_outputs, test_zero_query_is_the_mean_of_visible_values,
              test_shift_shared_by_all_keys_changes_nothing, test_grouped_heads_equal_repeated_heads]
    for name, (old, new) in mutants.items():
        assert src.count(old) == 1, name
        ns = {"__name__": "mutant"}
        exec(compile(src.replace(old, new), "mutant", "exec"), ns)
        saved = (globals()["oracle_tree_attention"], globals()["root_path"])
        globals()["oracle_tree_attention"], globals()["root_path"] = ns["oracle_tree_attention"], ns["root_path"]
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
            globals()["oracle_tree_attention"], globals()["root_path"] = saved
