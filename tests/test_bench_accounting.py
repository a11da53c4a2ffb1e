"""CPU checks of the benchmark's accounting and of the synthetic generators it uses.

The algorithmic bytes are the denominator-free half of the roofline: every tensor
of one fused launch moved once (h0 and h_new fp32, x and y in the input dtype, dt,
B, C, A, D, the tree and the path).  They are checked against the workloads' byte
counts worked out by hand (m2_2p7b 5.56 MB, hyb8b 37.8 MB, serve64 422 MB per
layer, wide256 1.63 GB) and against a direct recount from the tensor shapes.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from hybrid_packed_tree_b200 import workloads as wl  # noqa: E402


@pytest.mark.parametrize("name,mb", [("m2_2p7b", 5.56), ("hyb8b", 37.8), ("serve64", 422.0), ("wide256", 1630.0)])
def test_algorithmic_bytes_match_the_hand_counts(name, mb):
    w = wl.make_workload(name, layers=1)
    total = sum(bench.algorithmic_bytes(w).values())
    assert abs(total / 1e6 - mb) / mb < 0.01, (name, total)


def test_algorithmic_bytes_recount_from_tensor_shapes():
    w = wl.make_workload("hyb8b", layers=1)
    L = w.layers[0]
    e = 2                                          # bf16 inputs, stored as uint16 bits
    want = (L.h0.nbytes * 2 + L.x.size * e * 2 + L.dt.size * e + L.B.size * e + L.C.size * e
            + L.A.nbytes + L.D.nbytes + w.parent.nbytes + w.path.nbytes + w.path_len.nbytes)
    assert sum(bench.algorithmic_bytes(w).values()) == want


def test_unrolled_summary_divides_the_step_by_its_layers():
    o = {"ms_per_step": 0.8, "config": {"layers": 8}}
    u = bench.unrolled_summary(o, {"ms_per_launch": 4.0})
    assert u["packed_ms_per_layer"] == pytest.approx(0.1)
    assert u["unrolled_over_packed_time"] == pytest.approx(40.0)


def test_acceptance_inputs_plant_a_followable_path():
    """Distinct tokens among siblings, and along the planted path the largest logit
    after each node is the next node's token (the generator only; the verifier is
    pinned elsewhere)."""
    w = wl.make_workload("serve64", batch=3, layers=1)
    logits, tokens, planted = wl.acceptance_inputs(w.parent, 300, seed=3, dtype="f32")
    for s, nodes in enumerate(planted):
        for u in range(w.n_nodes):
            kids = np.nonzero(w.parent[s] == u)[0]
            assert len(set(tokens[s, kids].tolist())) == len(kids)
        assert nodes[0] == 0 and nodes[-1] in set(wl.leaves(w.parent[s]).tolist())
        for u, v in zip(nodes[:-1], nodes[1:]):
            assert int(np.argmax(logits[s, u])) == int(tokens[s, v])
    bits, _, _ = wl.acceptance_inputs(w.parent, 300, seed=3, dtype="bf16")
    assert bits.dtype == np.uint16 and bits.shape == logits.shape
