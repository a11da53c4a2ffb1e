"""Seeded synthetic inputs for the packed-tree SSM scan.

This module only draws inputs: tree topologies, accepted paths and the tensors
of the scan, with the value distributions of the workloads below.  It holds none
of the scan's arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it.

Every workload is one of the shapes the STree pages time (a Mamba2-2.7B layer
with a 15-token tree, an 8B-class hybrid layer, batched serving, wide trees);
the pages' own datasets are not needed because the scan's cost does not depend
on token values.  Draws are made in fp64 with ``numpy.random.default_rng`` and
then rounded to the stored dtype: fp32 by numpy's round-to-nearest-even, bf16 by
round-to-nearest-even of that fp32 value (``bf16_bits``).  bf16 tensors are kept
as raw uint16 bit patterns.

Distributions: x ~ N(0,1); dt = softplus(N(-2, 0.5)); A_h = -exp(U(0, ln 16));
D ~ N(0,1); B, C ~ N(0,1)/sqrt(dstate); h0 ~ N(0, 1) for the tiny case and
N(0, 0.1) (standard deviation 0.1) otherwise.  Draw order: parent, A, D, dt, x,
B, C, h0, path; layers draw A..h0 one after another.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# --------------------------------------------------------------------------- dtype helpers


def bf16_bits(a) -> np.ndarray:
    """fp64/fp32 values -> bf16 bit patterns (uint16), round to nearest even via fp32."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def stored_to_f64(a, dtype: str) -> np.ndarray:
    """Exact fp64 copy of a stored tensor (fp32 array, or bf16 bits for 'bf16')."""
    if dtype == "bf16":
        return bf16_to_f64(a)
    return np.asarray(a, dtype=np.float64)


def _round(a64, dtype: str) -> np.ndarray:
    return bf16_bits(a64) if dtype == "bf16" else np.asarray(a64, dtype=np.float32)


# --------------------------------------------------------------------------- trees


def bfs_relabel(parent) -> np.ndarray:
    """Relabel a rooted tree (root = node whose parent is -1) in breadth-first order.

    Children are visited in increasing old label.  Returns the new parent array.
    """
    parent = np.asarray(parent, np.int64)
    T = parent.shape[0]
    children = [[] for _ in range(T)]
    root = -1
    for i in range(T):
        if parent[i] < 0:
            root = i
        else:
            children[parent[i]].append(i)
    order = [root]
    head = 0
    while head < len(order):
        order.extend(sorted(children[order[head]]))
        head += 1
    new_of = np.empty(T, np.int64)
    new_of[np.asarray(order)] = np.arange(T)
    out = np.empty(T, np.int32)
    for old in range(T):
        out[new_of[old]] = -1 if parent[old] < 0 else new_of[parent[old]]
    return out


def random_tree(rng, T: int, max_depth: int, max_children: int | None = None,
                max_width: int | None = None, spine: int = 0) -> np.ndarray:
    """Random rooted tree of T nodes, attached one node at a time, BFS-relabelled.

    A node joins under a uniformly drawn eligible parent: depth < max_depth,
    fewer than ``max_children`` children, and a child level holding fewer than
    ``max_width`` nodes.  ``spine`` first lays a chain root->...->node ``spine``.
    """
    parent = np.full(T, -1, np.int64)
    depth = np.zeros(T, np.int64)
    nchild = np.zeros(T, np.int64)
    width = np.zeros(T + 1, np.int64)
    width[0] = 1
    for i in range(1, min(spine, T - 1) + 1):
        parent[i], depth[i] = i - 1, i
        nchild[i - 1] += 1
        width[i] += 1
    for i in range(min(spine, T - 1) + 1, T):
        elig = [p for p in range(i)
                if depth[p] < max_depth
                and (max_children is None or nchild[p] < max_children)
                and (max_width is None or width[depth[p] + 1] < max_width)]
        if not elig:
            raise ValueError("tree constraints cannot place every node")
        p = elig[int(rng.integers(len(elig)))]
        parent[i], depth[i] = p, depth[p] + 1
        nchild[p] += 1
        width[depth[i]] += 1
    return bfs_relabel(parent)


def chain_tree(T: int) -> np.ndarray:
    return np.arange(-1, T - 1, dtype=np.int32)


def node_depths(parent_row) -> np.ndarray:
    """Depth of every node (root 0); parents precede children."""
    d = np.zeros(len(parent_row), np.int64)
    for i, p in enumerate(parent_row):
        d[i] = 0 if p < 0 else d[p] + 1
    return d


def root_path_nodes(parent_row, node: int) -> list:
    out = []
    while node != -1:
        out.append(int(node))
        node = int(parent_row[node])
    return out[::-1]


def leaves(parent_row) -> np.ndarray:
    has_child = np.zeros(len(parent_row), bool)
    for p in parent_row:
        if p >= 0:
            has_child[p] = True
    return np.nonzero(~has_child)[0]


def unroll_paths(parent: np.ndarray):
    """Every root-to-leaf path of each sequence's tree (the unrolled form of the
    tree), leaves in increasing order, padded to the largest leaf count with
    empty paths.  Returns paths [b, n_paths, max_depth] int32 (-1 past each
    path's end) and path_len [b, n_paths] int32."""
    parent = np.asarray(parent)
    per_seq = [[root_path_nodes(row, int(l)) for l in leaves(row)] for row in parent]
    n_paths = max(len(ps) for ps in per_seq)
    max_depth = max(len(p) for ps in per_seq for p in ps)
    paths = np.full((len(per_seq), n_paths, max_depth), -1, np.int32)
    path_len = np.zeros((len(per_seq), n_paths), np.int32)
    for b, ps in enumerate(per_seq):
        for k, nodes in enumerate(ps):
            paths[b, k, :len(nodes)] = nodes
            path_len[b, k] = len(nodes)
    return paths, path_len


def acceptance_inputs(parent: np.ndarray, vocab: int, seed: int = 7, dtype: str = "bf16"):
    """Synthetic target logits and draft tokens for tree verification: tokens
    distinct among each node's children, logits ~ N(0,1) with, along one random
    root-to-leaf path per sequence, the next node's token raised above the row's
    maximum (so that a greedy verifier follows that path) and one raised token after
    the leaf.  Returns (logits [b,T,V] fp32 or bf16 bits, tokens [b,T] int32,
    planted paths as lists)."""
    parent = np.asarray(parent)
    rng = np.random.default_rng(seed)
    b, T = parent.shape
    tokens = np.zeros((b, T), np.int32)
    logits = rng.normal(size=(b, T, vocab)).astype(np.float32)
    planted = []
    for s_ in range(b):
        for u in range(T):
            kids = np.nonzero(parent[s_] == u)[0]
            if len(kids):
                tokens[s_, kids] = rng.choice(vocab, size=len(kids), replace=False)
        leaf = int(rng.choice(leaves(parent[s_])))
        nodes = root_path_nodes(parent[s_], leaf)
        for u, v in zip(nodes[:-1], nodes[1:]):
            logits[s_, u, tokens[s_, v]] = logits[s_, u].max() + 1.0
        logits[s_, leaf, int(rng.integers(vocab))] = logits[s_, leaf].max() + 1.0
        planted.append(nodes)
    if dtype == "bf16":
        logits = bf16_bits(logits)
    return logits, tokens, planted


def sampling_inputs(parent: np.ndarray, vocab: int, seed: int = 11, dtype: str = "bf16",
                    draft_std: float = 3.0, target_noise: float = 0.5):
    """Synthetic inputs for stochastic tree verification: draft logits ~ N(0,
    draft_std), target logits = draft logits + N(0, target_noise) (a draft close to
    the target), children's tokens distinct, each from the parent's four largest
    draft logits with probability 0.7 and uniform over the vocabulary otherwise,
    and the uniforms (u_accept [b,T], u_bonus [b], fp32 in [0, 1)).  Returns
    (target, draft) logits [b,T,V] (fp32, or bf16 bits), tokens, u_accept, u_bonus."""
    parent = np.asarray(parent)
    rng = np.random.default_rng(seed)
    b, T = parent.shape
    draft = rng.normal(0.0, draft_std, size=(b, T, vocab)).astype(np.float32)
    target = (draft + rng.normal(0.0, target_noise, size=(b, T, vocab))).astype(np.float32)
    tokens = np.zeros((b, T), np.int32)
    for s_ in range(b):
        for u in range(T):
            kids = np.nonzero(parent[s_] == u)[0]
            if not len(kids):
                continue
            top = np.argsort(draft[s_, u])[-4:]
            used = set()
            for c in kids:
                while True:
                    t = int(rng.choice(top)) if rng.uniform() < 0.7 else int(rng.integers(vocab))
                    if t not in used:
                        break
                used.add(t)
                tokens[s_, c] = t
    u_accept = rng.uniform(size=(b, T)).astype(np.float32)
    u_bonus = rng.uniform(size=b).astype(np.float32)
    if dtype == "bf16":
        target, draft = bf16_bits(target), bf16_bits(draft)
    return target, draft, tokens, u_accept, u_bonus


@dataclass
class GdnInputs:
    """One gated-delta-rule layer over packed trees (bf16 q/k/v, fp32 gates and state)."""
    q: np.ndarray          # [b, T, Hk, dk]  bf16 bits (or fp32)
    k: np.ndarray          # [b, T, Hk, dk]  unit rows before rounding
    v: np.ndarray          # [b, T, Hv, dv]
    alpha: np.ndarray      # [b, T, Hv] fp32 in (0, 1]
    beta: np.ndarray       # [b, T, Hv] fp32 in (0, 1)
    S0: np.ndarray         # [b, Hv, dv, dk] fp32
    parent: np.ndarray
    path: np.ndarray
    path_len: np.ndarray
    dtype: str

    def f64(self):
        return {"q": stored_to_f64(self.q, self.dtype), "k": stored_to_f64(self.k, self.dtype),
                "v": stored_to_f64(self.v, self.dtype), "alpha": self.alpha.astype(np.float64),
                "beta": self.beta.astype(np.float64), "S0": self.S0.astype(np.float64)}


def gdn_inputs(parent: np.ndarray, path: np.ndarray, path_len: np.ndarray, *, heads_v: int = 32,
               heads_k: int = 16, dk: int = 128, dv: int = 128, seed: int = 31, dtype: str = "bf16",
               s0_std: float = 0.1) -> GdnInputs:
    """Seeded inputs of a gated-delta-rule layer on the given trees: q, k unit
    vectors (Gaussian directions), v ~ N(0, 1), alpha = exp(-U(0.01, 0.3)),
    beta = 1 / (1 + exp(-N(0, 1))), S0 ~ N(0, s0_std)."""
    parent = np.asarray(parent, np.int32)
    rng = np.random.default_rng(seed)
    b, T = parent.shape

    def unit(shape):
        a = rng.normal(size=shape)
        return a / np.linalg.norm(a, axis=-1, keepdims=True)

    q = _round(unit((b, T, heads_k, dk)), dtype)
    k = _round(unit((b, T, heads_k, dk)), dtype)
    v = _round(rng.normal(size=(b, T, heads_v, dv)), dtype)
    alpha = np.exp(-rng.uniform(0.01, 0.3, size=(b, T, heads_v))).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-rng.normal(size=(b, T, heads_v))))).astype(np.float32)
    S0 = rng.normal(0.0, s0_std, size=(b, heads_v, dv, dk)).astype(np.float32)
    return GdnInputs(q=q, k=k, v=v, alpha=alpha, beta=beta, S0=S0, parent=parent,
                     path=np.asarray(path, np.int32), path_len=np.asarray(path_len, np.int32), dtype=dtype)


def attention_inputs(parent: np.ndarray, ctx_cap: int, ctx_len, *, heads_q: int = 32, heads_kv: int = 8,
                     head_dim: int = 128, seed: int = 51, stale=np.nan):
    """Seeded inputs of a tree-masked attention layer (bf16 bits): q [b, T, Hq, d],
    the context cache k_ctx, v_ctx [b, ctx_cap, Hkv, d] whose positions past each
    sequence's ctx_len hold `stale` (they must never be read), and the tree's own
    k_tree, v_tree [b, T, Hkv, d]; all valid values ~ N(0, 1)."""
    parent = np.asarray(parent, np.int32)
    rng = np.random.default_rng(seed)
    b, T = parent.shape
    ctx_len = np.asarray(ctx_len, np.int32).reshape(b)
    q = bf16_bits(rng.normal(size=(b, T, heads_q, head_dim)).astype(np.float32))
    kc = rng.normal(size=(b, ctx_cap, heads_kv, head_dim)).astype(np.float32)
    vc = rng.normal(size=(b, ctx_cap, heads_kv, head_dim)).astype(np.float32)
    for s_ in range(b):
        kc[s_, ctx_len[s_]:] = stale
        vc[s_, ctx_len[s_]:] = stale
    kt = bf16_bits(rng.normal(size=(b, T, heads_kv, head_dim)).astype(np.float32))
    vt = bf16_bits(rng.normal(size=(b, T, heads_kv, head_dim)).astype(np.float32))
    return {"q": q, "k_ctx": bf16_bits(kc), "v_ctx": bf16_bits(vc), "k_tree": kt, "v_tree": vt,
            "ctx_len": ctx_len, "parent": parent, "scale": 1.0 / np.sqrt(head_dim)}


# --------------------------------------------------------------------------- workloads


@dataclass
class LayerInputs:
    """One layer's tensors in their stored dtypes (bf16 as uint16 bits)."""
    x: np.ndarray    # [b,T,H,P]
    dt: np.ndarray   # [b,T,H]
    A: np.ndarray    # [H] fp32
    B: np.ndarray    # [b,T,G,N]
    C: np.ndarray    # [b,T,G,N]
    D: np.ndarray    # [H] fp32
    h0: np.ndarray   # [b,H,P,N] fp32


@dataclass
class Workload:
    name: str
    batch: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    n_nodes: int
    dtype: str                      # "f32" or "bf16": dtype of x, dt, B, C (and y)
    parent: np.ndarray              # int32 [b,T]
    path: np.ndarray                # int32 [b,maxlen], padded with -1
    path_len: np.ndarray            # int32 [b]
    layers: list = field(default_factory=list)

    @property
    def maxlen(self) -> int:
        return int(self.path.shape[1])

    @property
    def nlayers(self) -> int:
        return len(self.layers)

    def f64(self, layer: int = 0) -> dict:
        """Exact fp64 copies of one layer's stored tensors (what the oracle reads)."""
        L = self.layers[layer]
        return {k: stored_to_f64(getattr(L, k), self.dtype if k in ("x", "dt", "B", "C") else "f32")
                for k in ("x", "dt", "A", "B", "C", "D", "h0")}


# name: (config index, batch, layers, H, P, N, G, T, dtype, h0 std)
SPECS = {
    "tiny":          (0, 1, 1, 2, 16, 16, 1, 7, "f32", 1.0),
    "m2_2p7b":       (1, 1, 1, 80, 64, 128, 1, 15, "bf16", 0.1),
    "m2_2p7b_16":    (1, 1, 1, 80, 64, 128, 1, 16, "bf16", 0.1),
    "hyb8b":         (2, 8, 1, 32, 128, 128, 8, 26, "bf16", 0.1),
    "serve64":       (3, 64, 8, 80, 64, 128, 1, 64, "bf16", 0.1),
    "wide256":       (4, 256, 1, 64, 64, 128, 1, 128, "bf16", 0.1),
    "wide256_chain": (4, 256, 1, 64, 64, 128, 1, 128, "bf16", 0.1),
}

# Trees fixed by the workload descriptions.
TINY_PARENT = [-1, 0, 0, 1, 1, 2, 2]                       # full binary tree, depth 2
# Root, 3 children, 2 kids each, then 1 kid for the first five grandchildren in
# BFS order: 15 nodes (the listed shape has 16; 15 tokens is what is timed).
M2_PARENT_15 = [-1, 0, 0, 0, 1, 1, 2, 2, 3, 3, 4, 5, 6, 7, 8]
# The literal 16-node shape: root, 3 children, 2 kids each, 1 kid each.
M2_PARENT_16 = [-1, 0, 0, 0, 1, 1, 2, 2, 3, 3, 4, 5, 6, 7, 8, 9]


def _topologies(rng, name: str, batch: int, T: int) -> np.ndarray:
    if name == "tiny":
        rows = [TINY_PARENT] * batch
    elif name == "m2_2p7b":
        rows = [M2_PARENT_15] * batch
    elif name == "m2_2p7b_16":
        rows = [M2_PARENT_16] * batch
    elif name == "hyb8b":
        rows = [random_tree(rng, T, max_depth=5, max_children=4, spine=5) for _ in range(batch)]
    elif name == "serve64":
        rows = [random_tree(rng, T, max_depth=8) for _ in range(batch)]
    elif name == "wide256":
        rows = [random_tree(rng, T, max_depth=10, max_width=16) for _ in range(batch)]
    elif name == "wide256_chain":
        rows = [chain_tree(T)] * batch
    else:
        raise KeyError(name)
    return np.ascontiguousarray(np.asarray(rows, np.int32).reshape(batch, T))


def _paths(rng, name: str, parent: np.ndarray, maxlen: int):
    batch = parent.shape[0]
    path = np.full((batch, maxlen), -1, np.int32)
    plen = np.zeros(batch, np.int32)
    for b in range(batch):
        row = parent[b]
        if name == "tiny":
            nodes = [0, 1, 3]                                   # root -> node 3
        elif name == "serve64":
            d = node_depths(row)
            want = int(rng.integers(1, 9))                      # length 1..8
            want = min(want, int(d.max()) + 1)
            cand = np.nonzero(d == want - 1)[0]
            nodes = root_path_nodes(row, int(cand[int(rng.integers(len(cand)))]))
        else:                                                   # a random leaf
            lv = leaves(row)
            nodes = root_path_nodes(row, int(lv[int(rng.integers(len(lv)))]))
        path[b, :len(nodes)] = nodes
        plen[b] = len(nodes)
    return path, plen


def make_workload(name: str, seed: int | None = None, batch: int | None = None,
                  layers: int | None = None, maxlen: int | None = None) -> Workload:
    """Draw a workload by name; ``batch`` / ``layers`` override the sizes."""
    idx, b0, l0, H, P, N, G, T, dtype, h0_std = SPECS[name]
    batch = b0 if batch is None else int(batch)
    nl = l0 if layers is None else int(layers)
    rng = np.random.default_rng(1000 + idx if seed is None else seed)
    parent = _topologies(rng, name, batch, T)
    if maxlen is None:
        maxlen = T
    layer_list = []
    for _ in range(nl):
        A = np.asarray(-np.exp(rng.uniform(0.0, np.log(16.0), size=H)), np.float32)
        D = np.asarray(rng.normal(0.0, 1.0, size=H), np.float32)
        dt = _round(np.logaddexp(0.0, rng.normal(-2.0, 0.5, size=(batch, T, H))), dtype)
        x = _round(rng.normal(0.0, 1.0, size=(batch, T, H, P)), dtype)
        Bm = _round(rng.normal(0.0, 1.0, size=(batch, T, G, N)) / np.sqrt(N), dtype)
        Cm = _round(rng.normal(0.0, 1.0, size=(batch, T, G, N)) / np.sqrt(N), dtype)
        h0 = np.asarray(rng.normal(0.0, h0_std, size=(batch, H, P, N)), np.float32)
        layer_list.append(LayerInputs(x=x, dt=dt, A=A, B=Bm, C=Cm, D=D, h0=h0))
    path, plen = _paths(rng, name, parent, maxlen)
    return Workload(name=name, batch=batch, nheads=H, headdim=P, dstate=N, ngroups=G,
                    n_nodes=T, dtype=dtype, parent=parent, path=path, path_len=plen,
                    layers=layer_list)


def custom_workload(parent, *, nheads: int, headdim: int, dstate: int, ngroups: int = 1,
                    dtype: str = "f32", seed: int = 0, h0_std: float = 1.0,
                    path=None, path_len=None, nlayers: int = 1) -> Workload:
    """Same distributions on a caller-given parent array [b,T] (tests' edge cases)."""
    parent = np.ascontiguousarray(np.asarray(parent, np.int32))
    if parent.ndim == 1:
        parent = parent[None, :]
    batch, T = parent.shape
    H, P, N, G = nheads, headdim, dstate, ngroups
    rng = np.random.default_rng(seed)
    layer_list = []
    for _ in range(nlayers):
        A = np.asarray(-np.exp(rng.uniform(0.0, np.log(16.0), size=H)), np.float32)
        D = np.asarray(rng.normal(0.0, 1.0, size=H), np.float32)
        dt = _round(np.logaddexp(0.0, rng.normal(-2.0, 0.5, size=(batch, T, H))), dtype)
        x = _round(rng.normal(0.0, 1.0, size=(batch, T, H, P)), dtype)
        Bm = _round(rng.normal(0.0, 1.0, size=(batch, T, G, N)) / np.sqrt(N), dtype)
        Cm = _round(rng.normal(0.0, 1.0, size=(batch, T, G, N)) / np.sqrt(N), dtype)
        h0 = np.asarray(rng.normal(0.0, h0_std, size=(batch, H, P, N)), np.float32)
        layer_list.append(LayerInputs(x=x, dt=dt, A=A, B=Bm, C=Cm, D=D, h0=h0))
    if path is None:
        maxlen = max(T, 1)
        path = np.full((batch, maxlen), -1, np.int32)
        path_len = np.zeros(batch, np.int32)
        for b in range(batch):
            if T == 0:
                continue
            lv = leaves(parent[b])
            nodes = root_path_nodes(parent[b], int(lv[int(rng.integers(len(lv)))]))
            path[b, :len(nodes)] = nodes
            path_len[b] = len(nodes)
    path = np.ascontiguousarray(np.asarray(path, np.int32).reshape(batch, -1))
    path_len = np.ascontiguousarray(np.asarray(path_len, np.int32).reshape(batch))
    return Workload(name="custom", batch=batch, nheads=H, headdim=P, dstate=N, ngroups=G,
                    n_nodes=T, dtype=dtype, parent=parent, path=path, path_len=path_len,
                    layers=layer_list)
