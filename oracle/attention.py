"""Tree-masked attention over a packed draft tree -- TEST INFRASTRUCTURE ONLY.

The Transformer layers of a hybrid SSM-attention model verify the same packed
tree as its SSM layers ("STree: Speculative Tree Decoding for Hybrid State Space
Models": abstract, "hybrid architectures of SSMs and Transformer layers"; scime.ai
summary, "Approach": the packed tree sequence is processed "with a tree mask").
Read plainly: every tree node attends to the whole cached context and to the tree
nodes on its own root path (its ancestors and itself), never to its siblings or
their subtrees -- each node sees exactly the sequence it would see had its path
been decoded on its own.

Written out from that definition in fp64: for every sequence, node and query
head, walk the root path, gather the visible keys and values (context first,
then the path from the root), and apply softmax attention.  Grouped query heads
share key/value heads: query head h reads key/value head h // (Hq / Hkv).
"""
from __future__ import annotations

import numpy as np


def root_path(parent_row, i: int) -> list:
    """Nodes from the root to i (inclusive), following parent[] up to -1."""
    out = []
    j = int(i)
    while j >= 0:
        out.append(j)
        j = int(parent_row[j])
    return out[::-1]


def oracle_tree_attention(q, k_ctx, v_ctx, k_tree, v_tree, parent, scale: float, ctx_len=None):
    """q [b, T, Hq, d]; k_ctx, v_ctx [b, S, Hkv, d]; k_tree, v_tree [b, T, Hkv, d];
    parent [b, T] int (a packed tree per sequence); ctx_len [b] int (valid context
    positions per sequence, default S).  Returns o [b, T, Hq, d] in fp64:

        o[b, i, h] = sum_j w_j v_j,  w = softmax(scale * q[b, i, h] . k_j)

    over j = the context positions 0 .. ctx_len[b] - 1, then the root path of i."""
    q = np.asarray(q, np.float64)
    k_ctx, v_ctx = np.asarray(k_ctx, np.float64), np.asarray(v_ctx, np.float64)
    k_tree, v_tree = np.asarray(k_tree, np.float64), np.asarray(v_tree, np.float64)
    parent = np.asarray(parent)
    b, T, Hq, d = q.shape
    S, Hkv = k_ctx.shape[1], k_ctx.shape[2]
    if ctx_len is None:
        ctx_len = np.full(b, S)
    group = Hq // Hkv
    out = np.zeros((b, T, Hq, d))
    for s in range(b):
        L = int(ctx_len[s])
        for i in range(T):
            path = root_path(parent[s], i)
            for h in range(Hq):
                g = h // group
                keys = np.concatenate([k_ctx[s, :L, g], k_tree[s, path, g]], axis=0)
                vals = np.concatenate([v_ctx[s, :L, g], v_tree[s, path, g]], axis=0)
                scores = scale * (keys @ q[s, i, h])
                w = np.exp(scores - scores.max())
                out[s, i, h] = (w / w.sum()) @ vals
    return out
