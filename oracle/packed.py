"""Second fp64 formulation of the packed-tree scan -- a self-check of the walk only.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"STree: Speculative Tree Decoding for Hybrid State Space Models" (scime.ai
summary, section "Approach") states the packed form: accumulate the diagonal log
transitions along each node's ancestors, ``A_tree = L . log A``, where L is the
tree's ancestor (mask) matrix.  Written out for one (sequence, head):

    a_j   = dt_j * A_h                      (log of node j's own decay)
    Lc    = Anc @ a                         (tree cumsum; Anc[i,j] = j on root->i path)
    y_i   = exp(Lc_i) * (C_i . h0^T)                      (root term)
          + sum_{j in anc(i)} exp(Lc_i - Lc_j) (C_i . B_j) dt_j x_j   (tree term)
          + D_h x_i                                        (skip)
    h_new = exp(Lc_leaf) h0 + sum_{j on path} exp(Lc_leaf - Lc_j) dt_j outer(x_j, B_j)

This is the closed form the walk must equal; it uses numpy matmuls only and no
code of the walk.  Non-ancestor pairs are never exponentiated.
"""
from __future__ import annotations

import numpy as np


def ancestor_matrix(parent_row) -> np.ndarray:
    """Boolean [T,T]: Anc[i,j] is True iff j is i or one of i's ancestors."""
    parent_row = np.asarray(parent_row)
    T = parent_row.shape[0]
    anc = np.zeros((T, T), dtype=bool)
    for i in range(T):
        k = i
        steps = 0
        while k != -1:
            anc[i, k] = True
            k = int(parent_row[k])
            steps += 1
            if steps > T:
                raise ValueError("parent array has a cycle")
    return anc


def packed_scan(x, dt, A, B, C, D, h0, parent):
    x, dt, A, B, C, D, h0 = (np.asarray(v, np.float64) for v in (x, dt, A, B, C, D, h0))
    batch, T, H, P = x.shape
    G = B.shape[2]
    y = np.zeros_like(x)
    for b in range(batch):
        anc = ancestor_matrix(parent[b])
        for h in range(H):
            g = h // (H // G)
            a = dt[b, :, h] * A[h]
            Lc = anc.astype(np.float64) @ a
            diff = np.where(anc, Lc[:, None] - Lc[None, :], -np.inf)
            decay = np.where(anc, np.exp(diff), 0.0)
            CB = C[b, :, g, :] @ B[b, :, g, :].T
            M = decay * CB * dt[b, :, h][None, :]
            root = np.exp(Lc)[:, None] * (C[b, :, g, :] @ h0[b, h].T)
            y[b, :, h, :] = root + M @ x[b, :, h, :] + D[h] * x[b, :, h, :]
    return y


def packed_commit(x, dt, A, B, h0, parent, path, path_len):
    x, dt, A, B, h0 = (np.asarray(v, np.float64) for v in (x, dt, A, B, h0))
    batch, T, H, P = x.shape
    G = B.shape[2]
    h_new = h0.copy()
    for b in range(batch):
        n = int(path_len[b])
        if n == 0:
            continue
        leaf = int(path[b][n - 1])
        anc = ancestor_matrix(parent[b])
        nodes = np.nonzero(anc[leaf])[0]
        for h in range(H):
            g = h // (H // G)
            a = dt[b, :, h] * A[h]
            Lc = anc.astype(np.float64) @ a
            w = np.exp(Lc[leaf] - Lc[nodes]) * dt[b, nodes, h]
            upd = (x[b, nodes, h, :] * w[:, None]).T @ B[b, nodes, g, :]
            h_new[b, h] = np.exp(Lc[leaf]) * h0[b, h] + upd
    return h_new
