"""Gated delta rule over a packed draft tree -- TEST INFRASTRUCTURE ONLY.

The linear-attention layers of the hybrid models carry a fixed-size state updated
by the gated delta rule ("TreeWY" abstract: Gated DeltaNet layers, every draft
node's output from one triangular solve, only the accepted state rebuilt on
commit from a small pseudo-value matrix; "Bole" abstract: a tree-structured
closed form of the linear-attention recurrence).  Per sequence and value head,
with state S [d_v, d_k] and node i with parent p(i):

    S_i = alpha_i S_p(i) (I - a_i k_i k_i^T) + beta_i v_i k_i^T,   S_p(root) = S0
    o_i = S_i q_i

and the commit of an accepted path is its last node's state.  alpha (the gate,
in (0, 1]), beta (the write strength) and a (the erase strength) are taken as
given, after their activations; q and k as given (any normalisation happens
before this op).  The gated delta rule ties the two strengths, a = beta (the
default, ``erase=None``); given separately they are the decoupled erase and write
of "Gated DeltaNet-2" (related-papers entry on the TreeWY page), and a = 0 is
gated linear attention, the plain linear-attention recurrence of the "Bole"
abstract (S_i = alpha_i S_p(i) + beta_i v_i k_i^T).
Value head h reads query/key head h // (Hv / Hk).

``oracle_gdn_tree`` / ``oracle_gdn_commit`` are the plain definition: walk each
node's root path and apply the recurrence step by step, in fp64.
``packed_gdn`` is a second formulation used only to cross-check the walk: with
gamma_i the product of alpha over the root path of i and w_j = S0 k_j, the
pseudo-values solve the ancestor-triangular system

    u_j = beta_j v_j - a_j (gamma_j w_j + sum_{l ancestor of j} (gamma_j / gamma_l) (k_l . k_j) u_l)

and o_i = gamma_i S0 q_i + sum_{j in anc(i)} (gamma_i / gamma_j) (k_j . q_i) u_j,
S_new = gamma_leaf S0 + sum_{j on path} (gamma_leaf / gamma_j) u_j k_j^T
(it follows from S_t = alpha_t S_{t-1} + u_t k_t^T with u_t = beta_t v_t -
a_t alpha_t S_{t-1} k_t).
"""
from __future__ import annotations

import numpy as np


def _path(parent_row, i):
    out = []
    j = int(i)
    while j >= 0:
        out.append(j)
        j = int(parent_row[j])
    return out[::-1]


def _step(S, kj, vj, a, be, er):
    """One step of the rule: alpha S (I - er k k^T) + beta v k^T, with the erase
    applied as the rank-1 product S - er (S k) k^T (the same matrix product,
    without forming the d_k x d_k factor)."""
    return a * (S - er * np.outer(S @ kj, kj)) + be * np.outer(vj, kj)


def _f64(*arrays):
    return [np.asarray(a, np.float64) for a in arrays]


def oracle_gdn_tree(q, k, v, alpha, beta, S0, parent, erase=None):
    """q, k [b, T, Hk, dk]; v [b, T, Hv, dv]; alpha, beta, erase [b, T, Hv] (erase
    None: the delta rule, erase = beta); S0 [b, Hv, dv, dk]; parent [b, T].
    Returns o [b, T, Hv, dv] (fp64)."""
    q, k, v, alpha, beta, S0 = _f64(q, k, v, alpha, beta, S0)
    erase = beta if erase is None else np.asarray(erase, np.float64)
    parent = np.asarray(parent)
    b, T, Hk, dk = k.shape
    Hv, dv = v.shape[2], v.shape[3]
    grp = Hv // Hk
    o = np.zeros((b, T, Hv, dv))
    for s in range(b):
        for i in range(T):
            path = _path(parent[s], i)
            for h in range(Hv):
                g = h // grp
                S = S0[s, h].copy()
                for j in path:
                    S = _step(S, k[s, j, g], v[s, j, h], alpha[s, j, h], beta[s, j, h], erase[s, j, h])
                o[s, i, h] = S @ q[s, i, g]
    return o


def oracle_gdn_commit(k, v, alpha, beta, S0, parent, path, path_len, erase=None):
    """The state after each sequence's accepted path (path [b, maxlen], path_len [b];
    an empty path keeps S0).  The path must be a root-first chain of the tree.
    Returns S_new [b, Hv, dv, dk] (fp64)."""
    k, v, alpha, beta, S0 = _f64(k, v, alpha, beta, S0)
    erase = beta if erase is None else np.asarray(erase, np.float64)
    parent = np.asarray(parent)
    b, T, Hk, dk = k.shape
    Hv = v.shape[2]
    grp = Hv // Hk
    out = S0.copy()
    for s in range(b):
        n = int(path_len[s])
        nodes = [int(x) for x in path[s, :n]]
        if n:
            assert nodes == _path(parent[s], nodes[-1]), "accepted path is not a root-first chain"
        for h in range(Hv):
            g = h // grp
            S = S0[s, h].copy()
            for j in nodes:
                S = _step(S, k[s, j, g], v[s, j, h], alpha[s, j, h], beta[s, j, h], erase[s, j, h])
            out[s, h] = S
    return out


def packed_gdn(q, k, v, alpha, beta, S0, parent, path=None, path_len=None, erase=None):
    """Cross-check formulation (ancestor-triangular solve for the pseudo-values).
    Returns o [b, T, Hv, dv], and S_new [b, Hv, dv, dk] when a path is given."""
    q, k, v, alpha, beta, S0 = _f64(q, k, v, alpha, beta, S0)
    erase = beta if erase is None else np.asarray(erase, np.float64)
    parent = np.asarray(parent)
    b, T, Hk, dk = k.shape
    Hv, dv = v.shape[2], v.shape[3]
    grp = Hv // Hk
    o = np.zeros((b, T, Hv, dv))
    S_new = S0.copy() if path is not None else None
    for s in range(b):
        anc = [_path(parent[s], i) for i in range(T)]
        for h in range(Hv):
            g = h // grp
            lg = np.array([np.sum(np.log(alpha[s, anc[i], h])) for i in range(T)])   # log gamma
            K, Q = k[s, :, g], q[s, :, g]
            W = K @ S0[s, h].T                              # w_j = S0 k_j, [T, dv]
            U = np.zeros((T, dv))
            for j in range(T):                              # parents precede children
                acc = np.exp(lg[j]) * W[j]
                for l in anc[j][:-1]:
                    acc += np.exp(lg[j] - lg[l]) * (K[l] @ K[j]) * U[l]
                U[j] = beta[s, j, h] * v[s, j, h] - erase[s, j, h] * acc
            for i in range(T):
                oi = np.exp(lg[i]) * (S0[s, h] @ Q[i])
                for j in anc[i]:
                    oi += np.exp(lg[i] - lg[j]) * (K[j] @ Q[i]) * U[j]
                o[s, i, h] = oi
            if path is not None and int(path_len[s]) > 0:
                nodes = [int(x) for x in path[s, :int(path_len[s])]]
                leaf = nodes[-1]
                S = np.exp(lg[leaf]) * S0[s, h]
                for j in nodes:
                    S += np.exp(lg[leaf] - lg[j]) * np.outer(U[j], K[j])
                S_new[s, h] = S
    return o, S_new
