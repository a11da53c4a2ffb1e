"""Greedy (temperature 0) verification of a draft tree -- TEST INFRASTRUCTURE ONLY.

The rule follows the tree speculative decoding that STree builds on ("STree:
Speculative Tree Decoding for Hybrid State Space Models", scime.ai summary,
"Key results" at temperature 0 and "Builds on": SpecInfer, speculative
sampling): the target model's prediction after a node is its most probable
next token; starting at the root, a child is accepted when its draft token
equals the prediction after its parent, and the walk continues from it.  The
accepted path is the root-first chain of accepted nodes; the bonus token is the
prediction after the last accepted node.

Readings (the pages print no algorithm): the prediction is the first index of
the largest logit (ties go to the smaller token id); among children whose tokens
match, the smallest node index is taken; the path stops at `maxlen` nodes.

The argmax is numpy's (a library primitive); the walk is written out.
"""
from __future__ import annotations

import numpy as np


def oracle_accept_greedy(logits: np.ndarray, tokens: np.ndarray, parent: np.ndarray, maxlen: int):
    """logits [b, T, V] (any real dtype, compared exactly), tokens [b, T] int,
    parent [b, T] int (a valid packed tree per sequence).  Returns
    (pred [b, T], path [b, maxlen] with -1 past the end, path_len [b], bonus [b])."""
    logits = np.asarray(logits, dtype=np.float64)
    tokens = np.asarray(tokens)
    parent = np.asarray(parent)
    b, T, _ = logits.shape
    pred = np.argmax(logits, axis=-1).astype(np.int64)
    path = np.full((b, maxlen), -1, np.int64)
    plen = np.zeros(b, np.int64)
    bonus = np.zeros(b, np.int64)
    for s in range(b):
        cur, nodes = 0, [0]
        while len(nodes) < maxlen:
            nxt = -1
            for c in range(T):                       # children in increasing index order
                if parent[s, c] == cur and tokens[s, c] == pred[s, cur]:
                    nxt = c
                    break
            if nxt < 0:
                break
            nodes.append(nxt)
            cur = nxt
        path[s, :len(nodes)] = nodes
        plen[s] = len(nodes)
        bonus[s] = pred[s, cur]
    return pred, path, plen, bonus


def _softmax(z: np.ndarray) -> np.ndarray:
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


def oracle_accept_sampling(target_logits, draft_logits, tokens, parent, temperature: float, u_accept, u_bonus,
                           maxlen: int):
    """Stochastic verification of a draft tree by multi-step speculative sampling
    (the sampling STree uses at temperature > 0: "Builds on" SpecInfer and
    speculative sampling; the residual rule as the TreeSpark summary describes it).

    At the current node u with target distribution p = softmax(target_logits[u] / T)
    and draft distribution q = softmax(draft_logits[u] / T) (from which u's children's
    tokens were drawn), the children are tried in increasing index order: child c
    with token t is accepted when u_accept[c] * q[t] < p[t] (i.e. with probability
    min(1, p[t] / q[t])), and the walk moves on to c; after a rejection p becomes the
    residual max(p - q, 0), renormalised.  When no child is accepted (or u is a leaf,
    or the path holds maxlen nodes) the bonus token is drawn from the current p by
    inverse CDF with u_bonus.  Random numbers are inputs: u_accept [b, T] (one per
    node, used when that node is tested) and u_bonus [b], all in [0, 1).

    Returns (path [b, maxlen] with -1 past the end, path_len [b], bonus [b])."""
    tl = np.asarray(target_logits, dtype=np.float64)
    dl = np.asarray(draft_logits, dtype=np.float64)
    tokens = np.asarray(tokens)
    parent = np.asarray(parent)
    ua = np.asarray(u_accept, dtype=np.float64)
    ub = np.asarray(u_bonus, dtype=np.float64)
    b, T, V = tl.shape
    path = np.full((b, maxlen), -1, np.int64)
    plen = np.zeros(b, np.int64)
    bonus = np.zeros(b, np.int64)
    for s in range(b):
        cur, nodes = 0, [0]
        p = _softmax(tl[s, 0] / temperature)
        while True:
            q = _softmax(dl[s, cur] / temperature)
            nxt = -1
            if len(nodes) < maxlen:
                for c in range(T):
                    if parent[s, c] != cur:
                        continue
                    t = tokens[s, c]
                    if ua[s, c] * q[t] < p[t]:
                        nxt = c
                        break
                    r = np.maximum(p - q, 0.0)
                    if r.sum() > 0.0:
                        p = r / r.sum()
            if nxt < 0:
                break
            nodes.append(nxt)
            cur = nxt
            p = _softmax(tl[s, cur] / temperature)
        cdf = np.cumsum(p)
        bonus[s] = int(min(np.searchsorted(cdf, ub[s] * cdf[-1], side="right"), V - 1))
        path[s, :len(nodes)] = nodes
        plen[s] = len(nodes)
    return path, plen, bonus
