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
