"""EAGLE-1 static draft tree (fp64).

Source: "EAGLE" notes (s1mplewind), "1. EAGLE pipeline / Draft Model": EAGLE
drafts on one fixed tree, the same for every step, whose shape its appendix
describes by two rules: a node's children are its top-k tokens, and likelier
branches are made deeper and wider, so that within a level the nodes on the
left are the likelier ones and carry the deeper subtrees.  (EAGLE-2 replaces
it with the dynamic tree of tree.py.)

Readings the pages leave open, taken here:
  * The template is given before drafting as, for each node i = 1..n, its
    parent p_i (0 = the root, else a node before i) and its sibling rank r_i
    (0 = the parent's likeliest child).  Siblings have distinct ranks.
  * Node i's token is the rank-r_i token of its parent's draft row: the
    row's tokens ordered by logit, ties to the lower token id.
  * Draft rows: row 0 is the root's; every node that has a child owns a row,
    numbered 1, 2, ... in node order, so R = 1 + (number of such nodes).
  * log V = log V(parent) + log-confidence, as in the dynamic tree; it is
    reported, not used to select anything.  depth = depth(parent) + 1.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from .common import logsumexp


def template_rows(parents) -> np.ndarray:
    """draft_row[0..n]: 0 for the root, the row of each node with a child, -1 otherwise."""
    parents = np.asarray(parents, dtype=np.int64)
    n = parents.shape[0]
    has_child = np.zeros(n + 1, dtype=bool)
    for p in parents:
        has_child[int(p)] = True
    rows = np.full(n + 1, -1, dtype=np.int64)
    rows[0] = 0
    nxt = 1
    for i in range(1, n + 1):
        if has_child[i]:
            rows[i] = nxt
            nxt += 1
    return rows


def build_static_tree(logits: np.ndarray, parents, ranks) -> Dict:
    """One sequence's static tree from its draft rows [R][V] (fp64) and the template."""
    logits = np.asarray(logits, dtype=np.float64)
    parents = np.asarray(parents, dtype=np.int64)
    ranks = np.asarray(ranks, dtype=np.int64)
    n = parents.shape[0]
    rows = template_rows(parents)
    R = int(rows.max()) + 1
    assert logits.shape[0] == R, (logits.shape, R)
    for i in range(n):
        assert 0 <= parents[i] <= i, "a parent precedes its child"
    row_lse = np.array([logsumexp(logits[r]) for r in range(R)])

    tokens = np.zeros(n, dtype=np.int64)
    depth = np.zeros(n, dtype=np.int64)
    logV = np.zeros(n, dtype=np.float64)
    for i in range(n):
        p = int(parents[i])
        row = int(rows[p])
        order = np.lexsort((np.arange(logits.shape[1]), -logits[row]))   # by logit desc, then token id
        tok = int(order[int(ranks[i])])
        tokens[i] = tok
        lp = logits[row, tok] - row_lse[row]
        depth[i] = 1 if p == 0 else depth[p - 1] + 1
        logV[i] = lp if p == 0 else logV[p - 1] + lp
    return {"tokens": tokens, "parents": parents.copy(), "depth": depth, "logV": logV,
            "gid": np.arange(n, dtype=np.int64), "draft_row": rows, "row_lse": row_lse, "n": n}
