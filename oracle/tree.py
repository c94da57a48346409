"""EAGLE-2 dynamic draft tree, brute force (fp64).

Source: "EAGLE" notes (s1mplewind), EAGLE-2 sections:
  * "Well-Calibrated Draft Model": the draft confidence of token x is
    c(x) = exp(logit_x) / sum_i exp(logit_i).
  * "Expansion of tree": a token's value is its global acceptance
    V_i = product of the confidences on the path root -> i (rejecting a token
    cuts its whole subtree); each level keeps the top-k tokens by V and
    expands each kept token's top-k children.
  * "Reranking Nodes": after expansion, keep the m tokens with the largest V
    over all candidates.

Readings the pages leave open, taken here:
  * m does not count the root; the root is the last accepted token.
  * Draft rows without a draft model: row 0 is the root's distribution and the
    node in frontier slot s of level l (1 <= l <= depth-1) owns row
    1 + (l-1)*k + s.  The frontier slot is the node's rank in that level's
    selection, ordered by (-logV, candidate id).  R = 1 + (depth-1)*k rows.
  * Candidate id (gid): level 1 uses gid = r (child rank r of the root);
    level l >= 2 uses gid = k + (l-2)*k*k + s*k + r, with s the parent's
    frontier slot and r the child's rank in its row.  Every ordering is by
    (-logV, gid): ties go to the lower id, so a parent always precedes its child.
  * V is ranked in log space: logV = sum of log-confidences along the path,
    i.e. log of the product.  A child's logV is at most its parent's, so the
    kept set is closed under "parent of".
  * The top-k children of a row are its k largest raw logits, ties to the
    lower token id (the same order as by log-confidence).
  * Output nodes are numbered 1..n in ascending gid (parents before children,
    siblings in rank order); parent 0 is the root.
  * A logit of -inf has confidence 0 and is no child: a row with fewer than k
    finite logits fills its remaining children with token -1 and log V = -inf
    (a row of -inf marks a frontier node the caller chose not to draft from).
  * With per-level widths (the cost-aware harness's widening, see
    oracle.sizing): instead of the best m over all levels, the tree keeps the
    w_l best candidates of each level l (by the same ordering), for the levels
    given.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np

from .common import logsumexp, near_tie


def _row_topk(row: np.ndarray, k: int) -> np.ndarray:
    """Token ids of the k largest values, ties to the lower id (library sort);
    -1 in place of a logit of -inf."""
    order = np.lexsort((np.arange(row.shape[0]), -row))[:k]
    return np.where(np.isneginf(row[order]), -1, order)


def _sort_key(c):
    return (-c["logV"], c["gid"])


def _flag_adjacent(sorted_cands, upto: int, kind: str, level: int, out: list):
    """Record near-ties between neighbours of a selection (positions < upto+1).

    Each record names the decision: (kind, level) and the two candidate ids in
    the order this run ranked them, so that the same selection can be re-run
    with the pair the other way round (see `_apply_flips`)."""
    for i in range(min(upto, len(sorted_cands) - 1)):
        a, b = sorted_cands[i], sorted_cands[i + 1]
        if a["parent"] == b["parent"]:
            # siblings: logV differ only through their raw logits, whose order
            # (ties to the lower rank, hence lower gid) no rounding can change
            continue
        if near_tie(a["logV"], b["logV"]):
            out.append({"kind": kind, "level": level, "gids": (a["gid"], b["gid"]),
                        "logV": (a["logV"], b["logV"])})


def _apply_flips(ranked, kind: str, level: int, flip) -> list:
    """Resolve flagged near-ties the other way: for every record of `flip` that
    names this selection (kind, level) and whose two candidates are neighbours
    here in the recorded order, swap them.  A ranking within the near-tie band
    is decided by rounding, so either order is a correct result; the tests use
    this to tell a difference downstream of a flagged decision (allowed) from
    any other difference (a failure)."""
    for f in flip:
        if f["kind"] != kind or f["level"] != level:
            continue
        a, b = f["gids"]
        for i in range(len(ranked) - 1):
            if ranked[i]["gid"] == a and ranked[i + 1]["gid"] == b:
                if ranked[i + 1]["parent"] != a:  # a child never ranks above its parent
                    ranked[i], ranked[i + 1] = ranked[i + 1], ranked[i]
                break
    return ranked


def build_tree(logits: np.ndarray, depth: int, k: int, m: int, flip=(), widths=None) -> Dict:
    """Build one sequence's tree from its R = 1 + (depth-1)*k draft rows (fp64).

    `flip`: near-tie records (as returned in "near_ties") to resolve the other
    way; empty for the plain build.  `widths`: per-level widths w_1.. (at most
    depth of them) to keep the w_l best of each level instead of the best m."""
    logits = np.asarray(logits, dtype=np.float64)
    R, V = logits.shape
    assert depth >= 1 and 1 <= k <= V and m >= 1
    assert R == 1 + (depth - 1) * k, (R, depth, k)

    row_lse = np.array([logsumexp(logits[r]) for r in range(R)])
    topk = [_row_topk(logits[r], k) for r in range(R)]

    near_ties: List[dict] = []
    all_cands: List[dict] = []

    def make(row, r, gid, level, parent):
        tok = int(topk[row][r])
        lp = logits[row, tok] - row_lse[row] if tok >= 0 else -np.inf  # log confidence, <= 0
        base = 0.0 if parent is None else parent["logV"]
        return {"gid": gid, "level": level, "token": tok, "logit": logits[row, tok],
                "lp": lp, "logV": base + lp, "parent": None if parent is None else parent["gid"],
                "pnode": parent, "slot": -1, "row": -1}

    # level 1: the root's k children
    level_cands = [make(0, r, r, 1, None) for r in range(k)]
    all_cands += level_cands
    frontiers: List[dict] = []    # per expanded level: the k tokens by slot and their parents' slots
    gains: List[float] = []       # per level: sum of V over its k best candidates
    level_logv: List[np.ndarray] = []  # per level: log V of its k best candidates, in rank order
    for level in range(2, depth + 1):
        ranked = _apply_flips(sorted(level_cands, key=_sort_key), "frontier", level - 1, flip)
        _flag_adjacent(ranked, k, "frontier", level - 1, near_ties)
        frontier = ranked[:k]
        gains.append(float(sum(np.exp(c["logV"]) for c in frontier)))
        level_logv.append(np.array([c["logV"] for c in frontier]))
        frontiers.append({"tokens": np.array([c["token"] for c in frontier], dtype=np.int64),
                          "parent_slot": np.array([-1 if c["pnode"] is None else c["pnode"]["slot"]
                                                   for c in frontier], dtype=np.int64)})
        nxt = []
        off = k + (level - 2) * k * k
        for s, parent in enumerate(frontier):
            parent["slot"] = s
            parent["row"] = 1 + (level - 2) * k + s
            for r in range(k):
                nxt.append(make(parent["row"], r, off + s * k + r, level, parent))
        level_cands = nxt
        all_cands += level_cands

    last = sorted(level_cands, key=_sort_key)[:k]
    gains.append(float(sum(np.exp(c["logV"]) for c in last)))
    level_logv.append(np.array([c["logV"] for c in last]))
    P = len(all_cands)
    assert P == k + (depth - 1) * k * k
    if widths is None:
        n = min(m, P)
        ranked = _apply_flips(sorted(all_cands, key=_sort_key), "rerank", 0, flip)
        _flag_adjacent(ranked[n - 1:], 1, "rerank", 0, near_ties)
        kept = sorted(ranked[:n], key=lambda c: c["gid"])
    else:
        assert 1 <= len(widths) <= depth
        chosen = []
        for level, w in enumerate(widths, start=1):
            ranked = _apply_flips(sorted([c for c in all_cands if c["level"] == level], key=_sort_key), "width",
                                  level, flip)
            assert 0 <= w <= len(ranked)
            if 0 < w < len(ranked):
                _flag_adjacent(ranked[w - 1:], 1, "width", level, near_ties)
            chosen += ranked[:w]
        kept = sorted(chosen, key=lambda c: c["gid"])
        n = len(kept)
    node_of = {c["gid"]: i + 1 for i, c in enumerate(kept)}

    tokens = np.array([c["token"] for c in kept], dtype=np.int64)
    parents = np.array([0 if c["parent"] is None else node_of[c["parent"]] for c in kept],
                       dtype=np.int64)
    depth_arr = np.array([c["level"] for c in kept], dtype=np.int64)
    logV = np.array([c["logV"] for c in kept], dtype=np.float64)
    gid = np.array([c["gid"] for c in kept], dtype=np.int64)
    draft_row = np.full(n + 1, -1, dtype=np.int64)
    draft_row[0] = 0
    for i, c in enumerate(kept):
        draft_row[i + 1] = c["row"]
    return {"tokens": tokens, "parents": parents, "depth": depth_arr, "logV": logV,
            "gid": gid, "draft_row": draft_row, "row_lse": row_lse, "n": n, "P": P,
            "frontiers": frontiers, "gains": np.array(gains), "level_logv": level_logv, "near_ties": near_ties}


def build_trees(logits_b: np.ndarray, depth: int, k: int, m: int) -> List[Dict]:
    """One tree per sequence of a [B][R][V] fp64 batch."""
    return [build_tree(logits_b[b], depth, k, m) for b in range(logits_b.shape[0])]
