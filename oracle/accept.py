"""Acceptance walk over a verified tree (fp64).

Sources:
  * EAGLE notes, "Well-Calibrated Draft Model": acceptance rate
    min(1, P_target(x) / P_draft(x)); under greedy decoding a draft token is
    accepted when it is the target's most likely token; under sampling it is
    accepted outright when the target gives it at least the draft's
    probability, otherwise with that ratio.
  * aivaro.ru EAGLE-3 answer, section 4 steps 3-4: on rejection the target
    samples its own token from an adjusted distribution; the longest accepted
    prefix of the tree wins.  (Its step-3 test "p_target(x_draft) >=
    p_target(x_target)" contradicts the formula above and is not used.)
  * EAGLE-4 write-up, "Деревья проверки EAGLE-4 и утилита управления":
    verification follows the accepted path, then continues with the target's
    own token once the draft stops matching; rejection sampling keeps the
    longest matching prefix.

Inputs for one sequence: target logits [n+1][V] (row j = the target's
distribution after node j, row 0 after the root), the tree (tokens[n],
parents[n], draft_row[n+1]) and, for sampling, the draft logits [R][V] and
uniforms [2][n+1] (row 0: u_acc indexed by the tested child's node id; row 1:
u_res indexed by the node where the walk stops).

Readings:
  * Greedy: from the root, t = argmax of the current row (ties to the lower
    token id); move to the first child (node order) whose token is t, else
    stop.  The bonus token is t at the stop node.
  * Sampling: at node j, p = softmax(target row j), q = softmax(draft row
    draft_row[j]).  Children are tested in node order: accept child c iff
    u_acc[c] < p(x_c) / q(x_c) (this is "accept with probability
    min(1, p/q)").  Accepting moves to c with a fresh p and q.  Rejecting sets
    p <- max(0, p - q) / sum(max(0, p - q)) and keeps q.  With no child left
    the walk stops at j and the bonus is drawn from the current p by inverse
    CDF: the smallest token i with cumsum(p)_i > u_res[j] * sum(p).  If a
    rejection leaves max(0, p - q) identically zero (only possible when
    p == q, which accepts for every u < 1) the walk stops there and the bonus
    is the target argmax of that node.
  * Sampling without replacement (the pages are silent; the counterpart of the
    rule above for siblings that are distinct tokens, as the top-k children of
    a draft row always are): a rejected child's token can no longer be drawn,
    so after the residual step q <- q with q(x_c) = 0, renormalised.  Accept,
    residual and bonus are otherwise as above; with one child per node the two
    rules coincide.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np

from .common import near_tie, softmax


def _children(parents: np.ndarray, j: int) -> List[int]:
    return [c + 1 for c in range(parents.shape[0]) if int(parents[c]) == j]


def _residual(p: np.ndarray, q: np.ndarray):
    """The adjusted distribution after a rejection: max(0, p - q), normalised.
    None when it is identically zero."""
    resid = np.maximum(0.0, p - q)
    Z = resid.sum()
    return resid / Z if Z > 0.0 else None


def inverse_cdf(weights: np.ndarray, u: float):
    """Smallest index i with cumsum(weights)_i > u * sum(weights).

    Returns (index, near_tie) where near_tie flags a crossing within 1e-6 of
    the total from either neighbouring cumulative sum."""
    c = np.cumsum(np.asarray(weights, dtype=np.float64))
    Z = c[-1]
    thr = u * Z
    i = 0
    while i < c.shape[0] - 1 and not c[i] > thr:
        i += 1
    lo = c[i - 1] if i > 0 else 0.0
    tie = abs(c[i] - thr) <= 1e-6 * Z or abs(thr - lo) <= 1e-6 * Z
    return i, tie


def inverse_cdf_band(weights: np.ndarray, u: float, rel: float = 1e-6) -> List[int]:
    """Every index the inverse CDF returns for some threshold within rel * sum
    of u * sum: the smallest i with cumsum_i > t, for t in that band.  These
    are the results a draw near a cumulative-sum boundary may give once the
    sums are rounded differently."""
    c = np.cumsum(np.asarray(weights, dtype=np.float64))
    Z = c[-1]
    last = c.shape[0] - 1
    lo = min(int(np.searchsorted(c, u * Z - rel * Z, side="right")), last)
    hi = min(int(np.searchsorted(c, u * Z + rel * Z, side="right")), last)
    w = np.diff(np.concatenate([[0.0], c]))
    return [lo] + [i for i in range(lo + 1, hi + 1) if w[i] > 0.0]


def accept_greedy(target: np.ndarray, tokens, parents, max_depth: int) -> Dict:
    target = np.asarray(target, dtype=np.float64)
    tokens = np.asarray(tokens)
    parents = np.asarray(parents)
    j, path = 0, []
    while True:
        t = int(np.argmax(target[j]))   # first maximum = lower token id
        nxt = next((c for c in _children(parents, j) if int(tokens[c - 1]) == t), None)
        if nxt is None:
            bonus = t
            break
        path.append(nxt)
        j = nxt
    assert len(path) <= max_depth
    return {"accepted_len": len(path), "path": path + [-1] * (max_depth - len(path)),
            "bonus": bonus, "stop": j, "near_ties": []}


def _without(q: np.ndarray, x: int):
    """q with token x removed and the rest renormalised.  None when nothing is left."""
    q = q.copy()
    q[x] = 0.0
    S = q.sum()
    return q / S if S > 0.0 else None


def accept_stochastic(target: np.ndarray, draft: np.ndarray, tokens, parents, draft_row,
                      uniforms: np.ndarray, max_depth: int, without_replacement: bool = False,
                      flip=()) -> Dict:
    """`flip`: node ids whose accept test is decided the other way (for checking
    a result downstream of a flagged near-tie); empty for the plain walk."""
    target = np.asarray(target, dtype=np.float64)
    draft = np.asarray(draft, dtype=np.float64)
    tokens = np.asarray(tokens)
    parents = np.asarray(parents)
    u_acc, u_res = uniforms[0], uniforms[1]
    ties: List[dict] = []
    j, path = 0, []
    degenerate = False
    p = softmax(target[0])
    while True:
        kids = _children(parents, j)
        moved = False
        if kids:
            q = softmax(draft[int(draft_row[j])])
            for c in kids:
                x = int(tokens[c - 1])
                ratio = p[x] / q[x]
                u = float(u_acc[c])
                if near_tie(u, ratio):
                    ties.append({"kind": "accept", "node": c, "u": u, "ratio": ratio})
                if (u < ratio) != (c in flip):
                    path.append(c)
                    j = c
                    p = softmax(target[c])
                    moved = True
                    break
                p_new = _residual(p, q)
                if p_new is None:
                    # p == q leaves nothing to resample from; with u < 1 this is
                    # unreachable (p == q accepts).  Fall back to the target's argmax.
                    ties.append({"kind": "degenerate", "node": c})
                    degenerate = True
                    break
                p = p_new
                if without_replacement:
                    q = _without(q, x)
                    if q is None:
                        ties.append({"kind": "degenerate", "node": c})
                        degenerate = True
                        break
        if not moved:
            break
    if degenerate:
        bonus = int(np.argmax(target[j]))
    else:
        bonus, tie = inverse_cdf(p, float(u_res[j]))
        if tie:
            ties.append({"kind": "bonus", "node": j, "alternatives": inverse_cdf_band(p, float(u_res[j]))})
    assert len(path) <= max_depth
    return {"accepted_len": len(path), "path": path + [-1] * (max_depth - len(path)),
            "bonus": int(bonus), "stop": j, "near_ties": ties}
