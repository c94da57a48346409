"""Tree-masked attention with an explicit dense mask (fp64).

Source: "Технический анализ EAGLE-4", section "Деревья проверки EAGLE-4 и
утилита управления" (the mask: shared prefix, ancestors, self) and the
"Tree Attention" verification of the EAGLE notes ("3.Verify"); the sliding
window of the drafter's attention is from the "Архитектура EAGLE-4" section.

For query node i (position pos_i = L - 1 + depth_i) and query head h, the
keys are the prefix entries 0..L-1 of KV head h // (Hq/Hkv) followed by the n
tree entries; the scores q.k * scale over the visible keys go through a
softmax and weight the values.  Visible: prefix key p iff no window or
p >= pos_i - W + 1; tree key j iff node j+1 is node i+1 or an ancestor (and,
with a window, pos_j >= pos_i - W + 1).  scale defaults to 1/sqrt(D).
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Tuple

import numpy as np

from .mask import ancestor_mask


def _visible(L: int, parents, depth, window: int) -> np.ndarray:
    anc = ancestor_mask(parents)
    n = anc.shape[0]
    pos = L - 1 + np.asarray(depth, dtype=np.int64)
    vis = np.zeros((n, L + n), dtype=bool)
    for i in range(n):
        lo = 0 if window <= 0 else max(0, int(pos[i]) - window + 1)
        vis[i, lo:L] = True
        for j in range(n):
            if anc[i, j] and (window <= 0 or pos[j] >= pos[i] - window + 1):
                vis[i, L + j] = True
    return vis


def _softmax_rows(s: np.ndarray) -> np.ndarray:
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def tree_attention(q, k_cache, v_cache, L: int, k_tree, v_tree, parents, depth,
                   window: int = 0, scale: Optional[float] = None, return_weights: bool = False):
    """One sequence.  q [n][Hq][D]; k_cache, v_cache [Hkv][>=L][D];
    k_tree, v_tree [n][Hkv][D]; all fp64.  Returns out [n][Hq][D] fp64, and with
    return_weights also the softmax weights [n][Hq][L+n] over (prefix keys,
    tree keys) that produced it."""
    q = np.asarray(q, dtype=np.float64)
    n, Hq, D = q.shape
    Hkv = k_cache.shape[0]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    vis = _visible(L, parents, depth, window)
    out = np.empty((n, Hq, D), dtype=np.float64)
    weights = np.empty((n, Hq, L + n), dtype=np.float64) if return_weights else None
    for h in range(Hq):
        g = h // G
        keys = np.concatenate([k_cache[g, :L], k_tree[:, g]], axis=0).astype(np.float64)
        vals = np.concatenate([v_cache[g, :L], v_tree[:, g]], axis=0).astype(np.float64)
        s = (q[:, h] @ keys.T) * scale
        s = np.where(vis, s, -np.inf)
        p = _softmax_rows(s)
        out[:, h] = p @ vals
        if return_weights:
            weights[:, h] = p
    return (out, weights) if return_weights else out


def tree_attention_rows(q, k_cache, v_cache, L: int, k_tree, v_tree, parents, depth,
                        rows: Iterable[Tuple[int, int]], window: int = 0,
                        scale: Optional[float] = None, return_weights: bool = False):
    """The same, for selected (node index i, head h) pairs only -> [len(rows)][D]
    (and with return_weights the weights [len(rows)][L+n])."""
    n, Hq, D = q.shape
    Hkv = k_cache.shape[0]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    vis = _visible(L, parents, depth, window)
    res, ws = [], []
    for i, h in rows:
        g = h // G
        keys = np.concatenate([k_cache[g, :L], k_tree[:, g]], axis=0).astype(np.float64)
        vals = np.concatenate([v_cache[g, :L], v_tree[:, g]], axis=0).astype(np.float64)
        s = (keys @ np.asarray(q[i, h], dtype=np.float64)) * scale
        s = np.where(vis[i], s, -np.inf)
        p = _softmax_rows(s[None])[0]
        res.append(p @ vals)
        ws.append(p)
    return (np.array(res), np.array(ws)) if return_weights else np.array(res)
