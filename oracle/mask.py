"""Tree attention mask (fp64 oracle side; integer work).

Source: "Технический анализ EAGLE-4", section "Деревья проверки EAGLE-4 и
утилита управления": a custom attention mask lets every tree token attend to
the shared prefix, its ancestors and itself, and hides siblings and other
branches.  The EAGLE notes (EAGLE-3 "Training") describe the same structure:
a token sees only the keys on its own path.

Nodes are 1..n; parents[i] is the parent of node i+1 (0 = the root, which is
the last prefix entry).  The mask row of node i+1 has bit j set iff node j+1
is node i+1 itself or one of its ancestors.
"""
from __future__ import annotations

import numpy as np


def ancestor_mask(parents: np.ndarray) -> np.ndarray:
    """Dense bool [n][n]: walk each node's parent chain explicitly."""
    parents = np.asarray(parents)
    n = parents.shape[0]
    mask = np.zeros((n, n), dtype=bool)
    for i in range(n):
        node = i + 1
        while node != 0:
            mask[i, node - 1] = True
            node = int(parents[node - 1])
    return mask


def pack_mask(mask: np.ndarray, words: int = 2) -> np.ndarray:
    """Dense bool [n][n] -> uint64 [n][words]: bit (j % 64) of word j // 64."""
    n = mask.shape[0]
    out = np.zeros((n, words), dtype=np.uint64)
    for i in range(n):
        for j in range(n):
            if mask[i, j]:
                out[i, j // 64] |= np.uint64(1) << np.uint64(j % 64)
    return out


def positions(depth: np.ndarray, prefix_len: int) -> np.ndarray:
    """Position id of each node: the root sits at prefix_len - 1, a node at depth
    d sits d positions after it."""
    return (prefix_len - 1 + np.asarray(depth)).astype(np.int64)
