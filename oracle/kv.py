"""KV-cache compaction after acceptance (integer and copy work; no arithmetic).

Source: EAGLE-4 write-up ("Технический анализ EAGLE-4"), section "Деревья
проверки EAGLE-4 и утилита управления": after verification the harness keeps
the accepted continuation, frees the rejected KV-cache entries and starts the
next round.

Reading taken: the verification pass computed keys and values for every tree
node (k_tree / v_tree).  Keeping the accepted continuation appends the
accepted path's entries to the sequence's prefix cache in path order: the i-th
accepted node (depth i + 1) goes to position prefix_len + i, which is its
position id prefix_len - 1 + depth.  Entries of rejected nodes are not copied.
The bonus token has no key or value yet (the next round computes them).  A
position at or past the cache length Lmax is not written, and the new prefix
length is min(prefix_len + accepted, Lmax).
"""
from __future__ import annotations

import numpy as np


def compact_kv(k_cache, v_cache, prefix_len, k_tree, v_tree, path, accepted_len):
    """k_cache / v_cache [B][Hkv][Lmax][D], k_tree / v_tree [B][n][Hkv][D] (any
    dtype, copied as is), prefix_len [B], path [B][depth] (node ids 1..n, -1
    padded), accepted_len [B] -> (new k_cache, new v_cache, new prefix_len)."""
    k_out, v_out = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    B, Hkv, Lmax = k_out.shape[0], k_out.shape[1], k_out.shape[2]
    n = k_tree.shape[1]
    new_len = np.zeros(B, dtype=np.int64)
    for b in range(B):
        L = min(max(int(prefix_len[b]), 0), Lmax)
        a = int(accepted_len[b])
        written = 0
        for i in range(a):
            node = int(path[b][i])
            pos = L + i
            if pos >= Lmax or not (1 <= node <= n):
                break
            for h in range(Hkv):
                k_out[b, h, pos] = k_tree[b, node - 1, h]
                v_out[b, h, pos] = v_tree[b, node - 1, h]
            written += 1
        new_len[b] = L + written
    return k_out, v_out, new_len
