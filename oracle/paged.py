"""Paged prefix cache (plain numpy): the cache of each sequence as a list of
fixed-size pages in a shared pool, named by a block table.

A paged cache is a layout of the prefix cache the mask section of the EAGLE-4
write-up ("Деревья проверки EAGLE-4 и утилита управления") attends to and
whose rejected entries its harness frees; nothing in the arithmetic changes.
Readings taken here:
  * pools [num_pages][Hkv][page_size][D]; sequence b's key at position p sits
    at offset p % page_size of page block_table[b][p // page_size];
  * attention over a paged cache is tree attention over the gathered cache;
  * compaction writes the i-th accepted node at position prefix_len + i like
    compact_kv, and stops at a position whose page id lies outside the pool
    (a page not allocated yet) or beyond the table's capacity.
"""
from __future__ import annotations

import numpy as np


def gather_pages(pages: np.ndarray, table, L: int) -> np.ndarray:
    """The first L positions of one sequence as a dense [Hkv][L][D] array."""
    pages = np.asarray(pages)
    num_pages, Hkv, ps, D = pages.shape
    out = np.zeros((Hkv, L, D), dtype=pages.dtype)
    for p in range(L):
        page = int(table[p // ps])
        assert 0 <= page < num_pages, (p, page)
        out[:, p] = pages[page, :, p % ps]
    return out


def compact_kv_paged(k_pages, v_pages, table, prefix_len, k_tree, v_tree, path, accepted_len):
    """compact_kv for a paged cache -> (k_pages', v_pages', new_len).

    table [B][pages_per_seq]; k_tree / v_tree [B][n][Hkv][D]; path [B][depth]."""
    k_pages, v_pages = np.array(k_pages, copy=True), np.array(v_pages, copy=True)
    table = np.asarray(table)
    num_pages, _, ps, _ = k_pages.shape
    B, n = k_tree.shape[0], k_tree.shape[1]
    cap = table.shape[1] * ps
    new_len = np.zeros(B, dtype=np.int64)
    for b in range(B):
        L = min(max(int(prefix_len[b]), 0), cap)
        a = min(max(int(accepted_len[b]), 0), path.shape[1])
        cnt = 0
        while cnt < a:
            node, pos = int(path[b][cnt]), L + cnt
            if not (1 <= node <= n) or pos >= cap:
                break
            page = int(table[b][pos // ps])
            if not (0 <= page < num_pages):
                break
            k_pages[page, :, pos % ps] = k_tree[b, node - 1]
            v_pages[page, :, pos % ps] = v_tree[b, node - 1]
            cnt += 1
        new_len[b] = L + cnt
    return k_pages, v_pages, new_len
