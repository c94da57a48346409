"""Pins for the oracle's KV-cache compaction after acceptance (no GPU).

The compaction keeps the accepted path's keys and values (EAGLE-4 write-up,
section "Деревья проверки EAGLE-4 и утилита управления": the harness keeps the
accepted continuation and frees the rejected KV entries).  It is tied to a
hand-worked case, to the closed forms "nothing accepted" and "cache full", and
to attention itself: after compacting the root path of a node x, plain causal
attention (torch SDPA) of x's query over the compacted cache equals the tree
attention of x over the prefix and the tree, because x's tree context is exactly
the prefix plus its root path.
"""
import numpy as np
import torch

import oracle


def _arrays(B, Hkv, Lmax, n, D, seed=0):
    rng = np.random.default_rng(seed)
    kc = rng.normal(size=(B, Hkv, Lmax, D))
    vc = rng.normal(size=(B, Hkv, Lmax, D))
    kt = rng.normal(size=(B, n, Hkv, D))
    vt = rng.normal(size=(B, n, Hkv, D))
    return kc, vc, kt, vt


def test_hand_worked_case():
    kc, vc, kt, vt = _arrays(1, 2, 8, 4, 3)
    path = np.array([[2, 4, -1]])
    k2, v2, nl = oracle.compact_kv(kc, vc, np.array([3]), kt, vt, path, np.array([2]))
    assert nl.tolist() == [5]
    np.testing.assert_array_equal(k2[0, :, 3], kt[0, 1])   # node 2 -> position 3
    np.testing.assert_array_equal(k2[0, :, 4], kt[0, 3])   # node 4 -> position 4
    np.testing.assert_array_equal(v2[0, :, 3], vt[0, 1])
    np.testing.assert_array_equal(v2[0, :, 4], vt[0, 3])
    untouched = [p for p in range(8) if p not in (3, 4)]
    np.testing.assert_array_equal(k2[0][:, untouched], kc[0][:, untouched])
    np.testing.assert_array_equal(v2[0][:, untouched], vc[0][:, untouched])


def test_nothing_accepted_changes_nothing():
    kc, vc, kt, vt = _arrays(2, 2, 16, 5, 4, seed=1)
    k2, v2, nl = oracle.compact_kv(kc, vc, np.array([7, 16]), kt, vt, np.full((2, 3), -1), np.array([0, 0]))
    np.testing.assert_array_equal(k2, kc)
    np.testing.assert_array_equal(v2, vc)
    assert nl.tolist() == [7, 16]


def test_full_cache_keeps_what_fits():
    kc, vc, kt, vt = _arrays(1, 1, 10, 6, 2, seed=2)
    k2, _, nl = oracle.compact_kv(kc, vc, np.array([9]), kt, vt, np.array([[1, 3, 6]]), np.array([3]))
    assert nl.tolist() == [10]
    np.testing.assert_array_equal(k2[0, 0, 9], kt[0, 0, 0])


def test_an_invalid_node_ends_the_copy():
    kc, vc, kt, vt = _arrays(1, 1, 12, 4, 2, seed=3)
    k2, _, nl = oracle.compact_kv(kc, vc, np.array([2]), kt, vt, np.array([[1, 9, 2]]), np.array([3]))
    assert nl.tolist() == [3]
    np.testing.assert_array_equal(k2[0, 0, 2], kt[0, 0, 0])
    np.testing.assert_array_equal(k2[0, 0, 3:], kc[0, 0, 3:])


def test_compacted_cache_gives_the_accepted_node_its_tree_attention():
    rng = np.random.default_rng(4)
    Hq, Hkv, D, L, Lmax = 4, 2, 8, 11, 32
    parents = np.array([0, 0, 1, 1, 3, 2, 5, 4, 7])   # a tree of 9 nodes
    n = parents.shape[0]
    depth = np.zeros(n, dtype=int)
    for i in range(n):
        depth[i] = 1 if parents[i] == 0 else depth[parents[i] - 1] + 1
    kc, vc, kt, vt = _arrays(1, Hkv, Lmax, n, D, seed=5)
    q = rng.normal(size=(n, Hq, D))
    for x in range(1, n + 1):
        chain, node = [], x
        while node:
            chain.append(node)
            node = parents[node - 1]
        chain = chain[::-1]                              # root path of x, depth 1 first
        path = np.full((1, 6), -1)
        path[0, :len(chain)] = chain
        k2, v2, nl = oracle.compact_kv(kc, vc, np.array([L]), kt, vt, path, np.array([len(chain)]))
        T = int(nl[0])
        assert T == L + depth[x - 1]
        tree = oracle.tree_attention(q, kc[0], vc[0], L, kt[0], vt[0], parents, depth)[x - 1]
        G = Hq // Hkv
        kk = torch.from_numpy(np.repeat(k2[0][:, :T], G, axis=0))   # [Hq][T][D]
        vv = torch.from_numpy(np.repeat(v2[0][:, :T], G, axis=0))
        qq = torch.from_numpy(q[x - 1][:, None, :])                  # [Hq][1][D]
        plain = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0].numpy()
        np.testing.assert_allclose(tree, plain, rtol=1e-12, atol=1e-12)
