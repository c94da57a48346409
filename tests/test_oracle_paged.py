"""Pins for the oracle's paged prefix cache (no GPU).

Scattering a dense cache into pages of a shuffled pool and gathering it back
gives the dense cache for every page size; compaction into pages equals
compact_kv on the gathered view (same new lengths, same entries) and stops at a
page that is not allocated; tree attention over a gathered paged cache equals
tree attention over the dense cache it came from.
"""
import numpy as np
import pytest

import oracle


def _scatter(dense, ps, rng, spare=3):
    """dense [B][Hkv][Lmax][D] -> pools with the pages of all sequences shuffled, and the tables."""
    B, Hkv, Lmax, D = dense.shape
    pps = (Lmax + ps - 1) // ps
    num_pages = B * pps + spare
    ids = rng.permutation(num_pages)[:B * pps].reshape(B, pps)
    pool = rng.normal(size=(num_pages, Hkv, ps, D))
    for b in range(B):
        for e in range(pps):
            seg = dense[b, :, e * ps:(e + 1) * ps]
            pool[ids[b, e], :, :seg.shape[1]] = seg
    return pool, ids


@pytest.mark.parametrize("ps", [16, 32, 64, 128, 192])
def test_scatter_gather_round_trip(ps):
    rng = np.random.default_rng(ps)
    dense = rng.normal(size=(3, 2, 300, 8))
    pool, ids = _scatter(dense, ps, rng)
    for b, L in enumerate([300, 1, 157]):
        np.testing.assert_array_equal(oracle.gather_pages(pool, ids[b], L), dense[b][:, :L])


@pytest.mark.parametrize("ps", [16, 64])
def test_compaction_into_pages_equals_dense_compaction(ps):
    rng = np.random.default_rng(7)
    B, Hkv, Lmax, D, n, depth = 4, 2, 256, 8, 20, 5
    kc, vc = rng.normal(size=(B, Hkv, Lmax, D)), rng.normal(size=(B, Hkv, Lmax, D))
    kt, vt = rng.normal(size=(B, n, Hkv, D)), rng.normal(size=(B, n, Hkv, D))
    path = rng.integers(1, n + 1, size=(B, depth))
    acc = np.array([5, 0, 3, 5])
    plen = np.array([17, 100, 254, 64])
    kp, ids = _scatter(kc, ps, rng)
    vp, _ = _scatter(vc, ps, np.random.default_rng(7))
    vp = np.zeros_like(kp)
    for b in range(B):
        for e in range(ids.shape[1]):
            seg = vc[b, :, e * ps:(e + 1) * ps]
            vp[ids[b, e], :, :seg.shape[1]] = seg
    k2, v2, nl = oracle.compact_kv_paged(kp, vp, ids, plen, kt, vt, path, acc)
    kd, vd, nld = oracle.compact_kv(kc, vc, plen, kt, vt, path, acc)
    assert nl.tolist() == nld.tolist()
    for b in range(B):
        np.testing.assert_array_equal(oracle.gather_pages(k2, ids[b], int(nl[b])), kd[b][:, :nl[b]])
        np.testing.assert_array_equal(oracle.gather_pages(v2, ids[b], int(nl[b])), vd[b][:, :nl[b]])


def test_compaction_stops_at_an_unallocated_page():
    rng = np.random.default_rng(8)
    kp, vp = rng.normal(size=(4, 1, 16, 4)), rng.normal(size=(4, 1, 16, 4))
    kt, vt = rng.normal(size=(1, 6, 1, 4)), rng.normal(size=(1, 6, 1, 4))
    table = np.array([[2, 0, -1, 3]])
    k2, _, nl = oracle.compact_kv_paged(kp, vp, table, [30], kt, vt, np.array([[1, 2, 3, 4]]), [4])
    assert nl.tolist() == [32]                       # positions 30, 31 on page 0; 32 would need entry 2
    np.testing.assert_array_equal(k2[0, :, 14], kt[0, 0])
    np.testing.assert_array_equal(k2[0, :, 15], kt[0, 1])


def test_attention_over_gathered_pages_is_dense_attention():
    rng = np.random.default_rng(9)
    Hq, Hkv, D, L, n = 4, 2, 8, 150, 6
    kc, vc = rng.normal(size=(1, Hkv, L, D)), rng.normal(size=(1, Hkv, L, D))
    kp, ids = _scatter(kc, 32, rng)
    vp = np.zeros_like(kp)
    for e in range(ids.shape[1]):
        seg = vc[0, :, e * 32:(e + 1) * 32]
        vp[ids[0, e], :, :seg.shape[1]] = seg
    parents, depth = np.array([0, 1, 1, 2, 0, 5]), np.array([1, 2, 2, 3, 1, 2])
    q, kt, vt = rng.normal(size=(n, Hq, D)), rng.normal(size=(n, Hkv, D)), rng.normal(size=(n, Hkv, D))
    a = oracle.tree_attention(q, kc[0], vc[0], L, kt, vt, parents, depth)
    b = oracle.tree_attention(q, oracle.gather_pages(kp, ids[0], L), oracle.gather_pages(vp, ids[0], L), L, kt, vt,
                              parents, depth)
    np.testing.assert_array_equal(a, b)
