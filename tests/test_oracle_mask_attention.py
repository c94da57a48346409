"""Pins for the oracle's tree mask and tree attention (no GPU).

The mask is tied to closed forms (a chain gives the lower triangle, a star the
identity, popcount = depth) and to numpy's own bit unpacking.  Attention values
are not printed on the pages, so they are tied to library attention on the
special cases the tree reduces to: a chain tree is causal attention over
prefix + chain, a one-node tree is ordinary decode attention, GQA equals MHA
with each KV head repeated, a wide window is no window, a narrow window on a
chain is banded causal attention, and relabelling nodes permutes the outputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _sdpa(q, k, v, mask):
    """Library attention in fp64: q [Hq][nq][D], k/v [Hq][nk][D], mask [nq][nk] bool."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=torch.from_numpy(mask))
    return out.numpy()


def test_mask_chain_is_lower_triangle():
    n = 9
    parents = np.arange(n)
    assert (oracle.ancestor_mask(parents) == np.tril(np.ones((n, n), dtype=bool))).all()


def test_mask_star_is_identity():
    n = 7
    assert (oracle.ancestor_mask(np.zeros(n, dtype=int)) == np.eye(n, dtype=bool)).all()


def test_mask_rows_are_ancestor_sets_and_popcount_is_depth():
    # 1,2 children of root; 3,4 of 1; 5 of 3; 6 of 2; 7 of 5
    parents = np.array([0, 0, 1, 1, 3, 2, 5])
    depth = np.array([1, 1, 2, 2, 3, 2, 4])
    m = oracle.ancestor_mask(parents)
    expect = {1: {1}, 2: {2}, 3: {1, 3}, 4: {1, 4}, 5: {1, 3, 5}, 6: {2, 6}, 7: {1, 3, 5, 7}}
    for i in range(7):
        assert set((np.where(m[i])[0] + 1).tolist()) == expect[i + 1]
    packed = oracle.pack_mask(m, words=2)
    bits = np.unpackbits(packed.view(np.uint8), bitorder="little").reshape(7, 128)
    assert (bits[:, :7].astype(bool) == m).all() and not bits[:, 7:].any()
    assert (bits.sum(axis=1) == depth).all()


def test_mask_bits_cross_word_boundary():
    n = 100
    parents = np.arange(n)   # chain: row i has bits 0..i
    packed = oracle.pack_mask(oracle.ancestor_mask(parents), words=2)
    bits = np.unpackbits(packed.view(np.uint8), bitorder="little").reshape(n, 128)
    assert (bits[:, :n] == np.tril(np.ones((n, n), dtype=np.uint8))).all()


def test_positions():
    assert oracle.positions(np.array([1, 2, 3]), 10).tolist() == [10, 11, 12]


def _rand(rng, *shape):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("L,n,Hq,Hkv,D", [(17, 5, 4, 4, 16), (40, 8, 8, 2, 32)])
def test_chain_tree_is_causal_attention(L, n, Hq, Hkv, D):
    rng = np.random.default_rng(10)
    q = _rand(rng, n, Hq, D)
    kc, vc = _rand(rng, Hkv, L + 3, D), _rand(rng, Hkv, L + 3, D)
    kt, vt = _rand(rng, n, Hkv, D), _rand(rng, n, Hkv, D)
    parents = np.arange(n)
    depth = np.arange(1, n + 1)
    out = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth)
    G = Hq // Hkv
    K = np.concatenate([kc[:, :L], kt.transpose(1, 0, 2)], axis=1)     # [Hkv][L+n][D]
    Vv = np.concatenate([vc[:, :L], vt.transpose(1, 0, 2)], axis=1)
    K, Vv = np.repeat(K, G, axis=0), np.repeat(Vv, G, axis=0)
    causal = np.tril(np.ones((n, L + n), dtype=bool), k=L)             # query i sees keys <= L+i
    ref = _sdpa(q.transpose(1, 0, 2).copy(), K, Vv, causal).transpose(1, 0, 2)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_one_node_tree_is_decode_attention():
    rng = np.random.default_rng(11)
    L, Hq, Hkv, D = 33, 4, 2, 16
    q = _rand(rng, 1, Hq, D)
    kc, vc = _rand(rng, Hkv, L, D), _rand(rng, Hkv, L, D)
    kt, vt = _rand(rng, 1, Hkv, D), _rand(rng, 1, Hkv, D)
    out = oracle.tree_attention(q, kc, vc, L, kt, vt, np.array([0]), np.array([1]))
    K = np.repeat(np.concatenate([kc, kt.transpose(1, 0, 2)], axis=1), Hq // Hkv, axis=0)
    Vv = np.repeat(np.concatenate([vc, vt.transpose(1, 0, 2)], axis=1), Hq // Hkv, axis=0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2).copy()), torch.from_numpy(K),
        torch.from_numpy(Vv)).numpy().transpose(1, 0, 2)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def _tree_case(rng, L=29, Hq=8, Hkv=2, D=16):
    parents = np.array([0, 0, 1, 1, 3, 2, 5, 2])
    depth = np.array([1, 1, 2, 2, 3, 2, 4, 2])
    n = parents.shape[0]
    return (_rand(rng, n, Hq, D), _rand(rng, Hkv, L, D), _rand(rng, Hkv, L, D),
            _rand(rng, n, Hkv, D), _rand(rng, n, Hkv, D), parents, depth, L)


def test_gqa_equals_mha_with_repeated_heads():
    rng = np.random.default_rng(12)
    q, kc, vc, kt, vt, parents, depth, L = _tree_case(rng)
    G = q.shape[1] // kc.shape[0]
    a = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth)
    b = oracle.tree_attention(q, np.repeat(kc, G, axis=0), np.repeat(vc, G, axis=0), L,
                              np.repeat(kt, G, axis=1), np.repeat(vt, G, axis=1), parents, depth)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_tree_rows_match_sdpa_with_ancestor_mask():
    """General tree against library attention given the ancestor sets written out
    by hand for this tree."""
    rng = np.random.default_rng(13)
    q, kc, vc, kt, vt, parents, depth, L = _tree_case(rng)
    anc = {1: [1], 2: [2], 3: [1, 3], 4: [1, 4], 5: [1, 3, 5], 6: [2, 6], 7: [1, 3, 5, 7], 8: [2, 8]}
    n, Hq, D = q.shape
    G = Hq // kc.shape[0]
    mask = np.zeros((n, L + n), dtype=bool)
    mask[:, :L] = True
    for i, a in anc.items():
        for j in a:
            mask[i - 1, L + j - 1] = True
    K = np.repeat(np.concatenate([kc, kt.transpose(1, 0, 2)], axis=1), G, axis=0)
    Vv = np.repeat(np.concatenate([vc, vt.transpose(1, 0, 2)], axis=1), G, axis=0)
    ref = _sdpa(q.transpose(1, 0, 2).copy(), K, Vv, mask).transpose(1, 0, 2)
    out = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    rows = [(0, 0), (4, 3), (6, 7), (7, 5)]
    sub = oracle.tree_attention_rows(q, kc, vc, L, kt, vt, parents, depth, rows)
    np.testing.assert_allclose(sub, np.array([ref[i, h] for i, h in rows]), rtol=1e-10, atol=1e-12)


def test_wide_window_is_no_window_and_narrow_window_is_banded():
    rng = np.random.default_rng(14)
    q, kc, vc, kt, vt, parents, depth, L = _tree_case(rng)
    a = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth)
    b = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth, window=L + 5)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    # chain with window W: query at position L-1+i (i = 1..n) sees positions
    # within W back of itself, i.e. banded causal attention over prefix + chain
    n, W = 6, 9
    Hq, Hkv, D = 4, 4, 8
    qc = _rand(rng, n, Hq, D)
    kt2, vt2 = _rand(rng, n, Hkv, D), _rand(rng, n, Hkv, D)
    kcc, vcc = _rand(rng, Hkv, L, D), _rand(rng, Hkv, L, D)
    out = oracle.tree_attention(qc, kcc, vcc, L, kt2, vt2, np.arange(n), np.arange(1, n + 1), window=W)
    keypos = np.arange(L + n)                       # prefix 0..L-1, chain L..L+n-1
    qpos = L + np.arange(n)
    band = (keypos[None, :] <= qpos[:, None]) & (keypos[None, :] > qpos[:, None] - W)
    K = np.concatenate([kcc, kt2.transpose(1, 0, 2)], axis=1)
    Vv = np.concatenate([vcc, vt2.transpose(1, 0, 2)], axis=1)
    ref = _sdpa(qc.transpose(1, 0, 2).copy(), K, Vv, band).transpose(1, 0, 2)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_node_relabelling_permutes_outputs():
    rng = np.random.default_rng(15)
    q, kc, vc, kt, vt, parents, depth, L = _tree_case(rng)
    n = parents.shape[0]
    perm = np.array([1, 0, 5, 2, 3, 7, 4, 6])   # new index of old node i (0-based)
    newpar = np.zeros(n, dtype=int)
    for i in range(n):
        p = parents[i]
        newpar[perm[i]] = 0 if p == 0 else perm[p - 1] + 1
    q2, kt2, vt2, d2 = (np.empty_like(q), np.empty_like(kt), np.empty_like(vt), np.empty_like(depth))
    q2[perm], kt2[perm], vt2[perm], d2[perm] = q, kt, vt, depth
    a = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth)
    b = oracle.tree_attention(q2, kc, vc, L, kt2, vt2, newpar, d2)
    np.testing.assert_allclose(b[perm], a, rtol=1e-12, atol=1e-14)


def test_scale_default_is_inverse_sqrt_head_dim():
    rng = np.random.default_rng(16)
    q, kc, vc, kt, vt, parents, depth, L = _tree_case(rng)
    a = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth)
    b = oracle.tree_attention(q, kc, vc, L, kt, vt, parents, depth, scale=1 / math.sqrt(q.shape[2]))
    np.testing.assert_array_equal(a, b)
