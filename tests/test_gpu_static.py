"""GPU parity: EAGLE-1 static tree (eagle_static_tree_build) against the oracle.

Tokens, parents, depth, draft rows and node ids bit-exact; log V within
depth x 5e-7 (one row log-sum-exp per level) plus the fp32 store's half ulp,
row log-sum-exp within 5e-7.  Templates: the hand-worked
one, the full k-ary tree of depth 2, kept dynamic trees re-read as templates
(the shapes EAGLE-2 produces), a long rank-0 chain and a 128-node template;
then a whole step on a static tree (mask, attention, sampled acceptance)
against the oracle.
"""
import json
import os

import numpy as np
import pytest
import torch

import eagle_tree_verification_dynamic_b200 as et
import oracle
from workloads import gen_draft_logits, get_config, make_target_logits, make_workload

from parity import walk_match
from gpu_helpers import attention_ref, check_attention, dec, i32, to_dev_bf16, to_dev_logits

pytestmark = pytest.mark.gpu


def _check(x_stored, dtype, parents, ranks):
    B = x_stored.shape[0]
    tree = et.static_tree_build(to_dev_logits(x_stored, dtype), parents, ranks)
    torch.cuda.synchronize()
    x64 = oracle.decode_logits(x_stored, dtype)
    refs = []
    for b in range(B):
        ref = oracle.build_static_tree(x64[b], parents, ranks)
        for f in ("tokens", "parents", "depth", "draft_row", "gid"):
            assert getattr(tree, f)[b].cpu().numpy().tolist() == ref[f].tolist(), (b, f)
        # each row log-sum-exp on the path is within 5e-7 of fp64, and the fp32
        # store rounds by half an ulp of |log V|
        bound = ref["depth"] * 5e-7 + np.abs(ref["logV"]) * 2.0 ** -24 + 1e-7
        assert np.all(np.abs(tree.logV[b].cpu().numpy() - ref["logV"]) <= bound), b
        np.testing.assert_allclose(tree.row_lse[b].cpu().numpy(), ref["row_lse"], rtol=0, atol=5e-7)
        refs.append(ref)
    return tree, refs


def _rows_for(parents, ranks, B, V, dtype, seed):
    R = et.static_tree_rows(parents, ranks)
    cfg = get_config("tiny", B=B, V=V, logits_dtype=dtype, depth=2, k=R - 1)   # R = 1 + (2-1)(R-1) rows
    return gen_draft_logits(cfg, seed)


def test_handworked(golden_dir):
    with open(os.path.join(golden_dir, "static_tree_handworked.json")) as f:
        fx = json.load(f)
    x = np.array(fx["logits"], dtype=np.float32)[None]
    tree, _ = _check(x, "f32", fx["parents"], fx["ranks"])
    assert tree.tokens[0].cpu().numpy().tolist() == fx["tokens"]


@pytest.mark.parametrize("k,V,dtype", [(10, 32000, "f32"), (8, 128256, "bf16"), (4, 1000, "bf16")])
def test_full_kary_depth2(k, V, dtype):
    parents = [0] * k + [1 + s for s in range(k) for _ in range(k)]
    ranks = list(range(k)) + [r for _ in range(k) for r in range(k)]
    _check(_rows_for(parents, ranks, 3, V, dtype, k), dtype, parents, ranks)


def _child_rank(gid, level, k):
    return gid if level == 1 else (gid - k - (level - 2) * k * k) % k


@pytest.mark.parametrize("name", ["7b", "l3-8b", "serve"])
def test_kept_dynamic_trees_as_templates(name):
    cfg = get_config(name)
    x = oracle.decode_logits(gen_draft_logits(cfg, 5), cfg.logits_dtype)
    dyn = oracle.build_tree(x[0], cfg.depth, cfg.k, cfg.m)
    ranks = [_child_rank(int(g), int(d), cfg.k) for g, d in zip(dyn["gid"], dyn["depth"])]
    parents = dyn["parents"].tolist()
    _check(_rows_for(parents, ranks, 4, cfg.V, cfg.logits_dtype, 6), cfg.logits_dtype, parents, ranks)


def test_long_chain_and_largest_template():
    chain = list(range(40))
    _check(_rows_for(chain, [0] * 40, 2, 5000, "f32", 7), "f32", chain, [0] * 40)
    rng = np.random.default_rng(8)
    parents, ranks, used = [], [], {}
    for i in range(128):                        # random template, every rank below 32, unique per parent
        while True:
            p = int(rng.integers(0, i + 1))
            free = [r for r in range(32) if r not in used.get(p, set())]
            if free:
                break
        r = int(rng.choice(free))
        used.setdefault(p, set()).add(r)
        parents.append(p)
        ranks.append(r)
    _check(_rows_for(parents, ranks, 2, 3000, "bf16", 9), "bf16", parents, ranks)


def test_static_step_against_the_oracle():
    """A static tree of the 7b shape through mask, attention and sampled acceptance."""
    cfg = get_config("7b")
    x64 = oracle.decode_logits(gen_draft_logits(cfg, 1), cfg.logits_dtype)
    dyn = oracle.build_tree(x64[0], cfg.depth, cfg.k, cfg.m)
    ranks = [_child_rank(int(g), int(d), cfg.k) for g, d in zip(dyn["gid"], dyn["depth"])]
    parents = dyn["parents"].tolist()
    stored = _rows_for(parents, ranks, 1, cfg.V, cfg.logits_dtype, 2)
    tree, refs = _check(stored, cfg.logits_dtype, parents, ranks)
    ref = refs[0]
    n = tree.n
    w = make_workload(cfg, 3)
    plen = torch.from_numpy(w.prefix_len).cuda()
    mask, pos = et.tree_mask(tree.parents, tree.depth, plen)
    np.testing.assert_array_equal(mask[0].cpu().numpy().view(np.uint64),
                                  oracle.pack_mask(oracle.ancestor_mask(ref["parents"])))
    out = et.tree_attention(to_dev_bf16(w.q[:, :n]), to_dev_bf16(w.k_cache), to_dev_bf16(w.v_cache), plen,
                            to_dev_bf16(w.k_tree[:, :n]), to_dev_bf16(w.v_tree[:, :n]), mask, pos)
    torch.cuda.synchronize()
    rows = [(i, h) for i in range(0, n, 7) for h in (0, 13, cfg.Hq - 1)] + [(n - 1, 5)]
    want, s = attention_ref(dec(w.q[0, :n]), dec(w.k_cache[0]), dec(w.v_cache[0]), int(w.prefix_len[0]),
                            dec(w.k_tree[0, :n]), dec(w.v_tree[0, :n]), ref["parents"], ref["depth"], rows=rows)
    o = out[0].float().cpu().numpy()
    check_attention(np.array([o[i, h] for i, h in rows]), want, s)
    tgt = make_target_logits(cfg, 3, stored, ref["draft_row"][None])
    u = np.random.default_rng(10).random((1, 2, n + 1)).astype(np.float32)
    acc, path, bonus = et.accept(to_dev_logits(tgt, cfg.logits_dtype), tree.tokens, tree.parents, tree.draft_row,
                                 cfg.depth, torch.from_numpy(u).cuda(), to_dev_logits(stored, cfg.logits_dtype),
                                 tree.row_lse)
    T64 = oracle.decode_logits(tgt, cfg.logits_dtype)[0]
    D64 = oracle.decode_logits(stored, cfg.logits_dtype)[0]
    walk = lambda nodes=(): oracle.accept_stochastic(T64, D64, ref["tokens"], ref["parents"], ref["draft_row"],
                                                     u[0].astype(np.float64), cfg.depth, flip=set(nodes))
    got = (int(acc[0]), path[0].cpu().numpy().tolist(), int(bonus[0]))
    walk_match(got, walk(), walk)
