"""Pins for the oracle's EAGLE-1 static tree (no GPU).

A hand-worked template; the full k-ary tree of depth 2 equals the dynamic
EAGLE-2 tree of depth 2 that keeps every candidate (the level-1 frontier is the
whole first level, ordered by rank, which is the static row order); any kept
dynamic tree, re-read as a template (its parents and each node's child rank),
gives back the same tokens and log V from the same rows; a chain of rank-0
nodes is the argmax chain; relabelling the vocabulary relabels the tokens.
"""
import json
import os

import numpy as np
import pytest
from scipy.special import logsumexp as sp_logsumexp

import oracle
from workloads import gen_draft_logits, get_config


def test_handworked(golden_dir):
    with open(os.path.join(golden_dir, "static_tree_handworked.json")) as f:
        fx = json.load(f)
    x = np.array(fx["logits"], dtype=np.float64)
    t = oracle.build_static_tree(x, fx["parents"], fx["ranks"])
    assert t["tokens"].tolist() == fx["tokens"]
    assert t["depth"].tolist() == fx["depth"]
    assert t["draft_row"].tolist() == fx["draft_row"]
    lse = sp_logsumexp(x, axis=1)
    assert t["logV"][4] == pytest.approx((3 - lse[0]) + (5 - lse[1]) + (7 - lse[2]), abs=1e-12)
    np.testing.assert_allclose(t["row_lse"], lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("k,V,seed", [(2, 50, 0), (4, 300, 1), (10, 1000, 2)])
def test_full_kary_depth2_is_the_dynamic_tree(k, V, seed):
    cfg = get_config("tiny", depth=2, k=k, m=k + k * k, V=V, B=1, logits_dtype="f32")
    x = oracle.decode_logits(gen_draft_logits(cfg, seed), "f32")[0]
    dyn = oracle.build_tree(x, 2, k, k + k * k)
    parents = [0] * k + [1 + s for s in range(k) for _ in range(k)]
    ranks = list(range(k)) + [r for _ in range(k) for r in range(k)]
    st = oracle.build_static_tree(x, parents, ranks)
    for f in ("tokens", "parents", "depth", "draft_row"):
        assert st[f].tolist() == dyn[f].tolist(), f
    np.testing.assert_array_equal(st["logV"], dyn["logV"])


def _child_rank(gid, level, k):
    return gid if level == 1 else (gid - k - (level - 2) * k * k) % k


@pytest.mark.parametrize("name,seed", [("tiny", 0), ("7b", 1), ("l3-8b", 2), ("serve", 3)])
def test_kept_dynamic_tree_as_a_template(name, seed):
    cfg = get_config(name)
    x = oracle.decode_logits(gen_draft_logits(cfg, seed), cfg.logits_dtype)
    for b in range(min(cfg.B, 3)):
        dyn = oracle.build_tree(x[b], cfg.depth, cfg.k, cfg.m)
        ranks = [_child_rank(int(g), int(d), cfg.k) for g, d in zip(dyn["gid"], dyn["depth"])]
        rows = oracle.template_rows(dyn["parents"])
        # the static rows: for each node with a child, the dynamic row it was expanded from
        src = np.zeros(int(rows.max()) + 1, dtype=np.int64)
        for node in range(dyn["n"] + 1):
            if rows[node] >= 0:
                src[rows[node]] = dyn["draft_row"][node]
        st = oracle.build_static_tree(x[b][src], dyn["parents"], ranks)
        assert st["tokens"].tolist() == dyn["tokens"].tolist()
        assert st["depth"].tolist() == dyn["depth"].tolist()
        np.testing.assert_array_equal(st["logV"], dyn["logV"])


def test_rank0_chain_is_the_argmax_chain():
    rng = np.random.default_rng(5)
    x = rng.normal(size=(6, 40))
    st = oracle.build_static_tree(x, list(range(6)), [0] * 6)     # node i+1's parent is node i
    assert st["draft_row"].tolist() == [0, 1, 2, 3, 4, 5, -1]
    assert st["tokens"].tolist() == [int(np.argmax(x[r])) for r in range(6)]


def test_token_relabelling():
    rng = np.random.default_rng(6)
    V = 64
    parents, ranks = [0, 0, 0, 1, 1, 2, 4], [0, 1, 2, 0, 1, 0, 0]
    R = int(oracle.template_rows(parents).max()) + 1
    x = rng.normal(size=(R, V))
    perm = rng.permutation(V)
    y = np.empty_like(x)
    y[:, perm] = x                     # token v becomes perm[v]
    a = oracle.build_static_tree(x, parents, ranks)
    b = oracle.build_static_tree(y, parents, ranks)
    assert b["tokens"].tolist() == perm[a["tokens"]].tolist()
    np.testing.assert_allclose(b["logV"], a["logV"], rtol=0, atol=1e-12)


def test_rank_paths_to_template():
    """The binding's rank-path helper (host code) gives the template whose
    static tree, on rows from the oracle's dynamic depth-2 tree, is that tree."""
    import eagle_tree_verification_dynamic_b200 as et
    k = 3
    paths = [(s, r) for s in range(k) for r in range(k)] + [(r,) for r in range(k)]
    parents, ranks = et.static_template_from_paths(paths)
    assert parents == [0] * k + [1 + s for s in range(k) for _ in range(k)]
    assert ranks == list(range(k)) + [r for _ in range(k) for r in range(k)]
    cfg = get_config("tiny", depth=2, k=k, m=k + k * k, V=60, B=1, logits_dtype="f32")
    x = oracle.decode_logits(gen_draft_logits(cfg, 9), "f32")[0]
    st = oracle.build_static_tree(x, parents, ranks)
    dyn = oracle.build_tree(x, 2, k, k + k * k)
    assert st["tokens"].tolist() == dyn["tokens"].tolist()
    with pytest.raises(et.EagleError):
        et.static_template_from_paths([(0,), (1, 0)])          # (1,) is missing
    assert et.static_template_from_paths([(0, 0), (0,), (0, 0, 2)]) == ([0, 1, 2], [0, 0, 2])
