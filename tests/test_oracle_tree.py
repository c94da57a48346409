"""Pins for the oracle's EAGLE-2 tree builder (no GPU).

Each test ties the oracle to something other than itself: a fixture worked by
hand from the definitions, closed forms on special cases (k = 1, depth = 1,
m >= P) computed with library routines, the example shape of the EAGLE notes,
and invariants that a dropped term, a wrong index or a transposed operand would
break (shift invariance of each row, token relabelling, confidence products).
"""
import json
import os

import numpy as np
import pytest
from scipy.special import log_softmax, softmax

import oracle
from workloads import get_config, gen_draft_logits


def _fixture(golden_dir):
    with open(os.path.join(golden_dir, "tree_handworked.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("m", ["10", "7", "5"])
def test_handworked_tree(golden_dir, m):
    fx = _fixture(golden_dir)
    logits = np.log(np.array(fx["probs"], dtype=np.float64))
    t = oracle.build_tree(logits, fx["depth"], fx["k"], int(m))
    exp = fx["cases"][m]
    assert t["gid"].tolist() == exp["gid"]
    assert t["tokens"].tolist() == exp["tokens"]
    assert t["parents"].tolist() == exp["parents"]
    assert t["depth"].tolist() == exp["depth"]
    assert t["draft_row"].tolist() == exp["draft_row"]
    np.testing.assert_allclose(np.exp(t["logV"]), exp["V"], rtol=1e-12)


def test_example_shape_depth3_10_tokens():
    """The EAGLE notes' example draft tree has depth 3 and 10 tokens; with k=2 the
    pool is exactly 10, every candidate is kept, levels hold 2, 4, 4 nodes and two
    of the four level-2 nodes are expanded."""
    cfg = get_config("tiny")
    x = oracle.decode_logits(gen_draft_logits(cfg, 0), cfg.logits_dtype)
    t = oracle.build_tree(x[0], cfg.depth, cfg.k, cfg.m)
    assert t["n"] == 10 and t["P"] == 10
    assert t["depth"].max() == 3
    assert np.bincount(t["depth"], minlength=4)[1:].tolist() == [2, 4, 4]
    lvl2 = np.where(t["depth"] == 2)[0] + 1
    assert sum(int(t["draft_row"][n]) >= 0 for n in lvl2) == 2


def test_k1_is_argmax_chain():
    rng = np.random.default_rng(1)
    depth, V = 6, 50
    x = rng.normal(0, 3, size=(depth, V))
    t = oracle.build_tree(x, depth, 1, 6)
    assert t["tokens"].tolist() == [int(np.argmax(x[r])) for r in range(depth)]
    assert t["parents"].tolist() == list(range(depth))
    lp = [log_softmax(x[r])[int(np.argmax(x[r]))] for r in range(depth)]
    np.testing.assert_allclose(t["logV"], np.cumsum(lp), rtol=1e-12)
    assert t["draft_row"].tolist() == list(range(depth)) + [-1]


def test_depth1_is_topk_of_root():
    rng = np.random.default_rng(2)
    x = rng.normal(0, 3, size=(1, 40))
    x[0, 7] = x[0, 3]  # a tie: the lower token id must come first
    t = oracle.build_tree(x, 1, 5, 5)
    expect = np.argsort(-x[0], kind="stable")[:5]
    assert sorted(t["tokens"].tolist()) == sorted(expect.tolist())
    assert t["tokens"].tolist() == expect.tolist()  # ascending gid == rank order
    assert (t["parents"] == 0).all()


def test_m_at_least_pool_keeps_everything():
    rng = np.random.default_rng(3)
    depth, k, V = 4, 3, 30
    x = rng.normal(0, 3, size=(1 + (depth - 1) * k, V))
    P = k + (depth - 1) * k * k
    for m in (P, P + 5):
        t = oracle.build_tree(x, depth, k, m)
        assert t["n"] == P and t["gid"].tolist() == list(range(P))


def _invariants(t, x, k):
    n = t["n"]
    parents, depth, tokens, logV = t["parents"], t["depth"], t["tokens"], t["logV"]
    assert (parents < np.arange(1, n + 1)).all()           # parents precede children
    for i in range(n):
        p = parents[i]
        assert depth[i] == (1 if p == 0 else depth[p - 1] + 1)
        if p:
            assert logV[i] <= logV[p - 1]                  # monotone along paths
            assert t["draft_row"][p] >= 0                  # only expanded nodes have children
    counts = np.bincount(parents, minlength=n + 1)
    assert counts.max() <= k
    # exp(logV) equals the product of draft confidences along the path
    for i in range(n):
        prod, node = 1.0, i + 1
        while node:
            par = parents[node - 1]
            row = t["draft_row"][par]
            prod *= softmax(x[row])[tokens[node - 1]]
            node = par
        assert abs(np.exp(logV[i]) - prod) <= 1e-12 * prod


@pytest.mark.parametrize("name,seed", [("tiny", 0), ("7b", 0), ("7b", 3)])
def test_invariants_on_configs(name, seed):
    cfg = get_config(name)
    x = oracle.decode_logits(gen_draft_logits(cfg, seed), cfg.logits_dtype)[0]
    t = oracle.build_tree(x, cfg.depth, cfg.k, cfg.m)
    assert t["n"] == cfg.m
    _invariants(t, x, cfg.k)


def test_rerank_keeps_the_largest_values():
    """Every kept node's V is at least every dropped candidate's V (pool rebuilt
    from the kept frontier rows with library softmax)."""
    rng = np.random.default_rng(4)
    depth, k, V, m = 4, 3, 25, 12
    x = rng.normal(0, 3, size=(1 + (depth - 1) * k, V))
    t = oracle.build_tree(x, depth, k, m)
    full = oracle.build_tree(x, depth, k, 10 ** 6)
    kept = set(t["gid"].tolist())
    vk = [v for g, v in zip(full["gid"], full["logV"]) if g in kept]
    vd = [v for g, v in zip(full["gid"], full["logV"]) if g not in kept]
    assert min(vk) >= max(vd)
    _invariants(full, x, k)


def test_row_shift_invariance():
    """Adding a constant to a draft row changes no confidence, hence no tree."""
    rng = np.random.default_rng(5)
    depth, k, V, m = 5, 3, 40, 20
    x = rng.normal(0, 3, size=(1 + (depth - 1) * k, V))
    y = x + rng.normal(0, 10, size=(x.shape[0], 1))
    a = oracle.build_tree(x, depth, k, m)
    b = oracle.build_tree(y, depth, k, m)
    for key in ("tokens", "parents", "depth", "draft_row", "gid"):
        assert a[key].tolist() == b[key].tolist()
    np.testing.assert_allclose(a["logV"], b["logV"], rtol=1e-10)


def test_token_relabelling():
    """Permuting token ids in every row permutes the tree's tokens and nothing else."""
    rng = np.random.default_rng(6)
    depth, k, V, m = 4, 4, 60, 25
    x = rng.normal(0, 3, size=(1 + (depth - 1) * k, V))
    perm = rng.permutation(V)
    y = np.empty_like(x)
    y[:, perm] = x          # token t becomes perm[t]
    a = oracle.build_tree(x, depth, k, m)
    b = oracle.build_tree(y, depth, k, m)
    assert b["tokens"].tolist() == perm[a["tokens"]].tolist()
    assert a["parents"].tolist() == b["parents"].tolist()


def test_confident_draft_grows_deeper():
    """A confident draft concentrates V on one chain, so the reranked tree gets
    deeper; a flat draft keeps shallow nodes (EAGLE-2 "Reranking Nodes")."""
    rng = np.random.default_rng(7)
    depth, k, V, m = 6, 4, 100, 12
    flat = rng.normal(0, 0.1, size=(1 + (depth - 1) * k, V))
    sharp = flat.copy()
    sharp[:, 0] += 12.0
    assert oracle.build_tree(sharp, depth, k, m)["depth"].max() == depth
    assert oracle.build_tree(flat, depth, k, m)["depth"].max() <= 2


def test_frontiers_brute_force():
    """Each expanded level's frontier, by brute force: enumerate every root path
    of that depth from the rows' softmax (children of the previous frontier
    only), rank by the product of confidences, ties to the lower candidate id."""
    cfg = get_config("tiny", V=40, depth=4, k=3, B=1, logits_dtype="f32")
    x = gen_draft_logits(cfg, 11)[0].astype(np.float64)
    k = cfg.k
    t = oracle.build_tree(x, cfg.depth, k, 10**6)
    p = softmax(x, axis=1)
    # level 1: the root's children by probability, ties to the lower token
    order = sorted(range(x.shape[1]), key=lambda v: (-p[0, v], v))[:k]
    front = [(p[0, v], r, v) for r, v in enumerate(order)]          # (V, gid, token)
    for level in range(1, cfg.depth):
        ranked = sorted(front, key=lambda c: (-c[0], c[1]))[:k]
        got = t["frontiers"][level - 1]
        assert got["tokens"].tolist() == [c[2] for c in ranked]
        if level == 1:
            assert got["parent_slot"].tolist() == [-1] * k
        else:
            assert got["parent_slot"].tolist() == [(c[1] - k - (level - 2) * k * k) // k for c in ranked]
        nxt = []
        for s, (v, _, _) in enumerate(ranked):
            row = 1 + (level - 1) * k + s
            kids = sorted(range(x.shape[1]), key=lambda u: (-p[row, u], u))[:k]
            nxt += [(v * p[row, u], k + (level - 1) * k * k + s * k + r, u) for r, u in enumerate(kids)]
        front = nxt
    # with every candidate kept, frontier slot s of level l is the node owning row 1 + (l-1)k + s
    for level, f in enumerate(t["frontiers"], start=1):
        for s, tok in enumerate(f["tokens"]):
            node = int(np.nonzero(t["draft_row"][1:] == 1 + (level - 1) * k + s)[0][0])
            assert t["tokens"][node] == tok and t["depth"][node] == level
