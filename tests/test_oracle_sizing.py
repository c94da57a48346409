"""Pins for the oracle's cost-aware sizing (no GPU).

Interpolation: multilinear interpolation reproduces, on and off the grid and
outside it, any function that is linear in each of B, L and N separately, so a
table sampled from such a function must give its exact values anywhere.  Gains:
level 1 is the sum of the root's k largest probabilities; with k = 1 level l's
gain is the product of the argmax probabilities down the argmax chain; the
gains never grow from one level to the next (a child's V is at most its
parent's and the level's best k descend from the previous best k).  Decisions:
threshold 0 keeps every level; a hand-worked table; a table that is flat in N
at batch 1 and linear in B*N at large batch keeps fewer levels as B grows.
"""
import itertools

import numpy as np
import pytest
from scipy.special import softmax

import oracle
from sizing_helpers import confident_draft, oracle_grow_widths, saturating_table
from workloads import gen_draft_logits, get_config


def _f(B, L, N):
    return 3.0 + 0.5 * B + 0.01 * L + 2.0 * N + 0.002 * B * L + 0.25 * B * N + 1e-4 * L * N + 3e-6 * B * L * N


def test_interpolation_reproduces_multilinear_functions():
    Bs, Ls, Ns = [1, 4, 16, 64], [512, 2048, 8192], [0, 16, 64, 128]
    us = np.array([[[_f(b, l, n) for n in Ns] for l in Ls] for b in Bs])
    rng = np.random.default_rng(0)
    pts = list(itertools.product(Bs, Ls, Ns))
    pts += [(rng.uniform(0.5, 100), rng.uniform(100, 20000), rng.uniform(-5, 200)) for _ in range(300)]
    for B, L, N in pts:
        assert oracle.cost_at(Bs, Ls, Ns, us, B, L, N) == pytest.approx(_f(B, L, N), rel=1e-12, abs=1e-9)


def test_single_point_axes_are_constant():
    us = np.array([[[5.0, 9.0]]])
    assert oracle.cost_at([8], [1000], [0, 10], us, 1, 50000, 5) == pytest.approx(7.0)
    assert oracle.cost_at([8], [1000], [0, 10], us, 64, 1, 20) == pytest.approx(13.0)


def test_level_one_gain_is_the_root_topk_mass():
    cfg = get_config("7b")
    x = oracle.decode_logits(gen_draft_logits(cfg, 2), cfg.logits_dtype)[0]
    t = oracle.build_tree(x, cfg.depth, cfg.k, cfg.m)
    p = np.sort(softmax(x[0]))[::-1]
    assert t["gains"][0] == pytest.approx(p[:cfg.k].sum(), rel=1e-12)
    assert len(t["gains"]) == cfg.depth
    assert np.all(np.diff(t["gains"]) <= 1e-15)                 # never grows


def test_k1_gains_are_argmax_chain_products():
    cfg = get_config("tiny", depth=6, k=1, m=6, V=200, B=1, logits_dtype="f32")
    x = oracle.decode_logits(gen_draft_logits(cfg, 3), "f32")[0]
    t = oracle.build_tree(x, cfg.depth, 1, 6)
    prod = np.cumprod([softmax(x[r]).max() for r in range(cfg.depth)])
    np.testing.assert_allclose(t["gains"], prod, rtol=1e-12)


@pytest.mark.parametrize("name,seed", [("l3-8b", 1), ("serve", 2), ("long", 0)])
def test_gains_never_grow(name, seed):
    cfg = get_config(name)
    x = oracle.decode_logits(gen_draft_logits(cfg, seed), cfg.logits_dtype)
    for b in range(min(cfg.B, 3)):
        g = oracle.build_tree(x[b], cfg.depth, cfg.k, cfg.m)["gains"]
        assert np.all(np.diff(g) <= 1e-15) and g[0] <= cfg.k


def test_threshold_zero_keeps_every_level_and_a_handworked_case():
    # cost 10 + 2N at any B and L: each level of k = 4 costs 8
    Bs, Ls, Ns = [1, 2], [100, 200], [0, 100]
    us = np.array([[[10.0, 210.0]] * 2] * 2)
    table = (Bs, Ls, Ns, us)
    gains = [[0.9, 0.9], [0.5, 0.5], [0.2, 0.1], [0.05, 0.05]]   # batch sums 1.8, 1.0, 0.3, 0.1
    assert oracle.levels_kept(table, 2, 150, 4, gains, 0.0) == 4
    # ratios 1.8/8 = .225, 1/8 = .125, .3/8 = .0375: threshold .1 keeps two levels, .2 one, .3 none
    assert oracle.levels_kept(table, 2, 150, 4, gains, 0.1) == 2
    assert oracle.levels_kept(table, 2, 150, 4, gains, 0.2) == 1
    assert oracle.levels_kept(table, 2, 150, 4, gains, 0.3) == 0


def test_larger_batches_keep_fewer_levels():
    """Verification cost flat in N until the batch's tokens saturate the GPU,
    then linear in B*N (memory-bound at batch 1, compute-bound at large batch)."""
    Bs, Ls, Ns = [1, 2, 4, 8, 16, 32, 64], [1024, 4096], list(range(0, 161, 8))
    us = np.array([[[max(50.0, 0.05 * b * n) for n in Ns] for _ in Ls] for b in Bs])
    table = (Bs, Ls, Ns, us)
    cfg = get_config("tiny", depth=8, k=4, m=32, V=500, B=64, logits_dtype="f32")
    x = oracle.decode_logits(gen_draft_logits(cfg, 4), "f32")
    per_seq = [oracle.build_tree(x[b], cfg.depth, cfg.k, cfg.m)["gains"] for b in range(cfg.B)]
    kept = []
    for B in Bs:
        gl = [[per_seq[b][l] for b in range(B)] for l in range(cfg.depth)]
        kept.append(oracle.levels_kept(table, B, 2048, cfg.k, gl, 0.5))
    assert kept[0] == cfg.depth and kept[-1] < kept[0]
    assert all(a >= b for a, b in zip(kept, kept[1:])), kept


# ------------------------------------------------------- widening or deepening
def test_level_width_handworked():
    # cost 10 + 2N: every candidate costs 2 per step at any B, L
    table = ([1, 2], [100, 200], [0, 100], np.array([[[10.0, 210.0]] * 2] * 2))
    vals = [[0.9, 0.5, 0.2, 0.0], [0.7, 0.3, 0.1, 0.0]]   # batch gains 1.6, 0.8, 0.3, 0 -> ratios .8, .4, .15, 0
    assert oracle.level_width(table, 2, 150, 0, vals, 0.1)[0] == 3
    assert oracle.level_width(table, 2, 150, 0, vals, 0.4)[0] == 2
    assert oracle.level_width(table, 2, 150, 0, vals, 0.5)[0] == 1
    assert oracle.level_width(table, 2, 150, 0, vals, 0.9)[0] == 0
    assert oracle.level_width(table, 2, 150, 0, vals, 0.0)[0] == 3       # a candidate of V = 0 is never taken
    w, r = oracle.level_width(table, 2, 150, 5, vals, 0.1)
    np.testing.assert_allclose(r[:3], [0.8, 0.4, 0.15])


def test_level_width_flat_cost_takes_every_positive_candidate():
    # every candidate count on the grid: the cost difference is exactly 0 (an infinite ratio)
    table = ([1, 64], [128, 65536], list(range(40)), np.full((2, 2, 40), 40.0))
    assert oracle.level_width(table, 1, 128, 17, [[0.3, 1e-9, 1e-30, 0.0]], 1e6)[0] == 3


def test_batch_one_grows_wide_and_deep_large_batch_a_chain():
    """The harness's two ends: at batch 1 the cost does not grow with the tree, so every level keeps its
    full width; at batch 32 each further candidate costs 0.5 * 32 per step, which only each level's best
    candidate pays for (a chain)."""
    cfg, stored = confident_draft()
    x = oracle.decode_logits(stored, "f32")
    table = saturating_table()
    w1, t1 = oracle_grow_widths([x[0]], cfg.depth, cfg.k, table, 2048, 0.5)
    assert w1 == [cfg.k] * cfg.depth
    assert t1[0]["n"] == cfg.k * cfg.depth
    w32, t32 = oracle_grow_widths(list(x), cfg.depth, cfg.k, table, 2048, 0.5)
    assert w32 == [1] * cfg.depth, w32
    for t in t32:  # a chain: node i's parent is node i - 1
        assert t["parents"].tolist() == list(range(len(w32)))
