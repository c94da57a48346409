"""Pins for the oracle's small helpers and for the exact near-tie escape of the
GPU parity tests (no GPU).

* near_tie: the 1e-6 relative band of the parity rule, checked on planted
  pairs just inside and just outside it.
* decode_logits(.., "bf16"): fixed bit patterns with known values, and
  agreement with torch's own bfloat16 on random patterns.
* the tree builder's near-tie flags: a cross-parent pair planted at a frontier
  cut and at the rerank cut is flagged, the same pair 2e-6 apart is not, and
  siblings (whose order rounding cannot change) are never flagged.
* flips: resolving a flagged decision the other way equals running the oracle
  on inputs moved just across the tie; the parity helpers excuse such a
  result and nothing else.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import tree_match, walk_match


# ------------------------------------------------------------------ near_tie
@pytest.mark.parametrize("a", [1.0, -3.0, -0.05, 250.0])
def test_near_tie_band(a):
    assert oracle.near_tie(a, a)
    assert oracle.near_tie(a, a * (1 + 0.5e-6))
    assert oracle.near_tie(a * (1 + 0.5e-6), a)
    assert not oracle.near_tie(a, a * (1 + 2e-6))
    assert not oracle.near_tie(a * (1 - 2e-6), a)


def test_near_tie_is_relative_to_the_larger_magnitude():
    assert oracle.near_tie(0.0, 0.0)
    assert not oracle.near_tie(0.0, 1e-300)
    assert oracle.near_tie(1e6, 1e6 + 0.9)      # 0.9e-6 relative
    assert not oracle.near_tie(1e6, 1e6 + 1.1)  # 1.1e-6 relative


# --------------------------------------------------------------- bf16 decode
@pytest.mark.parametrize("bits,value", [(0x3F80, 1.0), (0xC000, -2.0), (0x4049, 3.140625), (0x0000, 0.0),
                                        (0x8000, -0.0), (0x3F00, 0.5), (0x4120, 10.0), (0xC2C8, -100.0),
                                        (0x0001, 2.0 ** -133), (0x7F7F, 3.3895313892515355e38),
                                        (0x7F80, np.inf), (0xFF80, -np.inf)])
def test_decode_bf16_fixed_patterns(bits, value):
    got = oracle.decode_logits(np.array([bits], dtype=np.uint16), "bf16")[0]
    assert got == value and np.signbit(got) == np.signbit(value)


def test_decode_bf16_agrees_with_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2 ** 16, size=20000, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite values only (NaN payloads compare unequal)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = oracle.decode_logits(bits.reshape(40, -1)[:, :] if bits.size % 40 == 0 else bits, "bf16").reshape(-1)
    np.testing.assert_array_equal(got, ref)


def test_decode_f32_is_exact():
    x = np.random.default_rng(1).normal(0, 3, 1000).astype(np.float32)
    assert (oracle.decode_logits(x, "f32") == x.astype(np.float64)).all()


# ------------------------------------------------- tree near-tie flags, flips
def _rows(a: float, root=(0.5, 0.3, 0.15, 0.05), row1=(0.62, 0.25, 0.08, 0.05)):
    """depth 3, k 2, V 4 (rows 0..4).  Level-2 candidates: gid 2 (V 0.31),
    gid 3 (V 0.125) under gid 0; gid 4 (V 0.3 a) and gid 5 (V 0.075) under gid 1."""
    row2 = (a, 0.25, 0.2, 1.0 - a - 0.45)
    probs = np.array([root, row1, row2, (0.4, 0.3, 0.2, 0.1), (0.7, 0.1, 0.1, 0.1)], dtype=np.float64)
    return np.log(probs)


def _a_for(rel: float) -> float:
    """a such that log V(gid 4) = log V(gid 3) shifted by rel of |log V(gid 3)|."""
    lv3 = np.log(0.125)
    return float(np.exp(lv3 + rel * abs(lv3)) / 0.3)


def _flags(t):
    return sorted((f["kind"], f["level"], tuple(f["gids"])) for f in t["near_ties"])


def test_cross_parent_frontier_near_tie_is_flagged():
    t = oracle.build_tree(_rows(_a_for(0.5e-6)), 3, 2, 10)
    assert _flags(t) == [("frontier", 2, (4, 3))]
    t = oracle.build_tree(_rows(_a_for(-0.5e-6)), 3, 2, 10)
    assert _flags(t) == [("frontier", 2, (3, 4))]


def test_pair_outside_the_band_is_not_flagged():
    for rel in (2e-6, -2e-6, 1e-3):
        assert oracle.build_tree(_rows(_a_for(rel)), 3, 2, 10)["near_ties"] == []


def test_rerank_cut_near_tie_is_flagged():
    # kept by V: gid 0 (.5), gid 2 (.31), gid 1 (.3), then gids 4 and 3 within the band at the cut m = 4
    t = oracle.build_tree(_rows(_a_for(0.5e-6)), 3, 2, 4)
    assert _flags(t) == [("frontier", 2, (4, 3)), ("rerank", 0, (4, 3))]
    # with m = 5 both are kept and the cut is elsewhere
    assert _flags(oracle.build_tree(_rows(_a_for(0.5e-6)), 3, 2, 5)) == [("frontier", 2, (4, 3))]


def test_siblings_are_never_flagged():
    """Two children of one parent whose log V differ by 1e-7 relative: their order
    comes from their raw logits alone, which no rounding can swap, so the pair is
    not flagged at the level-1 frontier (the root's children) nor at level 2."""
    near = 0.4 * (1 - 1e-7)
    root = (0.4, near, 0.15, 1 - 0.55 - near)
    row1 = (0.45, 0.45 * (1 - 1e-7), 0.05, 0.05)
    t = oracle.build_tree(_rows(0.2, root=root, row1=row1), 3, 2, 10)
    assert t["near_ties"] == []
    # the level-1 pair does sit within the band
    assert oracle.near_tie(np.log(0.4) - np.log(sum(root)), np.log(near) - np.log(sum(root)))


def test_frontier_flip_equals_the_build_across_the_tie():
    x = _rows(_a_for(0.5e-6))
    t = oracle.build_tree(x, 3, 2, 10)
    flipped = oracle.build_tree(x, 3, 2, 10, flip=t["near_ties"])
    across = oracle.build_tree(_rows(_a_for(-0.5e-6)), 3, 2, 10)
    for f in ("tokens", "parents", "depth", "draft_row", "gid"):
        assert flipped[f].tolist() == across[f].tolist(), f
    assert flipped["parents"].tolist() != t["parents"].tolist()  # the flip changed the tree


def test_rerank_flip_equals_the_build_across_the_tie():
    x = _rows(_a_for(0.5e-6))
    t = oracle.build_tree(x, 3, 2, 4)
    rr = [f for f in t["near_ties"] if f["kind"] == "rerank"]
    flipped = oracle.build_tree(x, 3, 2, 4, flip=rr)
    assert sorted(flipped["gid"].tolist()) == [0, 1, 2, 3]
    assert sorted(t["gid"].tolist()) == [0, 1, 2, 4]


def test_tree_match_excuses_only_a_flagged_flip():
    x = _rows(_a_for(0.5e-6))
    ref = oracle.build_tree(x, 3, 2, 10)
    rebuild = lambda fl: oracle.build_tree(x, 3, 2, 10, flip=fl)
    assert tree_match(ref, ref, rebuild)[0] == 0
    alt = rebuild(ref["near_ties"])
    assert tree_match(alt, ref, rebuild)[0] == 1
    bad = {k: np.array(v, copy=True) for k, v in ref.items() if k in ("tokens", "parents", "depth", "draft_row", "gid")}
    bad["tokens"][0] = 3  # a difference on a node no flagged decision reaches
    with pytest.raises(AssertionError):
        tree_match(bad, ref, rebuild)
    clean = oracle.build_tree(_rows(_a_for(1e-3)), 3, 2, 10)
    with pytest.raises(AssertionError):  # no flag at all: nothing is excused
        tree_match(alt, clean, lambda fl: oracle.build_tree(_rows(_a_for(1e-3)), 3, 2, 10, flip=fl))


# --------------------------------------------------------- acceptance flips
def _star():
    p = np.array([0.1, 0.4, 0.3, 0.2])
    q = np.array([0.5, 0.2, 0.2, 0.1])
    target = np.log(np.stack([p, [0.25] * 4, [0.25] * 4]))
    draft = np.log(q)[None]
    return target, draft, np.array([0, 3]), np.array([0, 0]), np.array([0, -1, -1])


def test_accept_flip_equals_moving_u_across_the_ratio():
    target, draft, tokens, parents, drow = _star()
    ratio = 0.1 / 0.5  # child 1 tests token 0: p/q
    res = lambda u1, fl=(): oracle.accept_stochastic(target, draft, tokens, parents, drow,
                                                     np.array([[0, u1, 0.99], [0.3, 0.3, 0.3]]), 2, flip=set(fl))
    below, above = res(ratio * (1 - 1e-7)), res(ratio * (1 + 1e-7))
    # below the ratio child 1 is accepted; above it child 1 is rejected and child 2
    # (token 3, residual 0.25 against q 0.1) is accepted
    assert below["path"][:1] == [1] and above["path"][:1] == [2]
    assert any(t["kind"] == "accept" and t["node"] == 1 for t in below["near_ties"])
    flipped = res(ratio * (1 - 1e-7), fl=[1])
    assert (flipped["accepted_len"], flipped["path"], flipped["bonus"]) == \
        (above["accepted_len"], above["path"], above["bonus"])
    u = np.array([[0, ratio * (1 - 1e-7), 0.99], [0.3, 0.3, 0.3]])
    rewalk = lambda nodes: oracle.accept_stochastic(target, draft, tokens, parents, drow, u, 2, flip=nodes)
    assert walk_match((above["accepted_len"], above["path"], above["bonus"]), below, rewalk) == 1
    with pytest.raises(AssertionError):  # a bonus off by one token with no flagged draw
        walk_match((below["accepted_len"], below["path"], (below["bonus"] + 1) % 4), below, rewalk)


def test_inverse_cdf_band():
    w = np.array([0.25, 0.0, 0.25, 0.5])
    assert oracle.inverse_cdf(w, 0.25 * (1 + 1e-7)) == (2, True)
    assert oracle.inverse_cdf_band(w, 0.25 * (1 + 1e-7)) == [0, 2]   # the zero-weight token is never drawn
    assert oracle.inverse_cdf_band(w, 0.6) == [3]
    assert oracle.inverse_cdf_band(w, 0.5 * (1 - 1e-7)) == [2, 3]
    assert oracle.inverse_cdf(w, 0.6) == (3, False)


def test_bonus_band_is_excused_only_on_the_same_path():
    p = np.array([0.1, 0.4, 0.3, 0.2])
    q = np.array([0.5, 0.2, 0.2, 0.1])
    target = np.log(np.stack([p, [0.25] * 4]))
    draft = np.log(q)[None]
    tokens, parents, drow = np.array([0]), np.array([0]), np.array([0, -1])
    # child 1 tests token 0 (ratio 0.2) and is rejected; the bonus is drawn from
    # the residual max(0, p - q) / 0.4 = (0, 0.5, 0.25, 0.25), cumulative (0, .5, .75, 1),
    # with u_res placed just above the boundary at 0.5
    u = np.array([[0, 0.9], [0.5 * (1 + 1e-8), 0.0]])
    r = oracle.accept_stochastic(target, draft, tokens, parents, drow, u, 1)
    assert (r["accepted_len"], r["bonus"]) == (0, 2)
    band = [t for t in r["near_ties"] if t["kind"] == "bonus"]
    assert band and band[0]["alternatives"] == [1, 2]
    rewalk = lambda nodes: oracle.accept_stochastic(target, draft, tokens, parents, drow, u, 1, flip=nodes)
    assert walk_match((0, r["path"], 1), r, rewalk) == 1
    with pytest.raises(AssertionError):
        walk_match((0, r["path"], 0), r, rewalk)  # token 0 has zero residual weight: never drawn
    with pytest.raises(AssertionError):
        walk_match((1, [1], 1), r, rewalk)  # accepting child 1 is no flagged decision here
