"""The library's cost-aware sizing (host functions of the C ABI) against the
oracle, and the harness loop of ``sizing.grow_sized`` with a stand-in grower.
No GPU: eagle_cost_at and eagle_size_keep_level touch no device memory.
"""
import numpy as np
import pytest
import torch

import oracle
from eagle_tree_verification_dynamic_b200.sizing import CostTable, grow_sized


def _random_table(rng):
    grid = lambda n, lo, hi: np.sort(rng.choice(np.arange(lo, hi), size=n, replace=False)).astype(np.float64)
    Bs, Ls, Ns = grid(int(rng.integers(1, 5)), 1, 65), grid(int(rng.integers(1, 4)), 128, 32769), \
        grid(int(rng.integers(1, 7)), 0, 161)
    us = rng.uniform(5.0, 500.0, size=(Bs.size, Ls.size, Ns.size))
    return CostTable(Bs, Ls, Ns, us)


def test_cost_matches_the_oracle():
    rng = np.random.default_rng(0)
    for _ in range(200):
        t = _random_table(rng)
        for _ in range(10):
            B, L, N = rng.uniform(0, 80), rng.uniform(0, 40000), rng.uniform(-10, 200)
            want = oracle.cost_at(t.B, t.L, t.N, t.us, B, L, N)
            assert t.at(B, L, N) == pytest.approx(want, rel=1e-12, abs=1e-9)


def test_decisions_match_the_oracle():
    rng = np.random.default_rng(1)
    agree = 0
    for _ in range(300):
        t = _random_table(rng)
        B, L, k, level = int(rng.integers(1, 33)), float(rng.uniform(100, 30000)), int(rng.integers(1, 11)), \
            int(rng.integers(1, 9))
        gains = rng.uniform(0, 1, size=B) * 0.8 ** level
        thr = float(rng.uniform(0, 0.1))
        keep, ratio = t.keep_level(B, L, k, level, gains, thr)
        want_ratio = oracle.level_ratio((t.B, t.L, t.N, t.us), B, L, k, level, gains)
        if np.isinf(want_ratio):
            assert np.isinf(ratio)
        else:
            assert ratio == pytest.approx(want_ratio, rel=1e-12)
        if abs(want_ratio - thr) > 1e-9 * max(1.0, abs(thr)):
            assert keep == oracle.keep_level((t.B, t.L, t.N, t.us), B, L, k, level, gains, thr)
            agree += 1
    assert agree > 250


def test_invalid_tables_and_arguments():
    good = CostTable([1, 2], [100, 200], [0, 10], np.ones((2, 2, 2)))
    assert np.isnan(CostTable([2, 1], [100, 200], [0, 10], np.ones((2, 2, 2))).at(1, 1, 1))   # descending
    assert np.isnan(CostTable([1, 2], [100, 200], [0, 10], np.full((2, 2, 2), np.inf)).at(1, 1, 1))
    with pytest.raises(Exception):
        good.keep_level(1, 100, 0, 1, [0.5], 0.1)          # k = 0
    with pytest.raises(ValueError):
        CostTable([1, 2], [100], [0, 10], np.ones((2, 2, 2)))


class _FakeGrower:
    """Stand-in for TreeGrower: fixed per-level gains, records the calls."""

    def __init__(self, gains_by_level, B=2, k=4, depth=6):
        self.g, self.B, self.k, self.depth, self.calls = gains_by_level, B, k, depth, []
        self.cur = 0

    def begin(self, root):
        self.cur = 1
        self.calls.append(("begin",))
        return torch.zeros(self.B, self.k), torch.zeros(self.B, self.k)

    def level(self, rows, level):
        self.cur = level
        self.calls.append(("level", level))
        return torch.zeros(self.B, self.k), torch.zeros(self.B, self.k)

    def gains(self):
        return torch.tensor(self.g[self.cur - 1], dtype=torch.float64)

    def finish(self, m, levels):
        self.calls.append(("finish", m, levels))
        return "tree"


def test_harness_stops_at_the_first_level_that_does_not_pay():
    table = CostTable([1, 2], [100, 200], [0, 100], np.array([[[10.0, 210.0]] * 2] * 2))   # 8 per level of 4
    gains = [[0.9, 0.9], [0.5, 0.5], [0.2, 0.1], [0.05, 0.05], [0.01, 0.0], [0.0, 0.0]]
    drafted = []
    fg = _FakeGrower(gains)
    r = grow_sized(fg, None, lambda lvl, t, p: drafted.append(lvl) or None, table, 150, 0.1)
    assert (r.levels_kept, r.levels_drafted, r.tree) == (2, 3, "tree")
    assert drafted == [2, 3] and fg.calls[-1] == ("finish", 8, 3)
    assert r.ratios == pytest.approx([1.8 / 8, 1.0 / 8, 0.3 / 8])
    fg = _FakeGrower(gains)
    r = grow_sized(fg, None, lambda *a: None, table, 150, 0.0)
    assert (r.levels_kept, r.levels_drafted) == (6, 6) and fg.calls[-1] == ("finish", 24, 6)
    fg = _FakeGrower(gains)
    r = grow_sized(fg, None, lambda *a: None, table, 150, 0.5)
    assert (r.levels_kept, r.levels_drafted, r.tree) == (0, 1, None)


def test_the_shipped_b200_table():
    from eagle_tree_verification_dynamic_b200.sizing import default_table
    t = default_table()
    assert t.us.shape == (t.B.size, t.L.size, t.N.size) and np.all(np.isfinite(t.us))
    for i, j, l in [(0, 0, 1), (3, 2, 6), (1, 1, 3)]:
        assert t.at(t.B[i], t.L[j], t.N[l]) == pytest.approx(t.us[i, j, l], rel=1e-12)
    assert np.all(t.us[:, :, 0] == 0.0) and np.all(t.us[:, :, 1:] > 0.0)
    # verification grows with the batch's work: the largest grid point costs the most
    assert t.us[-1, -1, -1] == t.us.max()


def test_level_widths_match_the_oracle():
    rng = np.random.default_rng(5)
    checked = 0
    for _ in range(300):
        t = _random_table(rng)
        B, L, k = int(rng.integers(1, 33)), float(rng.uniform(100, 30000)), int(rng.integers(1, 11))
        n_before = int(rng.integers(0, 40))
        v = np.sort(rng.uniform(0, 1, size=(B, k)) ** 3, axis=1)[:, ::-1]
        v[:, k - int(rng.integers(0, k)):] = 0.0 if rng.random() < 0.3 else v[:, k - 1:k].min()
        with np.errstate(divide="ignore"):
            logv = np.log(v)  # -inf for V = 0
        thr = float(rng.uniform(0, 0.05))
        w, ratios = t.level_width(B, L, n_before, logv, thr)
        want_w, want_r = oracle.level_width((t.B, t.L, t.N, t.us), B, L, n_before, np.exp(logv), thr)
        near = any(abs(r - thr) <= 1e-9 * max(1.0, abs(thr)) for r in want_r if np.isfinite(r))
        if not near:
            assert w == want_w
            checked += 1
        for j, r in enumerate(want_r):
            if np.isinf(r):
                assert np.isinf(ratios[j])
            else:
                assert ratios[j] == pytest.approx(r, rel=1e-12, abs=1e-300)
    assert checked > 250


def test_the_shipped_tables_by_shape():
    from eagle_tree_verification_dynamic_b200.sizing import table_for
    for shape in [(32, 8, 128, 128256, "bf16"), (32, 32, 128, 32000, "f32")]:
        t = table_for(*shape)
        assert t.us.shape == (t.B.size, t.L.size, t.N.size) and np.all(np.isfinite(t.us))
        assert np.all(t.us[:, :, 0] == 0.0) and np.all(t.us[:, :, 1:] > 0.0)
        # more candidates never cost less at the largest batch and context
        assert np.all(np.diff(t.us[-1, -1, :]) >= -0.05 * t.us[-1, -1, 1:])
    with pytest.raises(FileNotFoundError):
        table_for(7, 7, 64, 1000, "f32")
