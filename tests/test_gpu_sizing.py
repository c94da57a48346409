"""GPU: cost-aware sizing end to end.  The grower's per-level gains against the
oracle's (relative 1e-5: log V carries the rows' log-sum-exps, each within
5e-7 of fp64), the harness's decisions against the oracle's policy on the
oracle's gains (unless a ratio lies within 1e-4 of the threshold), and the tree
of the levels kept against the oracle's tree of the levels drafted (bit-exact
outside flagged near-ties).
"""
import numpy as np
import pytest
import torch

import eagle_tree_verification_dynamic_b200 as et
import oracle
from eagle_tree_verification_dynamic_b200.sizing import CostTable, grow_sized
from workloads import gen_draft_logits, get_config

from gpu_helpers import to_dev_logits, tree_of
from parity import tree_match

pytestmark = pytest.mark.gpu


def _linear_table():
    """20 + 0.5 B N (microseconds): each level costs 0.5 B k."""
    Bs, Ls, Ns = [1, 64], [128, 65536], [0, 256]
    us = np.array([[[20 + 0.5 * b * n for n in Ns] for _ in Ls] for b in Bs])
    return CostTable(Bs, Ls, Ns, us)


@pytest.mark.parametrize("name", ["7b", "serve", "l3-8b"])
@pytest.mark.parametrize("threshold", [0.0, 0.001, 0.02, 1.0])
def test_sized_growth_matches_the_oracle(name, threshold):
    cfg = get_config(name)
    stored = gen_draft_logits(cfg, 3)
    x = to_dev_logits(stored, cfg.logits_dtype)
    k = cfg.k
    table = _linear_table()
    grower = et.TreeGrower(cfg.B, cfg.V, cfg.depth, k, x.dtype, x.device)
    seen = []

    def draft_fn(level, tok, par):
        return x[:, 1 + (level - 2) * k: 1 + (level - 1) * k].contiguous()

    gains_gpu = []
    orig_gains = grower.gains

    def gains():
        g = orig_gains()
        gains_gpu.append(g.cpu().numpy().copy())
        return g
    grower.gains = gains
    r = grow_sized(grower, x[:, 0].contiguous(), draft_fn, table, float(cfg.L), threshold)
    torch.cuda.synchronize()
    x64 = oracle.decode_logits(stored, cfg.logits_dtype)
    full = [oracle.build_tree(x64[b], cfg.depth, k, cfg.m) for b in range(cfg.B)]
    for lvl, g in enumerate(gains_gpu):
        np.testing.assert_allclose(g, [t["gains"][lvl] for t in full], rtol=1e-5)
    gl = [[t["gains"][l] for t in full] for l in range(cfg.depth)]
    tab = (table.B, table.L, table.N, table.us)
    kept = oracle.levels_kept(tab, cfg.B, float(cfg.L), k, gl, threshold)
    for l in range(min(kept + 1, cfg.depth)):
        rho = oracle.level_ratio(tab, cfg.B, float(cfg.L), k, l + 1, gl[l])
        if abs(rho - threshold) <= 1e-4 * max(threshold, 1e-12):
            pytest.skip(f"level {l + 1}: ratio {rho} within 1e-4 of the threshold")
    drafted = min(kept + 1, cfg.depth)
    assert (r.levels_kept, r.levels_drafted) == (kept, drafted)
    if kept == 0:
        assert r.tree is None
        return
    m = min(k * kept, 128)
    R = 1 + (drafted - 1) * k
    excused = 0
    for b in range(cfg.B):
        ref = oracle.build_tree(x64[b][:R], drafted, k, m)
        got = tree_of(r.tree, b)
        got["row_lse"] = got["row_lse"][:R]
        excused += tree_match(got, ref, lambda fl, b=b: oracle.build_tree(x64[b][:R], drafted, k, m, flip=fl))[0]
        np.testing.assert_allclose(got["row_lse"], ref["row_lse"], rtol=0, atol=5e-7)
    assert excused <= 1, (name, threshold)


@pytest.mark.parametrize("B,threshold", [(1, 0.5), (32, 0.5), (8, 0.3), (32, 0.05)])
def test_widening_harness_matches_the_oracle(B, threshold):
    """grow_widths (the library's width decision between draft levels, each level drafted from the chosen
    nodes only) against the same harness on the oracle: the widths level by level and the tree of the
    chosen candidates.  At batch 1 on the saturating table every level keeps its full width; at batch 32
    with threshold 0.5 the tree is a chain."""
    from eagle_tree_verification_dynamic_b200.sizing import grow_widths
    from sizing_helpers import _masked, confident_draft, oracle_grow_widths, saturating_table

    cfg, stored = confident_draft()
    stored = stored[:B]
    x64 = oracle.decode_logits(stored, "f32")
    table = CostTable(*saturating_table())
    xd = torch.from_numpy(stored).cuda()
    g = et.TreeGrower(B, cfg.V, cfg.depth, cfg.k, torch.float32, "cuda")

    def draft_fn(level, tok, par, width):  # the rows the draft model gives the chosen frontier slots
        r0 = 1 + (level - 2) * cfg.k
        return xd[:, r0:r0 + width].contiguous()

    res = grow_widths(g, xd[:, 0].contiguous(), draft_fn, table, 2048, threshold)
    torch.cuda.synchronize()
    want_w, trees = oracle_grow_widths(list(x64), cfg.depth, cfg.k, (table.B, table.L, table.N, table.us), 2048,
                                       threshold)
    assert res.widths == want_w
    if B == 1:
        assert want_w == [cfg.k] * cfg.depth
    if B == 32 and threshold == 0.5:
        assert want_w == [1] * cfg.depth
    R = 1 + (len(want_w) - 1) * cfg.k
    excused = 0
    for b in range(B):
        rows = _masked(x64[b][:R], cfg.k, want_w)
        e, ref = tree_match(tree_of(res.tree, b), trees[b],
                            lambda fl, rows=rows: oracle.build_tree(rows, len(want_w), cfg.k, 1, widths=want_w,
                                                                    flip=fl))
        excused += e
    assert excused <= 1
