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
