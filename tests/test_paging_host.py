"""Host helpers around the paged cache and the calibration (no GPU): bench.py's
page_caches lays a dense cache into a shuffled pool that the oracle's
gather_pages reads back unchanged (every sequence, with room past its end), and
the calibration's tree template is a complete 4-ary tree within the walk's
depth limit.
"""
import os
import sys

import numpy as np
import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("ps", [16, 32, 64, 192])
def test_bench_paging_round_trip(ps):
    sys.path.insert(0, ROOT)
    import bench
    g = torch.Generator().manual_seed(ps)
    kc = torch.randn(3, 2, 150, 8, generator=g)
    vc = torch.randn(3, 2, 150, 8, generator=g)
    kp, vp, table = bench.page_caches(torch, kc, vc, ps, 6, seed=1)
    assert table.shape == (3, (150 + 6 + ps - 1) // ps) and table.dtype == torch.int32
    assert sorted(table.flatten().tolist()) == list(range(table.numel()))      # every page used once
    for b in range(3):
        np.testing.assert_array_equal(oracle.gather_pages(kp.numpy(), table[b].numpy(), 150), kc[b].numpy())
        np.testing.assert_array_equal(oracle.gather_pages(vp.numpy(), table[b].numpy(), 150), vc[b].numpy())


def test_calibration_tree_template():
    from eagle_tree_verification_dynamic_b200.calibrate import _tree
    for n in (1, 8, 64, 128):
        par, dep = _tree(n, None)
        assert all(0 <= par[j] <= j for j in range(n))
        assert dep.max() <= 5 and np.bincount(par, minlength=n + 1).max() <= 4
