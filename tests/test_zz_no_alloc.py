"""eagle_tree_build_noalloc: the tree build for callers that cannot allocate
device memory when they build a tree (a sealed memory pool, a plugin interface
that passes only buffers and a stream).  It takes no workspace argument and
uses a fixed scratch array inside the library instead.

Checked through the C ABI against eagle_tree_build with a caller-provided
workspace, on two calls in a row with different inputs (the shared scratch
keeps the previous call's contents, which must not leak into the result).
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import eagle_tree_verification_dynamic_b200 as et
from eagle_tree_verification_dynamic_b200 import _lib
from workloads import gen_draft_logits, get_config

pytestmark = pytest.mark.gpu


def _to_dev(stored, dtype):
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(stored)).cuda()
    return torch.from_numpy(np.ascontiguousarray(stored).view(np.int16)).cuda().view(torch.bfloat16)


def _noalloc_build(x, depth, k, m):
    B, R, V = x.shape
    tree = et.alloc_tree(B, R, depth, k, m, x.device)
    st = tree.struct()
    n = ctypes.c_int(0)
    status = et.lib().eagle_tree_build_noalloc(
        ctypes.c_void_p(x.data_ptr()), _lib._dtype_code(x), B, R, V, depth, k, m, ctypes.byref(st),
        ctypes.byref(n), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return status, n.value, tree


@pytest.mark.parametrize("name", ["l3-8b", "7b"])
def test_noalloc_build_matches_workspace_build_twice(name):
    cfg = get_config(name)
    for seed in (3, 4):  # two calls in a row, different inputs
        x = _to_dev(gen_draft_logits(cfg, seed), cfg.logits_dtype)
        ref = et.tree_build(x, cfg.depth, cfg.k, cfg.m)
        status, n, got = _noalloc_build(x, cfg.depth, cfg.k, cfg.m)
        torch.cuda.synchronize()
        assert status == 0, et.lib().eagle_status_string(status)
        assert n == ref.n
        for field in ("tokens", "parents", "depth", "gid", "draft_row"):
            assert torch.equal(getattr(got, field), getattr(ref, field)), field
        # same kernels, same order of operations: the floats agree exactly
        assert torch.equal(got.logV, ref.logV)
        assert torch.equal(got.row_lse, ref.row_lse)


def test_noalloc_build_rejects_shapes_beyond_its_scratch():
    # 4096 sequences x 41 rows of a 128k vocabulary need far more than the fixed scratch
    B, depth, k, m, V = 4096, 6, 8, 64, 128256
    R = 1 + (depth - 1) * k
    x = torch.empty(1, dtype=torch.bfloat16, device="cuda")  # never read: the call is refused first
    tree = et.alloc_tree(1, R, depth, k, m, x.device)
    st = tree.struct()
    status = et.lib().eagle_tree_build_noalloc(ctypes.c_void_p(x.data_ptr()), 1, B, R, V, depth, k, m,
                                               ctypes.byref(st), None, None)
    assert status == 4  # EAGLE_ERR_LIMIT
