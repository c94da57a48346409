"""GPU parity: the tree grown one level at a time (eagle_tree_grow_begin /
_level / _finish).

On the same draft rows the grown tree equals eagle_tree_build bit for bit
(tokens, parents, depth, candidate ids, draft rows, and the fp32 log V and fp64
log-sum-exp bits), and each level's frontier equals the oracle's (tokens and
parent slots, bit-exact; where the oracle flags a near-tie, equal to the
oracle's frontiers with that decision resolved the other way, as tests/parity.py
allows for the tree).  A
lazy draft model, whose rows depend on the frontier tokens it is handed, gives
the oracle's tree on the rows it produced.
"""
import numpy as np
import pytest
import torch

import eagle_tree_verification_dynamic_b200 as et
import oracle
from workloads import gen_draft_logits, get_config

from gpu_helpers import to_dev_logits, tree_of, trees_equal
from parity import tree_match

pytestmark = pytest.mark.gpu


def _grow(logits: torch.Tensor, depth: int, k: int, m: int):
    """Feed the one-shot layout's rows level by level; returns the tree and each level's frontier."""
    B, R, V = logits.shape
    g = et.TreeGrower(B, V, depth, k, logits.dtype, logits.device)
    fronts, gains = [], []
    tok, par = g.begin(logits[:, 0].contiguous())
    gains.append(g.gains().clone())
    if depth > 1:
        fronts.append((tok.clone(), par.clone()))
    for level in range(2, depth + 1):
        rows = logits[:, 1 + (level - 2) * k: 1 + (level - 1) * k].contiguous()
        tok, par = g.level(rows, level)
        gains.append(g.gains().clone())
        if level < depth:
            fronts.append((tok.clone(), par.clone()))
    _grow.gains = gains
    return g.finish(m), fronts


def _same_bits(a: torch.Tensor, b: torch.Tensor):
    assert a.shape == b.shape and a.dtype == b.dtype
    assert torch.equal(a.cpu().view(torch.uint8), b.cpu().view(torch.uint8))


@pytest.mark.parametrize("name", ["tiny", "7b", "l3-8b", "serve"])
def test_grown_tree_equals_one_shot_build(name):
    cfg = get_config(name)
    stored = gen_draft_logits(cfg, 3)
    x = to_dev_logits(stored, cfg.logits_dtype)
    one = et.tree_build(x, cfg.depth, cfg.k, cfg.m)
    grown, fronts = _grow(x, cfg.depth, cfg.k, cfg.m)
    torch.cuda.synchronize()
    assert grown.n == one.n
    for f in ("tokens", "parents", "depth", "gid", "draft_row", "logV", "row_lse"):
        _same_bits(getattr(grown, f), getattr(one, f))
    x64 = oracle.decode_logits(stored, cfg.logits_dtype)
    excused = 0
    for b in range(cfg.B):
        ref = oracle.build_tree(x64[b], cfg.depth, cfg.k, cfg.m)
        e, ref = tree_match(tree_of(grown, b), ref,
                            lambda fl, b=b: oracle.build_tree(x64[b], cfg.depth, cfg.k, cfg.m, flip=fl))
        excused += e
        # log V carries the rows' log-sum-exps (fp32 exponentials, within 5e-7 each): 1e-5 relative
        np.testing.assert_allclose([float(g[b]) for g in _grow.gains], ref["gains"], rtol=1e-5)
        for lvl, (tok, par) in enumerate(fronts, start=1):
            assert tok[b].cpu().numpy().tolist() == ref["frontiers"][lvl - 1]["tokens"].tolist(), (b, lvl)
            assert par[b].cpu().numpy().tolist() == ref["frontiers"][lvl - 1]["parent_slot"].tolist(), (b, lvl)
    assert excused <= 1


@pytest.mark.parametrize("depth,k,m,V,dtype", [(1, 4, 4, 50, "bf16"), (4, 1, 4, 300, "f32"), (2, 32, 128, 5000, "bf16"),
                                               (16, 2, 64, 64, "f32"), (3, 3, 100, 200, "bf16")])
def test_grown_tree_edge_shapes(depth, k, m, V, dtype):
    cfg = get_config("tiny", depth=depth, k=k, m=m, V=V, B=3, logits_dtype=dtype)
    x = to_dev_logits(gen_draft_logits(cfg, 7), dtype)
    one = et.tree_build(x, depth, k, m)
    grown, _ = _grow(x, depth, k, m)
    torch.cuda.synchronize()
    for f in ("tokens", "parents", "depth", "gid", "draft_row", "logV", "row_lse"):
        _same_bits(getattr(grown, f), getattr(one, f))


def test_lazy_draft_model():
    """Rows made only once the frontier is known: each row is a seeded function
    of the token path that leads to it, so no row can be prepared in advance."""
    B, V, depth, k, m = 3, 1000, 5, 4, 40
    dev = torch.device("cuda:0")

    def row_for(path):
        seed = int(np.uint64(1469598103934665603) ^ np.uint64(hash(tuple(path)) & 0xFFFFFFFF))
        return np.random.default_rng(seed).normal(scale=3.0, size=V).astype(np.float32)

    g = et.TreeGrower(B, V, depth, k, torch.float32, dev)
    used = np.zeros((B, 1 + (depth - 1) * k, V), dtype=np.float32)
    paths = [[[-1]] for _ in range(B)]                 # the token path of each frontier slot
    for b in range(B):
        used[b, 0] = row_for((b, -1))
    tok, par = g.begin(torch.from_numpy(used[:, 0]).to(dev))
    for level in range(2, depth + 1):
        tok_h, par_h = tok.cpu().numpy(), par.cpu().numpy()
        new_paths, rows = [], np.zeros((B, k, V), dtype=np.float32)
        for b in range(B):
            prev = paths[b]
            cur = [(prev[0] if level == 2 else prev[par_h[b, s]]) + [int(tok_h[b, s])] for s in range(k)]
            new_paths.append(cur)
            for s in range(k):
                rows[b, s] = row_for((b,) + tuple(cur[s]))
        paths = new_paths
        used[:, 1 + (level - 2) * k: 1 + (level - 1) * k] = rows
        tok, par = g.level(torch.from_numpy(rows).to(dev), level)
    tree = g.finish(m)
    torch.cuda.synchronize()
    for b in range(B):
        ref = oracle.build_tree(used[b].astype(np.float64), depth, k, m)
        assert not ref["near_ties"]
        got = tree_of(tree, b)
        assert trees_equal(got, ref)
        np.testing.assert_allclose(got["logV"], ref["logV"], rtol=0, atol=2e-6)
