"""GPU parity: tree-masked split-KV attention against the fp64 oracle with an
explicit dense mask.

Small shapes are compared element by element (several key tiles, ragged tails,
GQA, a sliding window, a batch of ragged prefix lengths).  The full-size
shapes of the five workloads are compared on sampled (node, head) rows, which
the oracle computes one by one.  Tolerance: see gpu_helpers.check_attention.
"""
import numpy as np
import pytest
import torch

import eagle_tree_verification_dynamic_b200 as et
import oracle
from workloads import gen_attention_inputs, gen_draft_logits, gen_prefix_len, get_config

from gpu_helpers import attention_ref, check_attention, dec, i32, to_dev_bf16, to_dev_logits, tree_of

pytestmark = pytest.mark.gpu


def _random_tree(rng, n, max_depth):
    parents = np.zeros(n, dtype=np.int64)
    depth = np.zeros(n, dtype=np.int64)
    for i in range(n):
        cands = [0] + [j + 1 for j in range(i) if depth[j] < max_depth]
        parents[i] = cands[rng.integers(0, len(cands))]
        depth[i] = 1 if parents[i] == 0 else depth[parents[i] - 1] + 1
    return parents, depth


def _run(B, n, Hq, Hkv, D, Lmax, plen, window, seed, parents_b, depth_b):
    cfg = get_config("tiny", B=B, m=n, Hq=Hq, Hkv=Hkv, D=D, L=Lmax)
    q, kc, vc, kt, vt = gen_attention_inputs(cfg, seed, Lmax)
    par = np.stack(parents_b)
    dep = np.stack(depth_b)
    mask, pos = et.tree_mask(i32(par), i32(dep), i32(plen))
    out = et.tree_attention(to_dev_bf16(q), to_dev_bf16(kc), to_dev_bf16(vc), i32(plen), to_dev_bf16(kt),
                            to_dev_bf16(vt), mask, pos, window=window)
    out = out.float().cpu().numpy()
    for b in range(B):
        ref, s = attention_ref(dec(q[b]), dec(kc[b]), dec(vc[b]), int(plen[b]), dec(kt[b]), dec(vt[b]),
                               par[b], dep[b], window=window)
        check_attention(out[b], ref, s)


@pytest.mark.parametrize("B,n,Hq,Hkv,D,Lmax,window", [
    (1, 10, 4, 4, 64, 128, 0),      # the tiny workload's shape
    (2, 37, 8, 2, 128, 700, 0),     # GQA, ragged tile tail, several splits
    (1, 1, 4, 4, 128, 333, 0),      # one-node tree = decode attention
    (3, 64, 4, 1, 64, 1029, 0),     # n = 64 (mask word boundary), MQA
    (1, 100, 2, 2, 128, 96, 0),     # n > 64 uses the second mask word
    (1, 20, 8, 4, 128, 2000, 300),  # sliding window
    (2, 9, 4, 4, 64, 50, 8),        # window shorter than the tree depth
    (1, 37, 12, 2, 128, 700, 0),    # G = 6 does not divide 128: the producer warp gathers Q; 2 row groups
    (2, 60, 40, 8, 128, 500, 0),    # G = 5, three row groups per KV head, the last one ragged
    (1, 21, 6, 2, 64, 300, 40),     # G = 3 at D = 64, with a window
])
def test_attention_small(B, n, Hq, Hkv, D, Lmax, window):
    rng = np.random.default_rng(n * 7 + Lmax)
    trees = [_random_tree(rng, n, 6) for _ in range(B)]
    plen = np.array([Lmax - 3 * b for b in range(B)], dtype=np.int32)
    _run(B, n, Hq, Hkv, D, Lmax, plen, window, seed=n, parents_b=[t[0] for t in trees],
         depth_b=[t[1] for t in trees])


def test_attention_ragged_batch_and_empty_prefix():
    rng = np.random.default_rng(77)
    B, n = 5, 12
    plen = np.array([0, 1, 63, 64, 257], dtype=np.int32)
    trees = [_random_tree(rng, n, 4) for _ in range(B)]
    _run(B, n, 8, 2, 128, 300, plen, 0, seed=3, parents_b=[t[0] for t in trees], depth_b=[t[1] for t in trees])


def test_prefix_lengths_outside_the_cache_are_clamped():
    """prefix_len is device data the host cannot check: the kernel clamps it to
    [0, Lmax], so -7 behaves as 0 and Lmax + 50 as Lmax, bit for bit."""
    rng = np.random.default_rng(5)
    B, n, Lmax = 3, 12, 200
    trees = [_random_tree(rng, n, 4) for _ in range(B)]
    par, dep = np.stack([t[0] for t in trees]), np.stack([t[1] for t in trees])
    cfg = get_config("tiny", B=B, m=n, Hq=8, Hkv=2, D=128, L=Lmax)
    q, kc, vc, kt, vt = (to_dev_bf16(a) for a in gen_attention_inputs(cfg, 4, Lmax))

    def run(plen):
        pl = i32(np.array(plen, dtype=np.int32))
        mask, pos = et.tree_mask(i32(par), i32(dep), pl)
        return et.tree_attention(q, kc, vc, pl, kt, vt, mask, pos)
    a, b = run([-7, Lmax + 50, Lmax]), run([0, Lmax, Lmax])
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_attention_chain_equals_causal():
    n, L = 16, 500
    par = np.arange(n)
    dep = np.arange(1, n + 1)
    _run(1, n, 4, 4, 128, L, np.array([L], dtype=np.int32), 0, seed=8, parents_b=[par], depth_b=[dep])


@pytest.mark.parametrize("name", ["7b", "l3-8b", "long", "long-window", "serve"])
def test_attention_full_size_sampled(name):
    cfg = get_config(name)
    stored = gen_draft_logits(cfg, 0)
    tree = et.tree_build(to_dev_logits(stored, cfg.logits_dtype), cfg.depth, cfg.k, cfg.m)
    plen = gen_prefix_len(cfg, 0)
    q, kc, vc, kt, vt = gen_attention_inputs(cfg, 0, cfg.L)
    mask, pos = et.tree_mask(tree.parents, tree.depth, i32(plen))
    out = et.tree_attention(to_dev_bf16(q), to_dev_bf16(kc), to_dev_bf16(vc), i32(plen), to_dev_bf16(kt),
                            to_dev_bf16(vt), mask, pos, window=cfg.window)
    out = out.float().cpu().numpy()
    rng = np.random.default_rng(1)
    for b in sorted(set(rng.integers(0, cfg.B, size=min(cfg.B, 4)).tolist())):
        t = tree_of(tree, b)
        rows = [(int(i), int(h)) for i, h in zip(rng.integers(0, cfg.m, 12), rng.integers(0, cfg.Hq, 12))]
        rows += [(cfg.m - 1, cfg.Hq - 1), (0, 0)]
        ref, s = attention_ref(dec(q[b]), dec(kc[b]), dec(vc[b]), int(plen[b]), dec(kt[b]), dec(vt[b]),
                               t["parents"], t["depth"], window=cfg.window, rows=rows)
        got = np.array([out[b, i, h] for i, h in rows])
        check_attention(got, ref, s)


def test_a_wait_that_runs_out_reports_status_1_and_the_next_call_is_clean():
    """The failure path of the bounded waits: with the wait probe on, every CTA's
    softmax warps wait 1 ms on a barrier nothing completes, give up, and the CTA
    aborts (the other roles stop, copies and MMAs in flight drain, TMEM is
    freed); the status word reads 1.  With the probe off again the same call
    returns status 0 and the same output as before, bit for bit."""
    rng = np.random.default_rng(31)
    B, n, Hq, Hkv, D, Lmax = 2, 30, 8, 2, 128, 1500
    trees = [_random_tree(rng, n, 5) for _ in range(B)]
    par, dep = np.stack([t[0] for t in trees]), np.stack([t[1] for t in trees])
    cfg = get_config("tiny", B=B, m=n, Hq=Hq, Hkv=Hkv, D=D, L=Lmax)
    q, kc, vc, kt, vt = (to_dev_bf16(a) for a in gen_attention_inputs(cfg, 12, Lmax))
    plen = i32(np.array([Lmax, Lmax - 77], dtype=np.int32))
    mask, pos = et.tree_mask(i32(par), i32(dep), plen)
    good = et.tree_attention(q, kc, vc, plen, kt, vt, mask, pos)
    try:
        et.attention_wait_probe(1_000_000)
        with pytest.raises(et.EagleError, match="device status 1"):
            et.tree_attention(q, kc, vc, plen, kt, vt, mask, pos)
    finally:
        et.attention_wait_probe(0)
    again = et.tree_attention(q, kc, vc, plen, kt, vt, mask, pos)
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), good.view(torch.int16))
