"""GPU parity: KV-cache compaction after acceptance (eagle_kv_compact) against
the oracle, bit for bit (it is a copy).  Random trees and paths with the edge
cases (nothing accepted, a cache that fills up, an invalid node id ending the
copy, D = 64), and the accepted paths of real steps of two workloads.
"""
import numpy as np
import pytest
import torch

import eagle_tree_verification_dynamic_b200 as et
import oracle
from eagle_tree_verification_dynamic_b200.step import StepShape, VerifyStep
from workloads import get_config, make_target_logits, make_workload

pytestmark = pytest.mark.gpu


def _bf16(rng, shape):
    x = torch.from_numpy(rng.normal(size=shape).astype(np.float32)).to(torch.bfloat16)
    return x.cuda()


def _root_path(parents, x, depth):
    chain, node = [], x
    while node:
        chain.append(node)
        node = int(parents[node - 1])
    chain = chain[::-1][:depth]
    return chain + [-1] * (depth - len(chain))


def _check(k_tree, v_tree, path, acc, plen, k_cache, v_cache):
    k0, v0 = k_cache.clone(), v_cache.clone()
    new_len = et.kv_compact(k_tree, v_tree, path, acc, plen, k_cache, v_cache)
    torch.cuda.synchronize()
    u16 = lambda t: t.view(torch.int16).cpu().numpy()
    k_ref, v_ref, nl_ref = oracle.compact_kv(u16(k0), u16(v0), plen.cpu().numpy(), u16(k_tree), u16(v_tree),
                                             path.cpu().numpy(), acc.cpu().numpy())
    assert new_len.cpu().numpy().tolist() == nl_ref.tolist()
    np.testing.assert_array_equal(u16(k_cache), k_ref)
    np.testing.assert_array_equal(u16(v_cache), v_ref)
    return nl_ref


@pytest.mark.parametrize("D", [128, 64])
def test_random_paths_and_edge_cases(D):
    rng = np.random.default_rng(D)
    B, n, Hkv, Lmax, depth = 6, 37, 4, 300, 6
    parents = np.zeros((B, n), dtype=np.int64)
    for b in range(B):
        for i in range(n):
            parents[b, i] = rng.integers(0, i + 1)
    paths, acc = [], []
    for b in range(B):
        p = _root_path(parents[b], int(rng.integers(1, n + 1)), depth)
        paths.append(p)
        acc.append(sum(1 for v in p if v > 0))
    acc[1] = 0                                   # nothing accepted
    paths[2][1] = n + 5                          # an invalid node id ends the copy after one entry
    acc[2] = max(acc[2], 3)
    plen = [120, 50, 17, Lmax - 2, 0, 299]       # sequence 3 fills up; sequence 5 has room for one
    k_tree, v_tree = _bf16(rng, (B, n, Hkv, D)), _bf16(rng, (B, n, Hkv, D))
    k_cache, v_cache = _bf16(rng, (B, Hkv, Lmax, D)), _bf16(rng, (B, Hkv, Lmax, D))
    i32 = lambda a: torch.tensor(a, dtype=torch.int32).cuda()
    nl = _check(k_tree, v_tree, i32(paths), i32(acc), i32(plen), k_cache, v_cache)
    assert nl[1] == 50 and nl[2] == 18 and nl[3] <= Lmax and nl[5] <= Lmax


@pytest.mark.parametrize("name", ["7b", "serve"])
def test_after_a_real_step(name):
    cfg = get_config(name)
    dev = torch.device("cuda")
    w = make_workload(cfg, 2)
    tdt = torch.float32 if cfg.logits_dtype == "f32" else torch.bfloat16
    logits = (lambda a: torch.from_numpy(a).to(dev)) if cfg.logits_dtype == "f32" else \
        (lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16))
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    inp = {"draft_logits": logits(w.draft_logits), "prefix_len": torch.from_numpy(w.prefix_len).to(dev),
           "q": bf(w.q), "k_cache": bf(w.k_cache), "v_cache": bf(w.v_cache), "k_tree": bf(w.k_tree),
           "v_tree": bf(w.v_tree), "uniforms": torch.from_numpy(w.uniforms).to(dev)}
    shape = StepShape(B=cfg.B, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, Lmax=cfg.L, depth=cfg.depth, k=cfg.k, m=cfg.m,
                      V=cfg.V, logits_dtype=tdt, window=cfg.window, stochastic=True)
    st = VerifyStep(shape, dev)
    st.build(inp["draft_logits"])
    torch.cuda.synchronize()
    inp["target_logits"] = logits(make_target_logits(cfg, 2, w.draft_logits, st.tree.draft_row.cpu().numpy()))
    st.fused(inp)
    torch.cuda.synchronize()
    # a cache with room past every prefix (the workloads fill the cache to Lmax)
    Lmax = cfg.L + cfg.depth
    pad = lambda t: torch.cat([t, torch.zeros_like(t[:, :, :cfg.depth])], dim=2).contiguous()
    k_cache, v_cache = pad(inp["k_cache"]), pad(inp["v_cache"])
    assert k_cache.shape[2] == Lmax
    _check(inp["k_tree"], inp["v_tree"], st.path, st.accepted_len, inp["prefix_len"], k_cache, v_cache)
