"""GPU parity: tree attention and KV compaction over a paged prefix cache.

Without a window the paged kernel visits the same 64-key tiles in the same
order as the dense one, so its output must equal the dense kernel's bit for bit
on the same logical cache (every page size, ragged lengths, shuffled pools,
unallocated table entries past each length).  With a window the first tile
starts at a 64-key boundary, so sums run in another order: checked against the
oracle on sampled rows.  A missing page for a key in use reports device status
3; compaction into pages equals the oracle bit for bit; the whole step on a
paged cache equals the step on the dense cache.
"""
import numpy as np
import pytest
import torch

import eagle_tree_verification_dynamic_b200 as et
import oracle
from eagle_tree_verification_dynamic_b200.step import StepShape, VerifyStep
from workloads import gen_attention_inputs, gen_draft_logits, gen_prefix_len, get_config, make_target_logits, \
    make_workload

from workloads.gen import bf16_bits_from_f32

from gpu_helpers import attention_ref, check_attention, dec, i32, to_dev_bf16, to_dev_logits

pytestmark = pytest.mark.gpu


def _page(cache: torch.Tensor, plen: torch.Tensor, ps: int, seed: int, spare: int = 7):
    """dense [B][Hkv][Lmax][D] -> (pool [num_pages][Hkv][ps][D], table [B][pps]); the pages of all
    sequences shuffled through the pool, entries past each sequence's length set to -1."""
    B, Hkv, Lmax, D = cache.shape
    pps = (Lmax + ps - 1) // ps
    pad = torch.zeros(B, Hkv, pps * ps, D, dtype=cache.dtype, device=cache.device)
    pad[:, :, :Lmax] = cache
    pages = pad.view(B, Hkv, pps, ps, D).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv, ps, D)
    g = torch.Generator().manual_seed(seed)
    num_pages = B * pps + spare
    perm = torch.randperm(num_pages, generator=g)[:B * pps].to(cache.device)
    pool = torch.randn(num_pages, Hkv, ps, D, dtype=torch.float32, device=cache.device).to(cache.dtype)
    pool[perm] = pages
    table = perm.view(B, pps).to(torch.int32).clone()
    used = (plen.to(torch.int64) + ps - 1) // ps
    table[torch.arange(pps, device=cache.device)[None, :] >= used[:, None]] = -1
    return pool.contiguous(), table.contiguous()


def _inputs(cfg, seed=0):
    stored = gen_draft_logits(cfg, seed)
    tree = et.tree_build(to_dev_logits(stored, cfg.logits_dtype), cfg.depth, cfg.k, cfg.m)
    plen = gen_prefix_len(cfg, seed)
    q, kc, vc, kt, vt = gen_attention_inputs(cfg, seed, cfg.L)
    mask, pos = et.tree_mask(tree.parents, tree.depth, i32(plen))
    return tree, plen, [to_dev_bf16(a) for a in (q, kc, vc, kt, vt)], mask, pos, (q, kc, vc, kt, vt)


@pytest.mark.parametrize("name,ps", [("serve", 16), ("serve", 64), ("serve", 256), ("7b", 32), ("7b", 128),
                                     ("l3-8b", 64), ("tiny", 16), ("tiny", 32)])
def test_paged_equals_dense_bit_for_bit(name, ps):
    cfg = get_config(name)
    tree, plen, (q, kc, vc, kt, vt), mask, pos, _ = _inputs(cfg)
    pl = i32(plen)
    dense = et.tree_attention(q, kc, vc, pl, kt, vt, mask, pos)
    kp, table = _page(kc, pl, ps, 1)
    vp, _ = _page(vc, pl, ps, 1)
    paged = et.tree_attention_paged(q, kp, vp, table, pl, kt, vt, mask, pos)
    torch.cuda.synchronize()
    assert torch.equal(paged.view(torch.int16), dense.view(torch.int16))


@pytest.mark.parametrize("ps", [16, 64, 128])
def test_paged_window_against_the_oracle(ps):
    cfg = get_config("serve", B=6, window=700)       # ragged prefixes, some shorter than the window
    tree, plen, (q, kc, vc, kt, vt), mask, pos, host = _inputs(cfg, 2)
    pl = i32(plen)
    kp, table = _page(kc, pl, ps, 3)
    vp, _ = _page(vc, pl, ps, 3)
    out = et.tree_attention_paged(q, kp, vp, table, pl, kt, vt, mask, pos, window=cfg.window).float().cpu().numpy()
    qh, kch, vch, kth, vth = host
    rng = np.random.default_rng(4)
    for b in range(cfg.B):
        par, dep = tree.parents[b].cpu().numpy(), tree.depth[b].cpu().numpy()
        rows = [(int(i), int(h)) for i, h in zip(rng.integers(0, tree.n, 10), rng.integers(0, cfg.Hq, 10))]
        rows += [(0, 0), (tree.n - 1, cfg.Hq - 1)]
        ref, s = attention_ref(dec(qh[b]), dec(kch[b]), dec(vch[b]), int(plen[b]), dec(kth[b]), dec(vth[b]),
                               par, dep, window=cfg.window, rows=rows)
        check_attention(np.array([out[b, i, h] for i, h in rows]), ref, s)


def test_missing_page_reports_status_3():
    cfg = get_config("serve", B=4)
    tree, plen, (q, kc, vc, kt, vt), mask, pos, _ = _inputs(cfg)
    pl = i32(plen)
    kp, table = _page(kc, pl, 64, 5)
    vp, _ = _page(vc, pl, 64, 5)
    et.tree_attention_paged(q, kp, vp, table, pl, kt, vt, mask, pos)       # every needed page present: status 0
    table[2, 3] = -1                                                         # a page inside sequence 2's prefix
    with pytest.raises(et.EagleError, match="status 3"):
        et.tree_attention_paged(q, kp, vp, table, pl, kt, vt, mask, pos)
    table[2, 3] = kp.shape[0] + 10                                           # past the pool
    with pytest.raises(et.EagleError, match="status 3"):
        et.tree_attention_paged(q, kp, vp, table, pl, kt, vt, mask, pos)


@pytest.mark.parametrize("ps", [16, 64])
def test_kv_compact_paged_against_the_oracle(ps):
    rng = np.random.default_rng(ps)
    B, n, Hkv, D, depth, Lmax = 5, 37, 4, 128, 6, 320
    kt = to_dev_bf16(bf16_bits_from_f32(rng.normal(size=(B, n, Hkv, D)).astype(np.float32)))
    vt = to_dev_bf16(bf16_bits_from_f32(rng.normal(size=(B, n, Hkv, D)).astype(np.float32)))
    kc = torch.randn(B, Hkv, Lmax, D, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, D, device="cuda").to(torch.bfloat16)
    plen = i32([100, 0, 318, 64, 250])
    kp, table = _page(kc, torch.full_like(plen, Lmax), ps, 6)
    vp, _ = _page(vc, torch.full_like(plen, Lmax), ps, 6)
    table[4, (250 + 3) // ps] = -1                 # sequence 4 runs into an unallocated page
    path = i32(rng.integers(1, n + 1, size=(B, depth)))
    acc = i32([6, 3, 6, 0, 6])
    k0, v0 = kp.clone(), vp.clone()
    nl = et.kv_compact_paged(kt, vt, path, acc, plen, kp, vp, table)
    torch.cuda.synchronize()
    u16 = lambda t: t.view(torch.int16).cpu().numpy()
    kr, vr, nlr = oracle.compact_kv_paged(u16(k0), u16(v0), table.cpu().numpy(), plen.cpu().numpy(), u16(kt), u16(vt),
                                          path.cpu().numpy(), acc.cpu().numpy())
    assert nl.cpu().numpy().tolist() == nlr.tolist()
    np.testing.assert_array_equal(u16(kp), kr)
    np.testing.assert_array_equal(u16(vp), vr)


@pytest.mark.parametrize("ps", [16, 128])
def test_step_on_a_paged_cache_equals_the_dense_step(ps):
    cfg = get_config("serve")
    dev = torch.device("cuda")
    w = make_workload(cfg, 1)
    tdt = torch.bfloat16
    lg = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    inp = {"draft_logits": lg(w.draft_logits), "prefix_len": torch.from_numpy(w.prefix_len).to(dev),
           "q": lg(w.q), "k_cache": lg(w.k_cache), "v_cache": lg(w.v_cache), "k_tree": lg(w.k_tree),
           "v_tree": lg(w.v_tree), "uniforms": torch.from_numpy(w.uniforms).to(dev)}
    shape = StepShape(B=cfg.B, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, Lmax=cfg.L, depth=cfg.depth, k=cfg.k, m=cfg.m,
                      V=cfg.V, logits_dtype=tdt, window=cfg.window, stochastic=True)
    dense = VerifyStep(shape, dev)
    dense.build(inp["draft_logits"])
    torch.cuda.synchronize()
    inp["target_logits"] = lg(make_target_logits(cfg, 1, w.draft_logits, dense.tree.draft_row.cpu().numpy()))
    dense.fused(inp)
    kp, table = _page(inp["k_cache"], inp["prefix_len"], ps, 7)
    vp, _ = _page(inp["v_cache"], inp["prefix_len"], ps, 7)
    pinp = dict(inp, k_cache=kp, v_cache=vp, block_table=table)
    pshape = StepShape(**{**shape.__dict__, "paged": True, "Lmax": table.shape[1] * ps})
    one, sep = VerifyStep(pshape, dev), VerifyStep(pshape, dev)
    one.fused(pinp)
    sep(pinp)
    torch.cuda.synchronize()
    one.fused_attention_status()
    for st in (one, sep):
        assert torch.equal(st.out.view(torch.int16), dense.out.view(torch.int16))
        for f in ("accepted_len", "path", "bonus"):
            assert torch.equal(getattr(st, f), getattr(dense, f)), f
