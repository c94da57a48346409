"""GPU: eagle_verify_step, the whole step as one call (mask fused into the tree
expansion, one clearing of the scratch, kernels chained by programmatic
dependent launch), against the four calls eagle_tree_build, eagle_tree_mask,
eagle_tree_attention and eagle_accept made one after another on the same inputs.

The separate calls run the same kernels with the same arithmetic, so every
output must agree bit for bit; the separate calls are themselves compared with
the oracle by the other GPU tests, and on the tiny workload the step is also
compared with the oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle
from eagle_tree_verification_dynamic_b200.step import StepShape, VerifyStep
from workloads import get_config, make_target_logits, make_workload

from parity import walk_match
from gpu_helpers import attention_ref, check_attention, dec

pytestmark = pytest.mark.gpu


def _inputs(cfg, seed, dev):
    w = make_workload(cfg, seed)
    tdt = torch.float32 if cfg.logits_dtype == "f32" else torch.bfloat16

    def logits(a):
        if cfg.logits_dtype == "f32":
            return torch.from_numpy(a).to(dev)
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    inp = {"draft_logits": logits(w.draft_logits), "prefix_len": torch.from_numpy(w.prefix_len).to(dev),
           "q": bf(w.q), "k_cache": bf(w.k_cache), "v_cache": bf(w.v_cache), "k_tree": bf(w.k_tree),
           "v_tree": bf(w.v_tree), "uniforms": torch.from_numpy(w.uniforms).to(dev)}
    return w, inp, tdt, logits


def _run_both(name, mode, seed=0):
    cfg = get_config(name)
    dev = torch.device("cuda")
    w, inp, tdt, logits = _inputs(cfg, seed, dev)
    shape = StepShape(B=cfg.B, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, Lmax=cfg.L, depth=cfg.depth, k=cfg.k, m=cfg.m,
                      V=cfg.V, logits_dtype=tdt, window=cfg.window, stochastic=mode.startswith("stochastic"),
                      without_replacement=(mode == "stochastic-wor"))
    sep, one = VerifyStep(shape, dev), VerifyStep(shape, dev)
    sep.build(inp["draft_logits"])
    torch.cuda.synchronize()
    inp["target_logits"] = logits(make_target_logits(cfg, seed, w.draft_logits, sep.tree.draft_row.cpu().numpy()))
    sep(inp)
    one.fused(inp)
    torch.cuda.synchronize()
    one.fused_attention_status()
    return cfg, w, inp, sep, one


@pytest.mark.parametrize("name,mode", [("tiny", "greedy"), ("tiny", "stochastic"), ("7b", "stochastic"),
                                       ("7b", "greedy"), ("l3-8b", "stochastic"), ("serve", "stochastic"),
                                       ("7b", "stochastic-wor"), ("serve", "stochastic-wor"),
                                       ("long-window", "greedy")])
def test_step_equals_the_separate_calls(name, mode):
    cfg, w, inp, sep, one = _run_both(name, mode)
    for field in ("tokens", "parents", "depth", "logV", "gid", "draft_row", "row_lse"):
        assert torch.equal(getattr(one.tree, field), getattr(sep.tree, field)), field
    assert torch.equal(one.mask, sep.mask)
    assert torch.equal(one.pos, sep.pos)
    assert torch.equal(one.out.view(torch.int16), sep.out.view(torch.int16))
    for field in ("accepted_len", "path", "bonus"):
        assert torch.equal(getattr(one, field), getattr(sep, field)), field


def test_step_matches_the_oracle_on_the_tiny_workload():
    cfg, w, inp, sep, one = _run_both("tiny", "stochastic")
    x = oracle.decode_logits(w.draft_logits, cfg.logits_dtype)[0]
    ref = oracle.build_tree(x, cfg.depth, cfg.k, cfg.m)
    assert one.tree.tokens[0].cpu().numpy().tolist() == ref["tokens"].tolist()
    assert one.tree.parents[0].cpu().numpy().tolist() == ref["parents"].tolist()
    np.testing.assert_array_equal(one.mask[0].cpu().numpy().view(np.uint64),
                                  oracle.pack_mask(oracle.ancestor_mask(ref["parents"])))
    np.testing.assert_array_equal(one.pos[0].cpu().numpy(), oracle.positions(ref["depth"], int(w.prefix_len[0])))
    ref_out, s = attention_ref(dec(w.q[0]), dec(w.k_cache[0]), dec(w.v_cache[0]), int(w.prefix_len[0]),
                               dec(w.k_tree[0]), dec(w.v_tree[0]), ref["parents"], ref["depth"])
    check_attention(one.out[0].float().cpu().numpy(), ref_out, s)
    tgt = oracle.decode_logits(make_target_logits(cfg, 0, w.draft_logits, ref["draft_row"][None]),
                               cfg.logits_dtype)[0]
    walk = lambda nodes=(): oracle.accept_stochastic(tgt, x, ref["tokens"], ref["parents"], ref["draft_row"],
                                                     w.uniforms[0].astype(np.float64), cfg.depth, flip=set(nodes))
    walk_match((one.accepted_len[0], one.path[0].cpu().numpy().tolist(), one.bonus[0]), walk(), walk)
