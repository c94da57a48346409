"""The attention parity bound of tests/gpu_helpers.check_attention, checked on
the CPU against an emulation of the kernel's arithmetic (no GPU).

The emulation rounds each unnormalised probability to bf16 for the P.V product,
sums the fp32 probabilities for the row sum, and rounds the output to bf16, as
the tree-attention kernel does.  It must pass, with the mean squared error near
half the rounding variance; emulations with a planted mistake (a visible key
dropped, a scale off by 1 %, probabilities rounded to 6 bits instead of 8) must
fail.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import attention_ref, check_attention


def _case(seed=0, n=24, Hq=4, Hkv=2, D=64, L=700):
    rng = np.random.default_rng(seed)
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).bfloat16().double().numpy()
    q, kc, vc = bf(rng.normal(size=(n, Hq, D))), bf(rng.normal(size=(Hkv, L, D))), bf(rng.normal(size=(Hkv, L, D)))
    kt, vt = bf(rng.normal(size=(n, Hkv, D))), bf(rng.normal(size=(n, Hkv, D)))
    parents = np.array([0] + [int(rng.integers(0, i + 1)) for i in range(1, n)])
    depth = np.zeros(n, dtype=np.int64)
    for i in range(n):
        depth[i] = 1 if parents[i] == 0 else depth[parents[i] - 1] + 1
    return q, kc, vc, L, kt, vt, parents, depth


def _emulate(q, kc, vc, L, kt, vt, parents, depth, p_bits=8, drop_key=None, scale_factor=1.0):
    n, Hq, D = q.shape
    G = Hq // kc.shape[0]
    anc = oracle.ancestor_mask(parents)
    out = np.empty((n, Hq, D))
    for h in range(Hq):
        g = h // G
        keys = np.concatenate([kc[g, :L], kt[:, g]])
        vals = np.concatenate([vc[g, :L], vt[:, g]]).astype(np.float32)
        s = (q[:, h] @ keys.T).astype(np.float32) * np.float32(scale_factor / math.sqrt(D))
        vis = np.concatenate([np.ones((n, L), dtype=bool), anc], axis=1)
        if drop_key is not None:
            vis[:, drop_key] = False
        s = np.where(vis, s, -np.inf)
        P = np.exp(s - s.max(axis=1, keepdims=True)).astype(np.float32)
        if p_bits == 8:
            Pr = torch.from_numpy(P).bfloat16().float().numpy()
        else:  # round to p_bits significant bits
            m, e = np.frexp(P)
            Pr = np.ldexp(np.round(m * 2.0 ** p_bits) / 2.0 ** p_bits, e).astype(np.float32)
        o = (Pr @ vals) / P.sum(axis=1, keepdims=True)
        out[:, h] = torch.from_numpy(o.astype(np.float32)).bfloat16().double().numpy()
    return out


def test_emulated_kernel_arithmetic_passes():
    case = _case()
    ref, s = attention_ref(*case)
    ratio = check_attention(_emulate(*case), ref, s)
    assert 0.2 < ratio < 0.8, ratio


@pytest.mark.parametrize("mistake", [{"drop_key": 5}, {"scale_factor": 1.01}, {"p_bits": 6}])
def test_planted_mistakes_fail(mistake):
    case = _case(seed=1)
    ref, s = attention_ref(*case)
    with pytest.raises(AssertionError):
        check_attention(_emulate(*case, **mistake), ref, s)


def test_rows_variant_gives_the_same_scale():
    case = _case(seed=2, n=10)
    ref, s = attention_ref(*case)
    rows = [(0, 0), (9, 3), (4, 1)]
    r2, s2 = attention_ref(*case, rows=rows)
    np.testing.assert_allclose(r2, np.array([ref[i, h] for i, h in rows]), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(s2, np.array([s[i, h] for i, h in rows]), rtol=1e-12)
