"""Helpers for the GPU parity tests: move seeded workloads to the device and
compare GPU results with the oracle.  Imports no CUDA code of the library's own
beyond its public binding."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def dev():
    return torch.device("cuda:0")


def to_dev_logits(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev()).view(torch.bfloat16)


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev()).view(torch.bfloat16)


def i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a), dtype=np.int32)).to(dev())


def dec(a: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    return oracle.decode_logits(a, dtype)


def tree_of(t, b: int) -> dict:
    """Sequence b of a GPU Tree as numpy arrays."""
    return {"tokens": t.tokens[b].cpu().numpy(), "parents": t.parents[b].cpu().numpy(),
            "depth": t.depth[b].cpu().numpy(), "logV": t.logV[b].cpu().numpy(),
            "gid": t.gid[b].cpu().numpy(), "draft_row": t.draft_row[b].cpu().numpy(),
            "row_lse": t.row_lse[b].cpu().numpy()}


from parity import trees_equal  # noqa: E402,F401  (re-exported for the GPU tests)


def attention_ref(q, k_cache, v_cache, L: int, k_tree, v_tree, parents, depth, window: int = 0, rows=None):
    """The oracle's attention output (fp64) and, per output element, the
    rounding scale s = sqrt(sum_j p_j^2 v_j^2) over the keys j it weighs (p the
    oracle's softmax weights, v the key's value in that dimension).  Inputs as
    oracle.tree_attention (fp64 arrays of one sequence); rows = None for every
    (node, head), else the (node, head) pairs of oracle.tree_attention_rows."""
    Hkv, Hq = k_cache.shape[0], q.shape[1]
    G = Hq // Hkv
    vals = [np.concatenate([v_cache[g, :L], v_tree[:, g]], axis=0) for g in range(Hkv)]
    if rows is None:
        out, w = oracle.tree_attention(q, k_cache, v_cache, L, k_tree, v_tree, parents, depth, window=window,
                                       return_weights=True)
        s = np.empty_like(out)
        for h in range(Hq):
            s[:, h] = np.sqrt((w[:, h] ** 2) @ (vals[h // G] ** 2))
        return out, s
    out, w = oracle.tree_attention_rows(q, k_cache, v_cache, L, k_tree, v_tree, parents, depth, rows, window=window,
                                        return_weights=True)
    s = np.stack([np.sqrt((w[r] ** 2) @ (vals[h // G] ** 2)) for r, (_, h) in enumerate(rows)])
    return out, s


def check_attention(got: np.ndarray, ref: np.ndarray, s: np.ndarray):
    """bf16 inputs and output, fp32 accumulation, against fp64.

    The kernel rounds each unnormalised probability P_j to bf16 before the P.V
    product (relative error delta_j, |delta_j| <= 2^-8, zero-mean under
    round-to-nearest-even) while its row sum adds the fp32 P_j, so an output
    element carries err = sum_j p_j delta_j v_j, plus the bf16 rounding of the
    output itself (at most 2^-8 |out|); the fp32 exponentials (about 2 ulp) and
    fp32 accumulation add terms below 1e-5 rms(ref).  Each summand of err lies
    in [-c_j, c_j] with c_j = 2^-8 p_j |v_j|, so by Hoeffding's inequality
    P(|err| > t) <= 2 exp(-t^2 / (2 * 2^-16 s^2)) with s = sqrt(sum_j p_j^2 v_j^2):
    t = 7 * 2^-8 s leaves a chance below 5e-11 per element.  Checked:
      * |gpu - ref| <= 2e-2 + 1e-2 |ref| (the stated bf16 tolerance);
      * |gpu - ref| <= 2^-8 |ref| + 7 * 2^-8 s + 1e-5 rms(ref), element by element;
      * mean of err^2 / var <= 1, var = (2^-16 / 3)(s^2 + ref^2) + (1e-5 rms)^2:
        the variance of the two roundings if each were uniform over its whole
        bound (for round-to-nearest the expected mean is about 0.5), so an
        error of the size of the rounding noise on every element fails."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    assert got.shape == ref.shape == s.shape
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    loose = 2e-2 + 1e-2 * np.abs(ref)
    tight = 2.0 ** -8 * np.abs(ref) + 7 * 2.0 ** -8 * s + 1e-5 * rms
    var = (2.0 ** -16 / 3) * (s ** 2 + ref ** 2) + (1e-5 * rms) ** 2
    where = lambda m: np.unravel_index(np.argmax(m), m.shape)
    assert (err <= loose).all(), f"max err {err.max():.3e} at {where(err - loose)}"
    assert (err <= tight).all(), f"err above the rounding bound: {(err - tight).max():.3e} at {where(err - tight)}"
    ratio = float(np.mean(err ** 2 / var))
    assert ratio <= 1.0, f"mean squared error is {ratio:.3f} of the rounding variance"
    return ratio
