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


def trees_equal(g: dict, r: dict) -> bool:
    return all(np.array_equal(np.asarray(g[k]).astype(np.int64), np.asarray(r[k]).astype(np.int64))
               for k in ("tokens", "parents", "depth", "draft_row", "gid"))


def check_attention(got: np.ndarray, ref: np.ndarray):
    """bf16 inputs and output, fp32 accumulation, against fp64:
      * elementwise |gpu - ref| <= 2e-2 + 1e-2 |ref| (the stated bf16 tolerance);
      * elementwise |gpu - ref| <= 2^-8 |ref| + 1e-2 rms(ref): the bf16 output
        rounding (at most 2^-8 relative) plus the bf16 rounding of the
        probabilities fed to the P.V product (about 2^-9 rms(ref)); it keeps the
        check meaningful when |out| ~ 0.02 makes the first one vacuous;
      * rms(gpu - ref) / rms(ref) <= 1e-2."""
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    loose = 2e-2 + 1e-2 * np.abs(ref)
    tight = 2.0 ** -8 * np.abs(ref) + 1e-2 * rms
    where = lambda m: np.unravel_index(np.argmax(m), m.shape)
    assert (err <= loose).all(), f"max err {err.max():.3e} at {where(err - loose)}"
    assert (err <= tight).all(), f"err above bf16 rounding: {(err - tight).max():.3e} at {where(err - tight)}"
    assert np.sqrt(np.mean(err ** 2)) <= 1e-2 * rms
