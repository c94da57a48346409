"""Small fp64 helpers of the oracle (its own; nothing here is shared)."""
from __future__ import annotations

import numpy as np

NEAR_TIE_REL = 1e-6


def decode_logits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored logits -> fp64.  bf16 is given as its uint16 bit patterns."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        u = np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16
        return u.view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def decode_bf16(x: np.ndarray) -> np.ndarray:
    return decode_logits(x, "bf16")


def logsumexp(row: np.ndarray) -> float:
    """log sum_i exp(row_i) in fp64, shifted by the maximum."""
    row = np.asarray(row, dtype=np.float64)
    mx = row.max()
    if mx == -np.inf:  # every term is exp(-inf) = 0: log 0
        return -np.inf
    return float(mx + np.log(np.exp(row - mx).sum()))


def softmax(row: np.ndarray) -> np.ndarray:
    """Draft confidence / target probability: exp(l_x) / sum_i exp(l_i)
    (EAGLE-2 notes, "Well-Calibrated Draft Model")."""
    row = np.asarray(row, dtype=np.float64)
    e = np.exp(row - row.max())
    return e / e.sum()


def near_tie(a: float, b: float, rel: float = NEAR_TIE_REL) -> bool:
    """True when two scores differ by at most `rel` of the larger magnitude."""
    return abs(a - b) <= rel * max(abs(a), abs(b))
