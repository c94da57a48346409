"""Cost-aware tree sizing (EAGLE-4 write-up, "Деревья проверки EAGLE-4 и
утилита управления"): a cost table of verification latency against batch
size, context length and number of candidates, measured once on the target
GPU; at each draft level the gain in cumulative probability divided by the
level's marginal cost, compared with a threshold; the tree grows while the
ratio stays at or above it.

Readings the pages leave open, taken here:
  * The table holds latencies C[i][j][l] at grid points B_i, L_j, N_l (N =
    candidates verified per sequence).  Between grid points C is
    interpolated linearly along each axis in turn (multilinear); outside the
    grid the end segment is extended; an axis with one point is constant.
  * A level's gain is, per sequence, the sum of V = exp(log V) over the
    level's k best candidates: the expected number of tokens they add.  The
    batch gain is the sum over the sequences.
  * Level l (l >= 1) would grow the verified set from (l-1)k to lk candidates
    per sequence.  Its marginal cost per token is
    (C(B, L, lk) - C(B, L, (l-1)k)) / (B k) and its gain per token
    gain_l / (B k); their ratio gain_l / (C(B, L, lk) - C(B, L, (l-1)k)) is
    compared with the threshold (tokens per unit of cost).  A level whose
    marginal cost is not positive is always kept.
  * Drafting stops at the first level below the threshold; the tree keeps
    m = k x (levels kept) candidates, the best by V among all levels drafted.
    With no level kept there is nothing to verify.
  * For a batch of mixed context lengths the caller passes one L (e.g. the
    mean).
  * Widening or deepening (the same passage: the harness "widens or deepens
    the tree while the ratio stays above the threshold", giving a wide, deep
    tree at batch 1 and a narrow tree or a chain at large batch, with no fixed
    top-k): at level l the level's candidates are taken one at a time in
    descending V, the j-th best of every sequence together.  With N
    candidates per sequence already chosen, the j-th adds the batch gain
    sum_b V_b,(j) at the marginal cost C(B, L, N + 1) - C(B, L, N); it is taken
    while its gain is positive and gain / cost >= threshold (a cost that does
    not grow always passes), and the first one that fails ends the level.  The
    level's width w_l is the number taken; w_l = 0 stops drafting.  The next
    level is drafted from the w_l chosen nodes only, and the tree verifies,
    level by level, the w_l best of each level (closed under "parent of",
    since each level's candidates are children of the previous level's
    chosen nodes).
"""
from __future__ import annotations

from typing import Sequence

import numpy as np


def _interp_axis(grid: np.ndarray, x: float):
    """(lower index, weight of the upper point) of x on an ascending grid,
    extending the end segments; a single point gives (0, 0)."""
    if grid.shape[0] == 1:
        return 0, 0.0
    i = int(np.searchsorted(grid, x, side="right")) - 1
    i = min(max(i, 0), grid.shape[0] - 2)
    return i, (x - grid[i]) / (grid[i + 1] - grid[i])


def cost_at(Bs: Sequence[float], Ls: Sequence[float], Ns: Sequence[float], us: np.ndarray,
            B: float, L: float, N: float) -> float:
    """Multilinear interpolation of the table us[len(Bs)][len(Ls)][len(Ns)] at (B, L, N)."""
    Bs, Ls, Ns = (np.asarray(a, dtype=np.float64) for a in (Bs, Ls, Ns))
    us = np.asarray(us, dtype=np.float64)
    ib, wb = _interp_axis(Bs, B)
    il, wl = _interp_axis(Ls, L)
    iN, wn = _interp_axis(Ns, N)
    total = 0.0
    for db, fb in ((0, 1.0 - wb), (1, wb)):
        for dl, fl in ((0, 1.0 - wl), (1, wl)):
            for dn, fn in ((0, 1.0 - wn), (1, wn)):
                f = fb * fl * fn
                if f != 0.0:
                    total += f * us[ib + db, il + dl, iN + dn]
    return float(total)


def level_ratio(table, B: float, L: float, k: int, level: int, gains: Sequence[float]) -> float:
    """Batch gain of `level` per unit of its marginal cost (inf when the cost does not grow)."""
    Bs, Ls, Ns, us = table
    dc = cost_at(Bs, Ls, Ns, us, B, L, level * k) - cost_at(Bs, Ls, Ns, us, B, L, (level - 1) * k)
    g = float(np.sum(np.asarray(gains, dtype=np.float64)))
    return np.inf if dc <= 0.0 else g / dc


def keep_level(table, B: float, L: float, k: int, level: int, gains: Sequence[float], threshold: float) -> bool:
    return level_ratio(table, B, L, k, level, gains) >= threshold


def levels_kept(table, B: float, L: float, k: int, gains_by_level: Sequence[Sequence[float]],
                threshold: float) -> int:
    """Levels kept when the gains of levels 1, 2, ... are as given (one list of per-sequence gains each)."""
    kept = 0
    for level, g in enumerate(gains_by_level, start=1):
        if not keep_level(table, B, L, k, level, g, threshold):
            break
        kept = level
    return kept


def level_width(table, B: float, L: float, n_before: int, values_by_seq: Sequence[Sequence[float]],
                threshold: float):
    """(width, ratios): how many of a level's candidates to verify.  values_by_seq[b] holds sequence b's
    candidate values V of this level in descending order (one list per sequence, equal lengths);
    n_before = candidates per sequence chosen at earlier levels.  ratios[j] is the j-th candidate's batch
    gain over its marginal cost, for the candidates examined."""
    Bs, Ls, Ns, us = table
    vals = np.asarray(values_by_seq, dtype=np.float64)
    width, ratios = 0, []
    for j in range(vals.shape[1]):
        g = float(np.sum(vals[:, j]))
        dc = cost_at(Bs, Ls, Ns, us, B, L, n_before + j + 1) - cost_at(Bs, Ls, Ns, us, B, L, n_before + j)
        r = np.inf if dc <= 0.0 else g / dc
        ratios.append(r)
        if not (g > 0.0 and r >= threshold):
            break
        width = j + 1
    return width, ratios
