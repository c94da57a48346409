"""Helpers shared by the sizing tests: the cost-aware harness's widening or
deepening run on the oracle, a saturating cost table and a confident draft.
Pure numpy on top of the oracle (no GPU)."""
import numpy as np

import oracle
from workloads import gen_draft_logits, get_config


def _masked(x, k, widths):
    """Rows of the one-shot layout with the rows of frontier slots beyond each level's width set to -inf
    (the level below was drafted from the chosen nodes only)."""
    y = np.array(x, copy=True)
    for level, w in enumerate(widths, start=1):
        r0 = 1 + (level - 1) * k
        if r0 < y.shape[0]:
            y[r0 + w: r0 + k] = -np.inf
    return y


def oracle_grow_widths(x_by_seq, depth, k, table, L, threshold):
    """The harness on the oracle: per level, the width from the level's k best V of every sequence;
    the next level drafted from the chosen slots only; the tree of the chosen candidates."""
    B = len(x_by_seq)
    widths, n = [], 0
    for level in range(1, depth + 1):
        R = 1 + (level - 1) * k
        logv = [oracle.build_tree(_masked(x[:R], k, widths), level, k, k)["level_logv"][-1] for x in x_by_seq]
        w, _ = oracle.level_width(table, B, L, n, np.exp(np.array(logv)), threshold)
        w = min(w, 128 - n)
        if w == 0:
            break
        widths.append(w)
        n += w
    R = 1 + (len(widths) - 1) * k
    trees = [oracle.build_tree(_masked(x[:R], k, widths), len(widths), k, 1, widths=widths) for x in x_by_seq]
    return widths, trees


def saturating_table():
    """Verification cost flat in N until the batch's tokens saturate the GPU, then linear in B*N."""
    Bs, Ls, Ns = [1, 2, 4, 8, 16, 32, 64], [1024, 4096], list(range(0, 161, 8))
    us = np.array([[[max(50.0, 0.5 * b * n) for n in Ns] for _ in Ls] for b in Bs])
    return (Bs, Ls, Ns, us)


def confident_draft():
    """32 sequences, depth 5, k 4, V 300 fp32 draft rows whose best token carries most of the mass."""
    cfg = get_config("tiny", depth=5, k=4, m=32, V=300, B=32, logits_dtype="f32")
    x = gen_draft_logits(cfg, 6).astype(np.float32)
    x[:, :, :8] += 8.0
    for r in range(cfg.R):
        x[:, r, r % 8] += 4.0
    return cfg, x
