"""Cost-aware tree sizing: the EAGLE-4 harness's level-by-level decision
(EAGLE-4 write-up, "Деревья проверки EAGLE-4 и утилита управления").

A CostTable holds verification latencies measured on the GPU against batch
size, context length and candidates per sequence (``calibrate.py`` measures
this library's share of verification).  ``grow_sized`` drafts a tree level by
level with a TreeGrower, asks the library after each level whether the level's
gain in cumulative probability is worth its marginal cost, stops drafting at
the first level that is not, and builds the tree of the levels kept.  The
decision itself is the library's (``eagle_size_keep_level``); this module only
marshals the table and drives the loop.
"""
from __future__ import annotations

import ctypes
import json
import os
from dataclasses import dataclass
from typing import Callable, Optional, Sequence, Tuple

import numpy as np
import torch

from . import _lib as L


@dataclass
class CostTable:
    """us[len(B)][len(L)][len(N)]: verification latency at each grid point (ascending grids)."""
    B: np.ndarray
    L: np.ndarray
    N: np.ndarray
    us: np.ndarray
    unit: str = "us"

    def __post_init__(self):
        self.B, self.L, self.N = (np.ascontiguousarray(a, dtype=np.float64) for a in (self.B, self.L, self.N))
        self.us = np.ascontiguousarray(self.us, dtype=np.float64)
        if self.us.shape != (self.B.size, self.L.size, self.N.size):
            raise ValueError(f"cost table: us has shape {self.us.shape}, grids give "
                             f"{(self.B.size, self.L.size, self.N.size)}")

    def struct(self) -> L.CostTableStruct:
        p = lambda a: ctypes.c_void_p(a.ctypes.data)
        return L.CostTableStruct(self.B.size, self.L.size, self.N.size, p(self.B), p(self.L), p(self.N), p(self.us))

    def at(self, B: float, L_: float, N: float) -> float:
        return float(L.lib().eagle_cost_at(ctypes.byref(self.struct()), B, L_, N))

    def keep_level(self, B: float, L_: float, k: int, level: int, gains: Sequence[float],
                   threshold: float) -> Tuple[bool, float]:
        g = np.ascontiguousarray(np.asarray(gains, dtype=np.float64).reshape(-1))
        keep, ratio = ctypes.c_int(0), ctypes.c_double(0.0)
        L._check(L.lib().eagle_size_keep_level(ctypes.byref(self.struct()), B, L_, k, level,
                                                   ctypes.c_void_p(g.ctypes.data), g.size, threshold,
                                                   ctypes.byref(keep), ctypes.byref(ratio)),
                 "eagle_size_keep_level")
        return bool(keep.value), float(ratio.value)

    def level_width(self, B: float, L_: float, n_before: int, logv, threshold: float) -> Tuple[int, np.ndarray]:
        """Width of a level (eagle_size_level_width): logv [nb][k] each sequence's k best log V, descending."""
        lv = np.ascontiguousarray(np.asarray(logv, dtype=np.float64))
        nb, k = lv.shape
        width = ctypes.c_int(0)
        ratios = np.zeros(k, dtype=np.float64)
        L._check(L.lib().eagle_size_level_width(ctypes.byref(self.struct()), B, L_, int(n_before),
                                                    ctypes.c_void_p(lv.ctypes.data), k, nb, threshold,
                                                    ctypes.byref(width), ctypes.c_void_p(ratios.ctypes.data)),
                 "eagle_size_level_width")
        return int(width.value), ratios

    def to_json(self, path: str, **meta):
        with open(path, "w") as f:
            json.dump({"B": self.B.tolist(), "L": self.L.tolist(), "N": self.N.tolist(), "us": self.us.tolist(),
                       "unit": self.unit, **meta}, f, indent=1)

    @classmethod
    def from_json(cls, path: str) -> "CostTable":
        with open(path) as f:
            d = json.load(f)
        return cls(np.array(d["B"]), np.array(d["L"]), np.array(d["N"]), np.array(d["us"]), d.get("unit", "us"))


# Measured on a B200 by calibrate.py (mask + tree attention + greedy acceptance as one CUDA graph, L2 flushed):
# Hq 32, Hkv 8, D 128, V 128256 bf16; B in {1, 4, 16, 32}, L in {1024, 4096, 16384}, N up to 128.
DEFAULT_TABLE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "data",
                             "cost_b200_hq32_hkv8_d128_v128256_bf16.json")


def default_table() -> CostTable:
    """The cost table measured on a B200 for the 32/8-head, D 128, 128k-vocabulary shape."""
    return CostTable.from_json(DEFAULT_TABLE)


def table_path(Hq: int, Hkv: int, D: int, V: int, dtype: str) -> str:
    """Where the shipped B200 table of a verification shape lives (it may not exist)."""
    return os.path.join(os.path.dirname(DEFAULT_TABLE), f"cost_b200_hq{Hq}_hkv{Hkv}_d{D}_v{V}_{dtype}.json")


def table_for(Hq: int, Hkv: int, D: int, V: int, dtype: str) -> CostTable:
    """The shipped B200 cost table measured for exactly this shape (query / KV heads, head dim,
    vocabulary, logit storage "bf16" or "f32"); FileNotFoundError when none was measured."""
    p = table_path(Hq, Hkv, D, V, dtype)
    if not os.path.exists(p):
        raise FileNotFoundError(f"no cost table measured for Hq={Hq} Hkv={Hkv} D={D} V={V} {dtype}: run "
                                f"python -m eagle_tree_verification_dynamic_b200.calibrate --out {p} ...")
    return CostTable.from_json(p)


@dataclass
class SizedTree:
    tree: Optional[L.Tree]     # None when no level was worth verifying
    levels_kept: int
    levels_drafted: int
    ratios: list               # each drafted level's gain / marginal cost


def grow_sized(grower: L.TreeGrower, root_logits: torch.Tensor,
               draft_fn: Callable[[int, torch.Tensor, torch.Tensor], torch.Tensor], table: CostTable,
               context_len: float, threshold: float) -> SizedTree:
    """Draft level by level while each level pays for itself.

    draft_fn(level, frontier_tokens [B][k], frontier_parents [B][k]) -> that level's rows [B][k][V] on the
    device (the draft model's distributions after each frontier node).  After each level the per-sequence
    gains are read back (one small device-to-host copy: the host decides whether to run the draft model
    again) and the library's decision applied.  The tree keeps m = k x (levels kept) candidates, the best
    by V over every level drafted."""
    B, k = grower.B, grower.k
    tok, par = grower.begin(root_logits)
    kept, drafted, ratios = 0, 0, []
    for level in range(1, grower.depth + 1):
        if level > 1:
            tok, par = grower.level(draft_fn(level, tok, par), level)
        drafted = level
        keep, ratio = table.keep_level(B, context_len, k, level, grower.gains().cpu().numpy(), threshold)
        ratios.append(ratio)
        if not keep:
            break
        kept = level
    if kept == 0:
        return SizedTree(None, 0, drafted, ratios)
    m = min(k * kept, L.MAX_NODES)
    return SizedTree(grower.finish(m, levels=drafted), kept, drafted, ratios)


@dataclass
class WidthTree:
    tree: Optional[L.Tree]     # None when not even the first candidate was worth verifying
    widths: list               # candidates kept per level (each level drafted from the previous width)
    ratios: list               # per level drafted: each examined candidate's gain / marginal cost


def grow_widths(grower: L.TreeGrower, root_logits: torch.Tensor,
                draft_fn: Callable[[int, torch.Tensor, torch.Tensor, int], torch.Tensor], table: CostTable,
                context_len: float, threshold: float) -> WidthTree:
    """Widen or deepen while each candidate pays for itself.

    After each level the level's k best log V per sequence are read back (one small device-to-host copy)
    and the library chooses the level's width; the next level is drafted from that many frontier slots:
    draft_fn(level, frontier_tokens [B][k], frontier_parents [B][k], width) -> rows [B][width][V] (the draft
    model runs on the chosen nodes only).  Drafting stops at a width of 0 or at the grower's depth; the
    tree keeps each level's chosen candidates (at most MAX_NODES in all)."""
    B = grower.B
    tok, par = grower.begin(root_logits)
    widths, ratios, n = [], [], 0
    for level in range(1, grower.depth + 1):
        if level > 1:
            tok, par = grower.level_width(draft_fn(level, tok, par, widths[-1]), level, widths[-1])
        w, r = table.level_width(B, context_len, n, grower.frontier_logv().cpu().numpy(), threshold)
        ratios.append(r)
        w = min(w, L.MAX_NODES - n)
        if w == 0:
            break
        widths.append(w)
        n += w
    if not widths:
        return WidthTree(None, [], ratios)
    return WidthTree(grower.finish_widths(widths), widths, ratios)
