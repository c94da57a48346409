"""One whole tree-verification step with preallocated buffers.

build (vocabulary sweep + EAGLE-2 expansion/rerank) -> mask -> tree attention
-> acceptance, enqueued on the current CUDA stream through the C ABI: either
as the four calls one after another (``__call__``) or as the single
``eagle_verify_step`` call (``fused``: the mask fused into the expansion, one
clearing of the scratch, kernels chained by programmatic dependent launch).
All buffers and workspaces are allocated once in the constructor, so a step
allocates nothing and can be captured in a CUDA graph.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib as L


@dataclass
class StepShape:
    B: int
    Hq: int
    Hkv: int
    D: int
    Lmax: int
    depth: int
    k: int
    m: int
    V: int
    logits_dtype: torch.dtype
    window: int = 0
    stochastic: bool = True
    without_replacement: bool = False   # sampled acceptance: a rejected child's token leaves q
    paged: bool = False                 # prefix cache as page pools + block table (Lmax = pages_per_seq x page_size)

    @property
    def R(self) -> int:
        return 1 + (self.depth - 1) * self.k

    @property
    def n(self) -> int:
        return min(self.m, L.pool_size(self.depth, self.k))


class VerifyStep:
    def __init__(self, shape: StepShape, device=None):
        self.s = shape
        dev = torch.device(device or "cuda")
        self.device = dev
        s = shape
        dcode = L.F32 if s.logits_dtype == torch.float32 else L.BF16
        self.tree = L.alloc_tree(s.B, s.R, s.depth, s.k, s.m, dev)
        n = self.tree.n
        self.mask = torch.empty(s.B, n, 2, dtype=torch.int64, device=dev)
        self.pos = torch.empty(s.B, n, dtype=torch.int32, device=dev)
        self.out = torch.empty(s.B, n, s.Hq, s.D, dtype=torch.bfloat16, device=dev)
        self.accepted_len = torch.empty(s.B, dtype=torch.int32, device=dev)
        self.path = torch.empty(s.B, s.depth, dtype=torch.int32, device=dev)
        self.bonus = torch.empty(s.B, dtype=torch.int32, device=dev)
        self.ws_build = L._workspace(L.tree_build_workspace_bytes(s.B, s.R, s.V, dcode, s.k), dev)
        self.ws_attn = L._workspace(L.attention_workspace_bytes(s.B, n, s.Hq, s.Hkv, s.D, s.Lmax, s.window), dev)
        self.ws_acc = L._workspace(L.accept_workspace_bytes(s.B, n, s.V, dcode), dev)
        shape_only = L.StepIn(None, None, dcode, s.B, s.V, s.depth, s.k, s.m, None, None, None, None, s.Lmax, None,
                              None, s.Hq, s.Hkv, s.D, s.window, 0.0, None, 0)
        self.ws_step = L._workspace(L.step_workspace_bytes(shape_only), dev)
        # the two vocabulary sweeps on their own (for timing them apart from the
        # expansion and the walk): draft rows top-k + lse, target rows argmax + lse
        rows_d, rows_t = s.B * s.R, s.B * (n + 1)
        self.sw_tok = torch.empty(rows_d, s.k, dtype=torch.int32, device=dev)
        self.sw_val = torch.empty(rows_d, s.k, dtype=torch.float32, device=dev)
        self.sw_lse = torch.empty(rows_d, dtype=torch.float64, device=dev)
        self.sw_amax = torch.empty(rows_t, 1, dtype=torch.int32, device=dev)
        self.sw_max = torch.empty(rows_t, 1, dtype=torch.float32, device=dev)
        self.sw_lse_t = torch.empty(rows_t, dtype=torch.float64, device=dev)
        self.ws_sweep_d = L._workspace(L.row_stats_workspace_bytes(rows_d, s.V, dcode, s.k), dev)
        self.ws_sweep_t = L._workspace(L.row_stats_workspace_bytes(rows_t, s.V, dcode, 1), dev)

    def draft_sweep(self, draft_logits: torch.Tensor):
        """The build's vocabulary sweep alone: top-k and log-sum-exp of every draft row."""
        L.row_stats_into(draft_logits, self.s.k, self.sw_tok, self.sw_val, self.sw_lse, self.ws_sweep_d)

    def accept_sweep(self, target_logits: torch.Tensor):
        """The acceptance's target sweep alone: argmax and log-sum-exp of every target row."""
        L.row_stats_into(target_logits, 1, self.sw_amax, self.sw_max, self.sw_lse_t, self.ws_sweep_t)

    def build(self, draft_logits: torch.Tensor):
        L.tree_build_into(draft_logits, self.s.depth, self.s.k, self.s.m, self.tree, self.ws_build)

    def mask_(self, prefix_len: torch.Tensor):
        L.tree_mask_into(self.tree.parents, self.tree.depth, prefix_len, self.mask, self.pos)

    def attention(self, q, k_cache, v_cache, prefix_len, k_tree, v_tree, block_table=None):
        if self.s.paged:
            L.tree_attention_paged_into(q, k_cache, v_cache, block_table, prefix_len, k_tree, v_tree, self.mask,
                                        self.pos, self.out, self.ws_attn, self.s.window)
        else:
            L.tree_attention_into(q, k_cache, v_cache, prefix_len, k_tree, v_tree, self.mask, self.pos, self.out,
                                  self.ws_attn, self.s.window)

    def accept(self, target_logits, uniforms: Optional[torch.Tensor], draft_logits):
        if self.s.stochastic:
            L.accept_into(target_logits, self.tree.tokens, self.tree.parents, self.tree.draft_row, self.s.depth,
                          uniforms, draft_logits, self.tree.row_lse, self.accepted_len, self.path, self.bonus,
                          self.ws_acc, self.s.without_replacement)
        else:
            L.accept_into(target_logits, self.tree.tokens, self.tree.parents, self.tree.draft_row, self.s.depth,
                          None, None, None, self.accepted_len, self.path, self.bonus, self.ws_acc)

    def fused(self, inp: dict):
        """The same step as one eagle_verify_step call (same outputs)."""
        s = self.s
        si = L.step_in(inp["draft_logits"], inp["target_logits"], s.depth, s.k, s.m, inp["q"], inp["k_cache"],
                       inp["v_cache"], inp["prefix_len"], inp["k_tree"], inp["v_tree"],
                       inp.get("uniforms") if s.stochastic else None, s.window,
                       without_replacement=s.without_replacement,
                       block_table=inp["block_table"] if s.paged else None)
        L.step_into(si, self.tree, self.mask, self.pos, self.out, self.accepted_len, self.path, self.bonus,
                    self.ws_step, self.device)
        self._step_in = si
        return self.accepted_len, self.path, self.bonus

    def fused_attention_status(self):
        """Raise if the last fused step's attention reported a device status."""
        L.step_attention_status(self._step_in, self.ws_step)

    def __call__(self, inp: dict):
        """inp: draft_logits, prefix_len, q, k_cache, v_cache, k_tree, v_tree, target_logits, uniforms."""
        self.build(inp["draft_logits"])
        self.mask_(inp["prefix_len"])
        self.attention(inp["q"], inp["k_cache"], inp["v_cache"], inp["prefix_len"], inp["k_tree"], inp["v_tree"],
                       inp.get("block_table"))
        self.accept(inp["target_logits"], inp.get("uniforms"), inp["draft_logits"])
        return self.accepted_len, self.path, self.bonus
