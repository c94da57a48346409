"""Measure the cost table for cost-aware tree sizing on this GPU.

The EAGLE-4 harness sizes its tree from a table of verification latency
against batch size, context length and number of candidates, calibrated once
offline on the target GPU (EAGLE-4 write-up, "Деревья проверки EAGLE-4 и
утилита управления").  This script measures this library's share of
verification for each grid point: the tree mask, the tree-masked attention
over the prefix cache and the tree, and greedy acceptance over the target's
n + 1 rows; a serving stack adds its target model's forward pass over the same
tokens to these numbers.  N = 0 costs nothing (there is nothing to verify).

    python -m eagle_tree_verification_dynamic_b200.calibrate --out cost.json \
        [--B 1,4,16,32] [--L 1024,4096,16384] [--N 0,8,16,32,64,96,128] \
        [--Hq 32 --Hkv 8 --D 128 --V 128256 --dtype bf16]

Inputs are random device tensors; the three calls are captured in one CUDA
graph (device time, without the host's per-call overhead), the L2 cache is
flushed before every timed replay and the median of the replays is kept.
"""
from __future__ import annotations

import argparse
import statistics

import numpy as np
import torch

from . import _lib as L
from .sizing import CostTable

_L2_FLUSH_BYTES = 256 << 20


def _ints(s: str):
    return [int(v) for v in s.split(",") if v]


def _tree(n: int, dev):
    """A complete 4-ary tree of n nodes (node j's parent (j-1)//4): depth <= 4 up to 84 nodes, 5 up to 340."""
    parents = np.array([(j - 1) // 4 for j in range(1, n + 1)], dtype=np.int32)
    depth = np.zeros(n, dtype=np.int32)
    for j in range(n):
        depth[j] = 1 if parents[j] == 0 else depth[parents[j] - 1] + 1
    return parents, depth


def measure_point(B: int, Lctx: int, n: int, Hq: int, Hkv: int, D: int, V: int, dtype: torch.dtype, reps: int,
                  flush: torch.Tensor, dev) -> float:
    if n == 0:
        return 0.0
    par, dep = _tree(n, dev)
    max_depth = int(dep.max())
    parents = torch.from_numpy(np.tile(par, (B, 1))).to(dev)
    depth = torch.from_numpy(np.tile(dep, (B, 1))).to(dev)
    tokens = torch.randint(0, V, (B, n), dtype=torch.int32, device=dev)
    draft_row = torch.full((B, n + 1), -1, dtype=torch.int32, device=dev)
    plen = torch.full((B,), Lctx, dtype=torch.int32, device=dev)
    bf = dict(dtype=torch.bfloat16, device=dev)
    q = torch.randn(B, n, Hq, D, **bf)
    kc, vc = torch.randn(B, Hkv, Lctx, D, **bf), torch.randn(B, Hkv, Lctx, D, **bf)
    kt, vt = torch.randn(B, n, Hkv, D, **bf), torch.randn(B, n, Hkv, D, **bf)
    target = torch.randn(B, n + 1, V, dtype=dtype, device=dev)
    mask = torch.empty(B, n, 2, dtype=torch.int64, device=dev)
    pos = torch.empty(B, n, dtype=torch.int32, device=dev)
    out = torch.empty(B, n, Hq, D, **bf)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    path = torch.empty(B, max_depth, dtype=torch.int32, device=dev)
    bonus = torch.empty(B, dtype=torch.int32, device=dev)
    ws_a = L._workspace(L.attention_workspace_bytes(B, n, Hq, Hkv, D, Lctx), dev)
    ws_c = L._workspace(L.accept_workspace_bytes(B, n, V, L.F32 if dtype == torch.float32 else L.BF16), dev)

    def verify():
        L.tree_mask_into(parents, depth, plen, mask, pos)
        L.tree_attention_into(q, kc, vc, plen, kt, vt, mask, pos, out, ws_a)
        L.accept_into(target, tokens, parents, draft_row, max_depth, None, None, None, acc, path, bonus, ws_c)

    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for _ in range(3):  # sets the kernels' attributes before capture
            verify()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        verify()
    times = []
    with torch.cuda.stream(stream):
        for _ in range(reps):
            flush.add_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b) * 1000.0)
    del graph
    return statistics.median(times)


def calibrate(Bs, Ls, Ns, Hq=32, Hkv=8, D=128, V=128256, dtype=torch.bfloat16, reps=15, device="cuda") -> CostTable:
    dev = torch.device(device)
    flush = torch.zeros(_L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    us = np.zeros((len(Bs), len(Ls), len(Ns)))
    for i, B in enumerate(Bs):
        for j, Lctx in enumerate(Ls):
            for l, n in enumerate(Ns):
                us[i, j, l] = measure_point(B, Lctx, n, Hq, Hkv, D, V, dtype, reps, flush, dev)
            torch.cuda.empty_cache()
    return CostTable(np.array(Bs), np.array(Ls), np.array(Ns), us)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", required=True)
    ap.add_argument("--B", default="1,4,16,32")
    ap.add_argument("--L", default="1024,4096,16384")
    ap.add_argument("--N", default="0,8,16,32,64,96,128")
    ap.add_argument("--Hq", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=8)
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--V", type=int, default=128256)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--reps", type=int, default=15)
    a = ap.parse_args()
    dtype = torch.bfloat16 if a.dtype == "bf16" else torch.float32
    t = calibrate(_ints(a.B), _ints(a.L), _ints(a.N), a.Hq, a.Hkv, a.D, a.V, dtype, a.reps)
    t.to_json(a.out, what="mask + tree attention + greedy acceptance as one CUDA graph, median microseconds, L2 flushed",
              Hq=a.Hq, Hkv=a.Hkv, D=a.D, V=a.V, dtype=a.dtype, gpu=torch.cuda.get_device_name())
    print(f"wrote {a.out}: {t.us.size} points, {t.us.min():.1f}..{t.us.max():.1f} us")


if __name__ == "__main__":
    main()
