#!/usr/bin/env python
"""Benchmark one EAGLE tree-verification step (tree build -> mask -> tree
attention -> acceptance) on B200.

Default workload: the Llama-7B-shaped verify (batch 1, 32 heads MHA,
head_dim 128, prefix 2048, depth 6, top-k 10, m = 60 nodes, vocab 32000 fp32
logits, sampled acceptance).  Inputs are seeded synthetic tensors; several
input sets whose total size exceeds twice the L2 cache are rotated between
steps, so every step reads its KV cache and logits from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--mode stochastic|stochastic-wor|greedy] [--impl ours|reference]
                    [--paged PAGE_SIZE]

With N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the workload (the step has no cross-sequence exchange); the job value is the
sum over ranks of steps, divided by the slowest rank's device time.
`--impl reference` times the CPU oracle on the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import get_config, gen_attention_inputs, gen_draft_logits, gen_prefix_len, gen_uniforms  # noqa: E402
from workloads import make_target_logits  # noqa: E402

L2_BYTES = 126 * 2 ** 20
METRIC = ("tree-verify steps/sec (and achieved KV HBM GB/s of the tree attention) at the 7B shape, "
          "prefix 2048, 60-node tree")
LAUNCHES_PER_STEP = 6  # one eagle_verify_step: row sweep, expand (+ mask), attention main + combine, target sweep, walk

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="7b")
    ap.add_argument("--mode", default="stochastic", choices=["stochastic", "stochastic-wor", "greedy"],
                    help="acceptance: sampled (rejected siblings' tokens kept in q, or removed: -wor) or greedy")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="report the headline workload only (default: the other workloads too, in per_config)")
    ap.add_argument("--cpu-seconds-per-config", type=float, default=8.0,
                    help="budget of each other workload's CPU-oracle sample")
    ap.add_argument("--paged", type=int, default=0, metavar="PAGE_SIZE",
                    help="prefix cache as a shuffled pool of pages of this many keys (16, 32 or a multiple of 64)")
    return ap.parse_args()


def workload_desc(cfg, mode):
    L = f"prefix {cfg.L}" if not cfg.ragged else f"prefix U[{cfg.L_min},{cfg.L}]"
    w = f", window {cfg.window}" if cfg.window else ""
    return (f"{cfg.name}: B={cfg.B}, Hq={cfg.Hq}/Hkv={cfg.Hkv}, D={cfg.D}, {L}{w}, depth {cfg.depth}, "
            f"top-k {cfg.k}, m={cfg.m}, V={cfg.V} {cfg.logits_dtype} logits, {mode} accept")


def step_bytes(cfg, plen, mode):
    """Algorithmic HBM bytes of one step: every input byte read once."""
    eb = 4 if cfg.logits_dtype == "f32" else 2
    draft = cfg.B * cfg.R * cfg.V * eb
    target = cfg.B * (cfg.m + 1) * cfg.V * eb
    kv = sum(2 * cfg.Hkv * min(int(p), cfg.window or int(p)) * cfg.D * 2 for p in plen)
    attn_other = cfg.B * cfg.m * (2 * cfg.Hq + 2 * cfg.Hkv) * cfg.D * 2  # q, out, tree K, tree V
    accept = target + (draft if mode.startswith("stochastic") else 0)
    return {"draft": draft, "attention": kv + attn_other, "kv": kv, "accept": accept,
            "step": draft + kv + attn_other + accept}


def page_caches(torch, kc, vc, ps: int, room: int, seed: int):
    """Dense caches [B][Hkv][L][D] -> pools [num_pages][Hkv][ps][D] whose pages (every sequence's, with room
    for `room` more keys) are shuffled through the pool, and the block table [B][pages_per_seq]."""
    B, Hkv, L, D = kc.shape
    pps = (L + room + ps - 1) // ps
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(B * pps, generator=g).to(kc.device)
    pools = []
    for c in (kc, vc):
        pad = torch.zeros(B, Hkv, pps * ps, D, dtype=c.dtype, device=c.device)
        pad[:, :, :L] = c
        pool = torch.empty(B * pps, Hkv, ps, D, dtype=c.dtype, device=c.device)
        pool[perm] = pad.view(B, Hkv, pps, ps, D).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv, ps, D)
        pools.append(pool)
    return pools[0], pools[1], perm.view(B, pps).to(torch.int32).contiguous()


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm = [float(r[0]) for r in self.rows if len(r) >= 7 and r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if len(r) >= 7 and r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows if len(r) >= 7 for i in range(4) if r[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


def gpu_id_for(torch, dev) -> str:
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")
        return vis[dev.index or 0] if dev.index is not None and dev.index < len(vis) else "0"


# ------------------------------------------------------------ CPU oracle leg
def oracle_step(cfg, seed, mode):
    """One verify step of the CPU oracle on seed `seed` (all B sequences)."""
    import oracle
    stored = gen_draft_logits(cfg, seed)
    x = oracle.decode_logits(stored, cfg.logits_dtype)
    plen = gen_prefix_len(cfg, seed)
    q, kc, vc, kt, vt = gen_attention_inputs(cfg, seed, cfg.L)
    u = gen_uniforms(cfg, seed)
    t0 = time.perf_counter()
    trees = [oracle.build_tree(x[b], cfg.depth, cfg.k, cfg.m) for b in range(cfg.B)]
    t_build = time.perf_counter() - t0
    tgt = oracle.decode_logits(make_target_logits(cfg, seed, stored, np.stack([t["draft_row"] for t in trees])),
                               cfg.logits_dtype)
    t1 = time.perf_counter()
    for b in range(cfg.B):
        _oracle_rest(cfg, mode, trees[b], tgt[b], x[b], q[b], kc[b], vc[b], kt[b], vt[b], int(plen[b]), u[b])
    return t_build + (time.perf_counter() - t1)


def _oracle_rest(cfg, mode, t, tgt, x, q, kc, vc, kt, vt, plen, u):
    """Mask, attention and acceptance of one sequence on the oracle."""
    import oracle
    dec = lambda a: oracle.decode_logits(a, "bf16")
    oracle.pack_mask(oracle.ancestor_mask(t["parents"]))
    oracle.tree_attention(dec(q), dec(kc), dec(vc), plen, dec(kt), dec(vt), t["parents"], t["depth"],
                          window=cfg.window)
    if mode.startswith("stochastic"):
        oracle.accept_stochastic(tgt, x, t["tokens"], t["parents"], t["draft_row"], u.astype(np.float64), cfg.depth,
                                 without_replacement=mode == "stochastic-wor")
    else:
        oracle.accept_greedy(tgt, t["tokens"], t["parents"], cfg.depth)


def cpu_baseline(cfg, mode, budget_s):
    """The oracle, as it stands, on one host thread: whole sequences of the
    workload (tree build, mask, attention, acceptance) until the budget is
    spent, scaled to steps of B sequences.  Input generation is not timed."""
    import oracle
    from threadpoolctl import threadpool_limits
    per_seq, seeds = [], []
    start = time.perf_counter()
    with threadpool_limits(limits=1):
        seed = 0
        while not per_seq or (time.perf_counter() - start < budget_s and len(per_seq) < 64):
            stored = gen_draft_logits(cfg, seed)
            x = oracle.decode_logits(stored, cfg.logits_dtype)
            plen = gen_prefix_len(cfg, seed)
            q, kc, vc, kt, vt = gen_attention_inputs(cfg, seed, cfg.L)
            u = gen_uniforms(cfg, seed)
            trees, t_build = [], []
            for b in range(cfg.B):  # build as many trees as the budget allows (at least one)
                t0 = time.perf_counter()
                trees.append(oracle.build_tree(x[b], cfg.depth, cfg.k, cfg.m))
                t_build.append(time.perf_counter() - t0)
                if time.perf_counter() - start > budget_s / 2:
                    break
            # target rows need every sequence's draft rows: the unsampled ones get the root's row only
            n1 = trees[0]["draft_row"].shape[0]
            drow = np.full((cfg.B, n1), -1, dtype=np.int64)
            drow[:, 0] = 0
            for b, t in enumerate(trees):
                drow[b] = t["draft_row"]
            tgt = oracle.decode_logits(make_target_logits(cfg, seed, stored, drow), cfg.logits_dtype)
            for b, t in enumerate(trees):
                t0 = time.perf_counter()
                _oracle_rest(cfg, mode, t, tgt[b], x[b], q[b], kc[b], vc[b], kt[b], vt[b], int(plen[b]), u[b])
                per_seq.append(t_build[b] + time.perf_counter() - t0)
                if time.perf_counter() - start > budget_s:
                    break
            seeds.append(seed)
            seed += 1
    step_s = float(np.mean(per_seq)) * cfg.B
    return {"value": round(1.0 / step_s, 4), "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(per_seq)} sequences of the {cfg.name} workload (seeds {seeds[0]}..{seeds[-1]}), each "
                      f"tree build + mask + attention + {mode} acceptance on the numpy fp64 oracle, 1 host thread; "
                      f"mean time per sequence x B={cfg.B} = one step; input generation not timed"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = get_config(args.config)
    from threadpoolctl import threadpool_limits
    budget = max(5.0, min(60.0, args.cpu_seconds))
    times = []
    with threadpool_limits(limits=1):
        for i in range(args.warmup + args.steps):
            t = oracle_step(cfg, i, args.mode)
            if i >= args.warmup:
                times.append(t)
            if sum(times) > budget and len(times) >= 1:
                break
    per = sum(times) / len(times)
    v = 1.0 / per
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "steps/s",
            "n_gpus": args.gpus, "steps": len(times), "warmup": args.warmup, "ms_per_step": round(per * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(cfg, args.mode)},
            "cpu_baseline": {"value": round(v, 4), "unit": "steps/s", "cores": 1, "kind": "oracle",
                             "sample": f"{len(times)} full steps after {args.warmup} warm-up (bounded to ~{budget:.0f} s), "
                                       f"numpy fp64, 1 host thread"},
            "e2e": {"value": round(v, 4), "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------- multi-rank helpers
def rank_env():
    """(world, rank, local_rank) of this process, as torchrun sets them (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def input_seed(rank: int, i: int) -> int:
    """Seed of input set i on a rank: every rank works on its own sequences."""
    return 1000 * rank + i


def max_over_ranks(values, dist, device):
    """Element-wise maximum of a list of floats over all ranks (the slowest rank
    sets every time); returns the list unchanged when running alone."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(world: int, ms_per_step: float) -> float:
    """Steps per second of the whole job: every rank completes one step of its
    own batch per ms_per_step (the max over ranks)."""
    return world * 1000.0 / ms_per_step


# ------------------------------------------------------------------ GPU leg
def attn_flops(cfg, plen):
    """4 * Hq * n * D per visible prefix key (QK^T and PV), unpadded rows; the tree block is left out."""
    keys = sum(min(int(p), cfg.window or int(p)) for p in plen)
    return 4 * cfg.Hq * cfg.m * cfg.D * keys


def attn_source_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("attention_tc.cu", "sm100_ptx.cuh", "attention.cu"):
        with open(os.path.join(ROOT, "eagle_tree_verification_dynamic_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# DRAM bytes (read + write) of one launch of the tree attention's main kernel,
# from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) on the named
# workload, valid only for the kernel sources whose digest is the key: after any
# change to the kernel the entry no longer matches and `traffic` reads null
# until a new capture is taken.
ATTN_TRAFFIC_BYTES = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum -k regex:attn_tc_kernel
    #     -s 8 -c 1 on `bench.py --config <name> --steps 3 --warmup 3 --no-cpu-baseline --no-per-config`
    ("7b", 0, "f5510cc048b9f0a0"): 35111936 + 0,
    ("l3-8b", 0, "f5510cc048b9f0a0"): 204041984 + 5385472,
    ("serve", 0, "f5510cc048b9f0a0"): 309454080 + 13574400,
    ("long", 0, "f5510cc048b9f0a0"): 194805504 + 3845632,
    # the serving mix over a paged cache (`--paged 64` / `--paged 16` added to the command above);
    # ncu printed these two in MB with two decimals, so they are rounded to 10 kB
    ("serve", 64, "f5510cc048b9f0a0"): 309370000 + 13850000,
    ("serve", 16, "f5510cc048b9f0a0"): 309470000 + 13980000,
}


def load_peaks():
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    src = "measured" if "hbm_gbs" in peaks else "fallback"
    return (float(peaks.get("hbm_gbs", 6650.0)), float(peaks.get("bf16_tflops", 1590.0)), src)


class Bench:
    """Rotating input sets of one workload, their step objects and CUDA graphs."""

    def __init__(self, torch, cfg, mode, dev, rank, paged=0):
        from eagle_tree_verification_dynamic_b200.step import StepShape, VerifyStep
        self.torch, self.cfg, self.mode, self.dev = torch, cfg, mode, dev
        stoch = mode.startswith("stochastic")
        tdt = torch.float32 if cfg.logits_dtype == "f32" else torch.bfloat16

        def to_logits(a):
            if cfg.logits_dtype == "f32":
                return torch.from_numpy(a).to(dev)
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

        def to_bf16(a):
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

        ps = paged
        pps = (cfg.L + cfg.depth + ps - 1) // ps if ps else 0
        shape = StepShape(B=cfg.B, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, Lmax=pps * ps if ps else cfg.L, depth=cfg.depth,
                          k=cfg.k, m=cfg.m, V=cfg.V, logits_dtype=tdt, window=cfg.window, stochastic=stoch,
                          without_replacement=mode == "stochastic-wor", paged=ps > 0)
        sb0 = step_bytes(cfg, gen_prefix_len(cfg, 0), mode)
        self.n_sets = min(16, max(3, int(np.ceil(2.2 * L2_BYTES / sb0["step"]))))
        self.sets, self.hosts, self.steps = [], [], []
        for i in range(self.n_sets):
            seed = input_seed(rank, i)
            stored = gen_draft_logits(cfg, seed)
            plen = gen_prefix_len(cfg, seed)
            q, kc, vc, kt, vt = gen_attention_inputs(cfg, seed, cfg.L)
            inp = {"draft_logits": to_logits(stored), "prefix_len": torch.from_numpy(plen).to(dev),
                   "q": to_bf16(q), "k_cache": to_bf16(kc), "v_cache": to_bf16(vc), "k_tree": to_bf16(kt),
                   "v_tree": to_bf16(vt), "uniforms": torch.from_numpy(gen_uniforms(cfg, seed)).to(dev)}
            if ps:
                inp["k_cache"], inp["v_cache"], inp["block_table"] = page_caches(torch, inp["k_cache"],
                                                                                 inp["v_cache"], ps, cfg.depth, seed)
            st = VerifyStep(shape, dev)
            st.build(inp["draft_logits"])
            torch.cuda.synchronize()
            tgt = make_target_logits(cfg, seed, stored, st.tree.draft_row.cpu().numpy())
            inp["target_logits"] = to_logits(tgt)
            self.sets.append(inp)
            self.steps.append(st)
            self.hosts.append({k: v.cpu().pin_memory() for k, v in inp.items()
                               if k not in ("k_cache", "v_cache", "block_table")})
        self.set_bytes = sum(sum(t.numel() * t.element_size() for t in s.values()) for s in self.sets)
        self.flush_between = self.set_bytes < 2 * L2_BYTES
        self.flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if self.flush_between else None
        self.stream = torch.cuda.Stream(dev)
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            for st, inp in zip(self.steps, self.sets):  # eager warm-up (sets kernel attributes)
                st(inp)
                st.fused(inp)
        self.stream.synchronize()
        for st in self.steps:
            st.fused_attention_status()
        self.launch_mode = "torch replay"
        try:
            from cuda.bindings import runtime as cudart
        except Exception:  # pragma: no cover
            cudart = None
        self.cudart = cudart

    def capture(self, fn):
        """One CUDA graph of fn; launched with cudaGraphLaunch when available (torch's replay also
        refreshes its RNG state with a small fill kernel, which would land in the timed region)."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            fn()
        if self.cudart is not None:
            try:
                exec_h = g.raw_cuda_graph_exec()
                st_h = self.stream.cuda_stream
                err = self.cudart.cudaGraphLaunch(exec_h, st_h)[0]
                if int(err) == 0:
                    self.stream.synchronize()
                    self.launch_mode = "cudaGraphLaunch"
                    g._eagle_launch = lambda e=exec_h, h=st_h: self.cudart.cudaGraphLaunch(e, h)
                    return g
            except Exception:
                pass
        g._eagle_launch = g.replay
        return g

    def graphs(self, f):
        return [self.capture(lambda st=st, inp=inp: f(st, inp)) for st, inp in zip(self.steps, self.sets)]

    def timed(self, gs, K, W, barrier=lambda: None):
        """Mean device time (ms) of one launch, CUDA events on the launching stream.  Input sets rotate;
        a workload whose sets fit in twice the L2 cache flushes L2 (a 252 MiB write) before every
        timed launch, outside the event pair."""
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for i in range(W):
                gs[i % len(gs)]._eagle_launch()
        self.stream.synchronize()
        barrier()
        torch.cuda.synchronize()
        if not self.flush_between:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(self.stream):
                e0.record(self.stream)
                for i in range(K):
                    gs[i % len(gs)]._eagle_launch()
                e1.record(self.stream)
            self.stream.synchronize()
            torch.cuda.synchronize()
            barrier()
            return e0.elapsed_time(e1) / K
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        with torch.cuda.stream(self.stream):
            for i in range(K):
                self.flush_buf.fill_(float(i))
                ev[i][0].record(self.stream)
                gs[i % len(gs)]._eagle_launch()
                ev[i][1].record(self.stream)
        self.stream.synchronize()
        torch.cuda.synchronize()
        barrier()
        return sum(a.elapsed_time(b) for a, b in ev) / K

    def l2_note(self):
        if self.flush_between:
            return (f"{self.n_sets} rotating input sets ({self.set_bytes / 2**20:.1f} MiB, under 2x L2): "
                    f"L2 flushed by a 252 MiB write before every timed step, outside the timed interval")
        return f"{self.n_sets} rotating input sets, {self.set_bytes / 2**20:.0f} MiB > 2x L2"


STAGES = {
    "build": lambda st, inp: st.build(inp["draft_logits"]),
    "draft_sweep": lambda st, inp: st.draft_sweep(inp["draft_logits"]),
    "mask": lambda st, inp: st.mask_(inp["prefix_len"]),
    "attention": lambda st, inp: st.attention(inp["q"], inp["k_cache"], inp["v_cache"], inp["prefix_len"],
                                              inp["k_tree"], inp["v_tree"], inp.get("block_table")),
    "accept": lambda st, inp: st.accept(inp["target_logits"], inp["uniforms"], inp["draft_logits"]),
    "accept_sweep": lambda st, inp: st.accept_sweep(inp["target_logits"]),
}


def rooflines(cfg, mode, ms, stage_ms, hbm_peak, tc_peak, peak_src, traffic_key):
    """Roofline figures of one workload: the tree attention (slower of its bytes at the copy bandwidth and
    its flops at the bf16 peak), the acceptance's target sweep (bytes at the copy bandwidth) and the step."""
    plen = gen_prefix_len(cfg, 0)
    sb = step_bytes(cfg, plen, mode)
    fl = attn_flops(cfg, plen)
    t_attn = stage_ms["attention"] * 1e-3
    t_hbm, t_tc = sb["attention"] / (hbm_peak * 1e9), fl / (tc_peak * 1e12)
    if t_hbm >= t_tc:
        ach, peak, unit, bound = sb["attention"] / t_attn / 1e9, hbm_peak, "GB/s", "hbm"
    else:
        ach, peak, unit, bound = fl / t_attn / 1e12, tc_peak, "TFLOP/s", "tensor"
    traffic = ATTN_TRAFFIC_BYTES.get(traffic_key)
    attn = {"kernel": "tree attention (split-KV main + combine)", "bound": bound, "achieved": round(ach, 2),
            "peak": peak, "unit": unit, "frac": round(max(t_hbm, t_tc) / t_attn, 4), "traffic": traffic,
            "peak_source": f"{peak_src} ({'copy bandwidth' if bound == 'hbm' else 'cuBLAS bf16 GEMM'}, burst)",
            "algorithmic_bytes": sb["attention"], "flops": fl, "t_roof_us": round(max(t_hbm, t_tc) * 1e6, 3),
            "gbs": round(sb["attention"] / t_attn / 1e9, 1), "tflops": round(fl / t_attn / 1e12, 1)}
    sweep_bytes = cfg.B * (cfg.m + 1) * cfg.V * (4 if cfg.logits_dtype == "f32" else 2)
    t_sw = stage_ms["accept_sweep"] * 1e-3
    sweep = {"kernel": "acceptance vocab sweep (argmax + log-sum-exp of every target row)", "bound": "hbm",
             "achieved": round(sweep_bytes / t_sw / 1e9, 1), "peak": hbm_peak, "unit": "GB/s",
             "frac": round(sweep_bytes / t_sw / 1e9 / hbm_peak, 4), "algorithmic_bytes": sweep_bytes,
             "peak_source": f"{peak_src} copy bandwidth (burst)"}
    t_step = max(sb["step"] / (hbm_peak * 1e9), t_tc)
    step = {"bytes": sb["step"], "flops": fl, "t_min_us": round(t_step * 1e6, 3),
            "frac": round(t_step / (ms * 1e-3), 4)}
    return attn, sweep, step, sb


def measure(torch, cfg, mode, dev, rank, K, W, barrier, paged=0, e2e=False, compact=False, clocks=None):
    """Time one workload: the whole step (one eagle_verify_step call per graph), each stage, and
    optionally the KV compaction after it and the end-to-end step with host copies."""
    import eagle_tree_verification_dynamic_b200 as et
    bn = Bench(torch, cfg, mode, dev, rank, paged)
    graphs = bn.graphs(lambda st, inp: st.fused(inp))
    stage_graphs = {name: bn.graphs(f) for name, f in STAGES.items()}
    res = {"n_sets": bn.n_sets, "l2": bn.l2_note()}
    if clocks is not None:
        with clocks:
            res["ms"] = bn.timed(graphs, K, W, barrier)
    else:
        res["ms"] = bn.timed(graphs, K, W, barrier)
    for st in bn.steps:  # every timed step's attention finished without a device error
        st.fused_attention_status()
    res["stage_ms"] = {name: bn.timed(gs, K, W, barrier) for name, gs in stage_graphs.items()}
    res["launch_mode"] = bn.launch_mode
    acc_now = [int(st.accepted_len.sum()) for st in bn.steps]
    res["accepted_mean"] = sum(acc_now) / len(acc_now)
    if compact:
        # the row after the step: compaction of each input set's accepted path into copies of its caches
        # with room past the prefix (the workloads fill theirs)
        def room(t):
            return torch.cat([t, torch.zeros_like(t[:, :, :cfg.depth])], dim=2).contiguous()
        if paged:  # the pools already hold a page past each prefix
            cc = [(inp["k_cache"].clone(), inp["v_cache"].clone(), torch.empty_like(inp["prefix_len"]))
                  for inp in bn.sets]
            cg = [bn.capture(lambda st=st, inp=inp, c=c: et.kv_compact_paged_into(
                inp["k_tree"], inp["v_tree"], st.path, st.accepted_len, inp["prefix_len"], c[0], c[1],
                inp["block_table"], c[2])) for st, inp, c in zip(bn.steps, bn.sets, cc)]
        else:
            cc = [(room(inp["k_cache"]), room(inp["v_cache"]), torch.empty_like(inp["prefix_len"])) for inp in bn.sets]
            cg = [bn.capture(lambda st=st, inp=inp, c=c: et.kv_compact_into(
                inp["k_tree"], inp["v_tree"], st.path, st.accepted_len, inp["prefix_len"], c[0], c[1], c[2]))
                for st, inp, c in zip(bn.steps, bn.sets, cc)]
        res["compact_ms"] = bn.timed(cg, K, W, barrier)
        res["compact_bytes"] = 2 * 2 * res["accepted_mean"] * cfg.Hkv * cfg.D * 2  # K+V, read+write, bf16
        del cc, cg
    if e2e:
        # end to end through the public API: per-step inputs copied from pinned host memory, results read
        # back; the KV cache stays resident on the device
        h2d = sum(t.numel() * t.element_size() for t in bn.hosts[0].values())
        out_host = [torch.empty(s.numel(), dtype=torch.int32).pin_memory()
                    for s in (bn.steps[0].accepted_len, bn.steps[0].path, bn.steps[0].bonus)]
        d2h = sum(t.numel() * 4 for t in out_host)

        # Double-buffered like a serving loop: step i's inputs go up on a copy stream while step i - 1
        # computes; a step waits for its own copies, and a set's buffers are overwritten only after the
        # step that last read them.  Every step's copies and its readback are inside the timed region.
        copy_stream = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(bn.n_sets)]
        used = [torch.cuda.Event() for _ in range(bn.n_sets)]
        used_once = [False] * bn.n_sets

        def e2e_once(i):
            j = i % bn.n_sets
            with torch.cuda.stream(copy_stream):
                if used_once[j]:
                    copy_stream.wait_event(used[j])
                for k, hv in bn.hosts[j].items():
                    bn.sets[j][k].copy_(hv, non_blocking=True)
                copied[j].record(copy_stream)
            bn.stream.wait_event(copied[j])
            graphs[j]._eagle_launch()
            used[j].record(bn.stream)
            used_once[j] = True
            for hb, dv in zip(out_host, (bn.steps[j].accepted_len, bn.steps[j].path, bn.steps[j].bonus)):
                hb.copy_(dv.reshape(-1), non_blocking=True)

        with torch.cuda.stream(bn.stream):
            for i in range(W):
                e2e_once(i)
        bn.stream.synchronize()
        copy_stream.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(bn.stream):
            e0.record(bn.stream)
            copy_stream.wait_event(e0)  # the first copies start inside the timed region
            for i in range(K):
                e2e_once(i)
            e1.record(bn.stream)
        bn.stream.synchronize()
        copy_stream.synchronize()
        barrier()
        res["e2e_ms"] = e0.elapsed_time(e1) / K
        res["h2d"], res["d2h"] = h2d, d2h
    del graphs, stage_graphs, bn
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


# the other workloads reported beside the headline, each with its acceptance mode
PER_CONFIG = [("tiny", "greedy", 0), ("7b", "greedy", 0), ("l3-8b", "stochastic", 0), ("long", "greedy", 0),
              ("long-window", "greedy", 0), ("serve", "stochastic", 0),
              # the serving mix over a paged prefix cache (page size in keys)
              ("serve", "stochastic", 64), ("serve", "stochastic", 16)]


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    cfg = get_config(args.config)
    hbm_peak, tc_peak, peak_src = load_peaks()
    digest = attn_source_digest()
    ps = args.paged
    K, W = args.steps, max(3, args.warmup)

    clk = ClockSampler(gpu_id_for(torch, dev))
    r = measure(torch, cfg, args.mode, dev, rank, K, W, barrier, paged=ps, e2e=True, compact=True, clocks=clk)
    clocks = clk.summary()
    names = list(STAGES)
    red = max_over_ranks([r["ms"], r["e2e_ms"], r["compact_ms"]] + [r["stage_ms"][k] for k in names],
                         dist if world > 1 else None, dev)
    ms, ms_e2e, compact_ms = red[0], red[1], red[2]
    stage_ms = {k: red[3 + i] for i, k in enumerate(names)}
    attn, sweep, step_rf, sb = rooflines(cfg, args.mode, ms, stage_ms, hbm_peak, tc_peak, peak_src,
                                         (cfg.name, ps, digest))
    stages = {k: {"ms": round(v, 5)} for k, v in stage_ms.items()}
    stages["build"]["gbs"] = round(sb["draft"] / (stage_ms["build"] * 1e-3) / 1e9, 1)
    stages["draft_sweep"]["gbs"] = round(sb["draft"] / (stage_ms["draft_sweep"] * 1e-3) / 1e9, 1)
    stages["attention"]["gbs"] = attn["gbs"]
    stages["accept"]["gbs"] = round(sb["accept"] / (stage_ms["accept"] * 1e-3) / 1e9, 1)
    stages["accept_sweep"]["gbs"] = sweep["achieved"]
    stages["kv_compact"] = {"ms": round(compact_ms, 5),
                            "gbs": round(r["compact_bytes"] / (compact_ms * 1e-3) / 1e9, 1),
                            "note": "after the step, not part of it: the accepted path's K/V into the cache"}
    line = {
        "metric": METRIC,
        "value": round(whole_job_rate(world, ms), 2), "unit": "steps/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 attention (fp32 accumulate), " + cfg.logits_dtype + " logits",
        "data": "synthetic (seeded; no weights or datasets)",
        "config": {"workload": workload_desc(cfg, args.mode) + (f", paged KV cache ({ps}-key pages)" if ps else ""),
                   "l2": r["l2"],
                   "graph": f"each step one eagle_verify_step call, as one CUDA graph ({r['launch_mode']})",
                   "parallelism": f"replicas x{world}"},
        "kv_hbm_gbs": round(sb["kv"] / (stage_ms["attention"] * 1e-3) / 1e9, 1),
        "stages": stages,
        "roofline": attn,
        "accept_sweep_roofline": sweep,
        "step_roofline": step_rf,
        "e2e": {"value": round(whole_job_rate(world, ms_e2e), 2), "unit": "steps/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clocks,
        "attention_source": digest,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.mode, args.cpu_seconds)
    if not args.no_per_config and not ps and args.config == "7b" and world == 1:
        per = {}
        Kc = max(20, K // 4)
        for name, mode, pg in PER_CONFIG:
            c = get_config(name)
            rc = measure(torch, c, mode, dev, rank, Kc, W, barrier, paged=pg)
            a2, s2, st2, sb2 = rooflines(c, mode, rc["ms"], rc["stage_ms"], hbm_peak, tc_peak, peak_src,
                                         (name, pg, digest))
            desc = workload_desc(c, mode) + (f", paged KV cache ({pg}-key pages)" if pg else "")
            entry = {"workload": desc, "steps": Kc, "l2": rc["l2"],
                     "ms_per_step": round(rc["ms"], 5), "steps_per_s": round(1000.0 / rc["ms"], 2),
                     "stages_ms": {k: round(v, 5) for k, v in rc["stage_ms"].items()},
                     "roofline": a2, "accept_sweep_roofline": s2, "step_roofline": st2,
                     "accepted_mean": rc["accepted_mean"]}
            if not args.no_cpu_baseline and not pg:  # (the oracle's work does not depend on the paging)
                entry["cpu_baseline"] = cpu_baseline(c, mode, args.cpu_seconds_per_config)
            per[f"{name} {mode}" + (f" paged{pg}" if pg else "")] = entry
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
