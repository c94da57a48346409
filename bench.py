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

# DRAM bytes (read + write) of one launch of the tree attention's main kernel,
# from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of this
# kernel version on the named workload; a workload without a capture reports null.
ATTN_TRAFFIC_BYTES = {"7b": 35108352 + 0}


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
    dec = lambda a: oracle.decode_logits(a, "bf16")
    t1 = time.perf_counter()
    for b in range(cfg.B):
        t = trees[b]
        oracle.pack_mask(oracle.ancestor_mask(t["parents"]))
        oracle.tree_attention(dec(q[b]), dec(kc[b]), dec(vc[b]), int(plen[b]), dec(kt[b]), dec(vt[b]),
                              t["parents"], t["depth"], window=cfg.window)
        if mode.startswith("stochastic"):
            oracle.accept_stochastic(tgt[b], x[b], t["tokens"], t["parents"], t["draft_row"],
                                     u[b].astype(np.float64), cfg.depth, without_replacement=mode == "stochastic-wor")
        else:
            oracle.accept_greedy(tgt[b], t["tokens"], t["parents"], cfg.depth)
    return t_build + (time.perf_counter() - t1)


def cpu_baseline(cfg, mode, budget_s):
    from threadpoolctl import threadpool_limits
    times = []
    with threadpool_limits(limits=1):
        start = time.perf_counter()
        seed = 0
        while not times or (time.perf_counter() - start < budget_s and len(times) < 50):
            times.append(oracle_step(cfg, seed, mode))
            seed += 1
    per = sum(times) / len(times)
    return {"value": round(1.0 / per, 4), "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(times)} full {cfg.name} steps (seeds 0..{len(times) - 1}), input generation "
                      f"excluded, numpy fp64 on 1 host thread"}


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
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import eagle_tree_verification_dynamic_b200 as et
    from eagle_tree_verification_dynamic_b200.step import StepShape, VerifyStep

    world, rank, local = rank_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    cfg = get_config(args.config)
    stoch = args.mode.startswith("stochastic")
    tdt = torch.float32 if cfg.logits_dtype == "f32" else torch.bfloat16

    def to_logits(a):
        if cfg.logits_dtype == "f32":
            return torch.from_numpy(a).to(dev)
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    def to_bf16(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    ps = args.paged
    pps = (cfg.L + cfg.depth + ps - 1) // ps if ps else 0
    shape = StepShape(B=cfg.B, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, Lmax=pps * ps if ps else cfg.L, depth=cfg.depth,
                      k=cfg.k, m=cfg.m, V=cfg.V, logits_dtype=tdt, window=cfg.window, stochastic=stoch,
                      without_replacement=args.mode == "stochastic-wor", paged=ps > 0)

    # input sets: enough distinct sets that their bytes exceed 2x L2
    sb0 = step_bytes(cfg, gen_prefix_len(cfg, 0), args.mode)
    n_sets = max(3, int(np.ceil(2.2 * L2_BYTES / sb0["step"])))
    n_sets = min(n_sets, 16)
    sets, hosts, steps = [], [], []
    for i in range(n_sets):
        seed = input_seed(rank, i)
        stored = gen_draft_logits(cfg, seed)
        plen = gen_prefix_len(cfg, seed)
        q, kc, vc, kt, vt = gen_attention_inputs(cfg, seed, cfg.L)
        inp = {"draft_logits": to_logits(stored), "prefix_len": torch.from_numpy(plen).to(dev),
               "q": to_bf16(q), "k_cache": to_bf16(kc), "v_cache": to_bf16(vc), "k_tree": to_bf16(kt),
               "v_tree": to_bf16(vt), "uniforms": torch.from_numpy(gen_uniforms(cfg, seed)).to(dev)}
        if ps:
            inp["k_cache"], inp["v_cache"], inp["block_table"] = page_caches(torch, inp["k_cache"], inp["v_cache"],
                                                                             ps, cfg.depth, seed)
        st = VerifyStep(shape, dev)
        st.build(inp["draft_logits"])
        torch.cuda.synchronize()
        tgt = make_target_logits(cfg, seed, stored, st.tree.draft_row.cpu().numpy())
        inp["target_logits"] = to_logits(tgt)
        sets.append(inp)
        steps.append(st)
        hosts.append({k: v.cpu().pin_memory() for k, v in inp.items()
                      if k not in ("k_cache", "v_cache", "block_table")})
    set_bytes = sum(sum(t.numel() * t.element_size() for t in s.values()) for s in sets)

    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for st, inp in zip(steps, sets):      # eager warm-up (sets kernel attributes)
            st(inp)
            st.fused(inp)
    stream.synchronize()
    for st in steps:
        st.fused_attention_status()

    # Replaying a torch graph also refreshes torch's RNG state with a small fill
    # kernel; launching the instantiated graph directly keeps the timed region
    # to the step's own kernels.
    launch_mode = ["torch replay"]
    try:
        from cuda.bindings import runtime as cudart
    except Exception:  # pragma: no cover
        cudart = None

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        if cudart is not None:
            try:
                exec_h = g.raw_cuda_graph_exec()
                st_h = stream.cuda_stream
                err = cudart.cudaGraphLaunch(exec_h, st_h)[0]
                if int(err) == 0:
                    stream.synchronize()
                    launch_mode[0] = "cudaGraphLaunch"
                    g._eagle_launch = lambda e=exec_h, h=st_h: cudart.cudaGraphLaunch(e, h)
                    return g
            except Exception:
                pass
        g._eagle_launch = g.replay
        return g

    graphs = [capture(lambda st=st, inp=inp: st.fused(inp)) for st, inp in zip(steps, sets)]
    stage_fns = {
        "build": lambda st, inp: st.build(inp["draft_logits"]),
        "mask": lambda st, inp: st.mask_(inp["prefix_len"]),
        "attention": lambda st, inp: st.attention(inp["q"], inp["k_cache"], inp["v_cache"], inp["prefix_len"],
                                                  inp["k_tree"], inp["v_tree"], inp.get("block_table")),
        "accept": lambda st, inp: st.accept(inp["target_logits"], inp["uniforms"], inp["draft_logits"]),
    }
    stage_graphs = {name: [capture(lambda st=st, inp=inp, f=f: f(st, inp)) for st, inp in zip(steps, sets)]
                    for name, f in stage_fns.items()}

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(gs, K, W):
        with torch.cuda.stream(stream):
            for i in range(W):
                gs[i % len(gs)]._eagle_launch()
        stream.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(K):
                gs[i % len(gs)]._eagle_launch()
            e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        barrier()
        return e0.elapsed_time(e1) / K

    K, W = args.steps, max(3, args.warmup)
    with ClockSampler(gpu_id_for(torch, dev)) as clk:
        ms = timed(graphs, K, W)
    clocks = clk.summary()
    for st in steps:  # every timed step's attention finished without a device error
        st.fused_attention_status()
    stage_ms = {name: timed(gs, K, W) for name, gs in stage_graphs.items()}

    # the row after the step: compaction of each input set's accepted path into
    # copies of its caches with room past the prefix (the workloads fill theirs)
    def room(t):
        return torch.cat([t, torch.zeros_like(t[:, :, :cfg.depth])], dim=2).contiguous()
    if ps:  # the pools already hold a page past each prefix
        cc = [(inp["k_cache"].clone(), inp["v_cache"].clone(), torch.empty_like(inp["prefix_len"])) for inp in sets]
        comp_graphs = [capture(lambda st=st, inp=inp, c=c: et.kv_compact_paged_into(
            inp["k_tree"], inp["v_tree"], st.path, st.accepted_len, inp["prefix_len"], c[0], c[1],
            inp["block_table"], c[2])) for st, inp, c in zip(steps, sets, cc)]
    else:
        cc = [(room(inp["k_cache"]), room(inp["v_cache"]), torch.empty_like(inp["prefix_len"])) for inp in sets]
        comp_graphs = [capture(lambda st=st, inp=inp, c=c: et.kv_compact_into(
            inp["k_tree"], inp["v_tree"], st.path, st.accepted_len, inp["prefix_len"], c[0], c[1], c[2]))
            for st, inp, c in zip(steps, sets, cc)]
    compact_ms = timed(comp_graphs, K, W)
    torch.cuda.synchronize()
    acc_now = [int(st.accepted_len.sum()) for st in steps]
    compact_bytes = 2 * 2 * (sum(acc_now) / len(acc_now)) * cfg.Hkv * cfg.D * 2  # K+V, read+write, bf16
    del cc, comp_graphs

    # end to end through the public API: per-step inputs copied from pinned host
    # memory, results read back; the KV cache stays resident on the device
    h2d = sum(t.numel() * t.element_size() for t in hosts[0].values())
    out_host = [torch.empty(s.numel(), dtype=torch.int32).pin_memory() for s in (steps[0].accepted_len, steps[0].path,
                                                                                 steps[0].bonus)]
    d2h = sum(t.numel() * 4 for t in out_host)

    def e2e_once(i):
        j = i % n_sets
        for k, hv in hosts[j].items():
            sets[j][k].copy_(hv, non_blocking=True)
        graphs[j]._eagle_launch()
        for hb, dv in zip(out_host, (steps[j].accepted_len, steps[j].path, steps[j].bonus)):
            hb.copy_(dv.reshape(-1), non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(W):
            e2e_once(i)
    stream.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K):
            e2e_once(i)
        e1.record(stream)
    stream.synchronize()
    barrier()
    ms_e2e = e0.elapsed_time(e1) / K

    red = max_over_ranks([ms, ms_e2e, compact_ms] + [stage_ms[k] for k in stage_fns], dist if world > 1 else None,
                         dev)
    ms, ms_e2e, compact_ms = red[0], red[1], red[2]
    stage_ms = {k: red[3 + i] for i, k in enumerate(stage_fns)}

    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"

    sb = step_bytes(cfg, gen_prefix_len(cfg, 0), args.mode)
    attn_gbs = sb["attention"] / (stage_ms["attention"] * 1e-3) / 1e9
    value = whole_job_rate(world, ms)
    stages = {k: {"ms": round(v, 5)} for k, v in stage_ms.items()}
    stages["build"]["gbs"] = round(sb["draft"] / (stage_ms["build"] * 1e-3) / 1e9, 1)
    stages["attention"]["gbs"] = round(attn_gbs, 1)
    stages["accept"]["gbs"] = round(sb["accept"] / (stage_ms["accept"] * 1e-3) / 1e9, 1)
    stages["kv_compact"] = {"ms": round(compact_ms, 5), "gbs": round(compact_bytes / (compact_ms * 1e-3) / 1e9, 1),
                            "note": "after the step, not part of it: the accepted path's K/V into the cache"}

    line = {
        "metric": METRIC,
        "value": round(value, 2), "unit": "steps/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 attention (fp32 accumulate), " + cfg.logits_dtype + " logits",
        "data": "synthetic (seeded; no weights or datasets)",
        "config": {"workload": workload_desc(cfg, args.mode) + (f", paged KV cache ({ps}-key pages)" if ps else ""),
                   "l2": f"{n_sets} rotating input sets, {set_bytes / 2**20:.0f} MiB > 2x L2",
                   "graph": f"each step one eagle_verify_step call, as one CUDA graph ({launch_mode[0]})",
                   "parallelism": f"replicas x{world}"},
        "kv_hbm_gbs": round(sb["kv"] / (stage_ms["attention"] * 1e-3) / 1e9, 1),
        "stages": stages,
        "roofline": {"kernel": "tree attention (split-KV + combine)", "bound": "hbm",
                     "achieved": round(attn_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(attn_gbs / hbm_peak, 4), "traffic": ATTN_TRAFFIC_BYTES.get(cfg.name),
                     "peak_source": f"{peak_src} copy bandwidth (burst)",
                     "algorithmic_bytes": sb["attention"]},
        "step_roofline": {"bytes": sb["step"], "t_min_us": round(sb["step"] / hbm_peak / 1e3, 3),
                          "frac": round(sb["step"] / hbm_peak / 1e3 / (ms * 1e3), 4)},
        "e2e": {"value": round(whole_job_rate(world, ms_e2e), 2), "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.mode, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs, stage_graphs
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
