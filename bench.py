#!/usr/bin/env python
"""Benchmark of the rolling-window chunk attention path on B200.

One step = one chunk of one layer, the whole hot path: four denoise reads
(chunk attention over sinks + window + chunk, with the flow x0 / renoise
epilogue fused into the output store, sigma = 1.0, 0.75, 0.5, 0.25) and the
clean t=0 commit (chunk attention plus the K/V write-back into the ring).
RoPE (relative or absolute) runs on the way in. Inputs are synthetic (seeded
counter-based generator), resident in HBM before timing; the cache is rolled
to steady state (full window, evictions firing) before warm-up.

Metric: query tokens / s per layer (5 * Lq per layer per step), whole job over all ranks.
Multi-GPU: independent replicas (one layer each), no data-path collective.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 720p|480p|abot|long|abot_cfg] [--impl rkv|reference]

The default workload is the 720p one (the largest that fits one GPU); the line also carries
compact records of the ABot and 480P workloads (``workloads``). ``--gpus N`` outside a
launcher starts N ranks under torch.distributed.run itself.

``--config abot_cfg`` measures the guided (classifier-free guidance) mode instead: two caches,
40 guided steps per chunk with the guidance combine fused into the unconditional read.
``--config long`` stacks the ABot layer 30 deep (one cache per layer): each step is one chunk
through all 30 layers.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "query tokens/s per layer; attn TFLOP/s as % of B200 dense BF16 peak"
UNIT = "query tokens/s"

CONFIGS = {
    "abot": dict(workload="ABot-style relative RoPE: 1 layer, H=24, d=128, 880 tokens/frame (22x40 grid), "
                          "chunk 3 frames (2640 queries), window 21 frames (18480 keys), 5 sink reference frames, "
                          "4 denoise reads (fused x0/renoise) + 1 commit per chunk",
                 H=24, gh=22, gw=40, C=3, W=21, S=5, refs=5, mode=1, rollout_chunks=64),
    "480p": dict(workload="LingBot-style 480P: 1 layer, H=40, d=128, 1560 tokens/frame (30x52 grid), chunk 4 frames "
                          "(6240 queries), window 18 frames (28080 keys), sink 6, absolute RoPE, "
                          "4 denoise reads (fused x0/renoise) + 1 commit per chunk",
                 H=40, gh=30, gw=52, C=4, W=18, S=6, refs=0, mode=0, rollout_chunks=22),
    "720p": dict(workload="720p: 1 layer, H=40, d=128, 3600 tokens/frame (45x80 grid), chunk 4 frames (14400 queries), "
                          "window 18 frames (64800 keys), sink 6, absolute RoPE, fused x0/renoise on the "
                          "[14400 x 5120] latent, 4 denoise reads + 1 commit per chunk",
                 H=40, gh=45, gw=80, C=4, W=18, S=6, refs=0, mode=0, rollout_chunks=30),
}
# the long-rollout stress shape: the ABot layer stacked 30 deep, one rolling cache per layer,
# every step = one chunk through all layers (the layers reuse one seeded input set per call;
# the caches, 6.8 GB in all, are per layer)
CONFIGS["long"] = dict(CONFIGS["abot"], layers=30, workload=(
    "Long rollout stress: ABot shape (H=24, d=128, 880 tokens/frame, chunk 3 frames, window 21 frames, 5 sink "
    "reference frames, relative RoPE) stacked 30 layers with one rolling cache each; each step is one chunk "
    "through all 30 layers, 4 denoise reads (fused x0/renoise) + 1 commit per layer"))
# classifier-free guidance (causal pre-training mode): a second cache per layer for the
# unconditional branch, 40 guided steps per chunk, guidance scale 5.0
CFG_CONFIGS = {
    "abot_cfg": dict(CONFIGS["abot"], workload=(
        "ABot-style shape in the guided causal pre-training mode: 1 layer, two rolling caches (conditional, "
        "unconditional), H=24, d=128, 880 tokens/frame (22x40 grid), chunk 3 frames (2640 queries), window 21 "
        "frames (18480 keys), 5 sink reference frames, relative RoPE; per chunk 40 guided steps (conditional read, "
        "then unconditional read with the guidance combine and x0 / renoise fused, scale 5.0) + 2 commits")),
}
CFG_SCALE = 5.0
CFG_STEPS = 40
SIGMAS = [1.0, 0.75, 0.5, 0.25]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# every source file the attention kernel is compiled from
ATTN_SRCS = [os.path.join(ROOT, "rolling_kv_chunked_b200", "csrc", f)
             for f in ("rkv_attention.cu", "numeric.cuh", "ptx_sm100.cuh", "rkv_internal.h")]


def attention_source_sha256():
    import hashlib
    h = hashlib.sha256()
    for path in ATTN_SRCS:
        with open(path, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(config_name):
    """(DRAM bytes per attention launch, where from, the launch's algorithmic bytes) from the
    committed ncu record of this workload, if that record was taken on the current kernel
    sources (same sha256); (None, reason, None) otherwise."""
    config_name = {"long": "abot"}.get(config_name, config_name)  # the same launch shape
    rec = os.path.join(ROOT, "profiles", f"chunk_attention_{config_name}.traffic.json")
    if not os.path.exists(rec):
        return None, None, None
    with open(rec) as fh:
        r = json.load(fh)
    if r.get("kernel_sources_sha256") != attention_source_sha256():
        return None, "kernel changed since the counters were taken", None
    return r["dram_bytes_per_launch"], os.path.relpath(rec, ROOT), r.get("algorithmic_bytes_per_launch")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.path = None
        self.window = [None, None]
        if gpu_id is None:
            return
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="rkv_clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark_start(self):
        import datetime
        self.window[0] = datetime.datetime.now()

    def mark_end(self):
        import datetime
        self.window[1] = datetime.datetime.now()

    def stop(self):
        """Median SM clock and throttle reasons of the samples taken inside the marked window
        (all samples if none fell inside it)."""
        import datetime
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows, mx = [], None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                    rows.append((ts, float(parts[1]), [n for n, v in zip(names, parts[5:9]) if v.lower() == "active"]))
                    mx = float(parts[2])
                except ValueError:
                    continue
        t0, t1 = self.window
        inside = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        use = inside if inside else rows
        sm = [r[1] for r in use]
        reasons = {n for r in use for n in r[2]}
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "samples_in_timed_region": len(inside)}


# ---------------------------------------------------------------------- ranks
def reduce_max(x, device="cpu"):
    """Max of x over all ranks (x itself without a process group): every multi-GPU time
    reported is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


# ---------------------------------------------------------------------- CUDA arm
def visible_keys(cfg, committed, f0):
    import rolling_kv_chunked_b200 as rkv
    T = cfg["gh"] * cfg["gw"]
    return sum(n for _, _, n, _ in rkv.plan_window(cfg["W"], cfg["S"], committed, cfg["C"], f0)) * T


def attention_launches(cfg, committed, f0, sms):
    """Kernel launches of one attention call's attention part: 1, or 2 when the library runs the
    long-stream launch's partial last wave split by keys (then a combine launch follows). The
    same rule as the library's launcher: more units than SMs, a tail of at most half the SMs,
    and at least 32 key tiles."""
    import rolling_kv_chunked_b200 as rkv
    T = cfg["gh"] * cfg["gw"]
    Lq = cfg["C"] * T
    tiles = sum(-(-n * T // 128) for _, _, n, _ in rkv.plan_window(cfg["W"], cfg["S"], committed, cfg["C"], f0))
    units = -(-Lq // 256) * cfg["H"]
    tail = units % sms
    return 2 if tiles > 16 and tiles >= 32 and units > sms and 0 < tail and 2 * tail <= sms else 1


# a timed region at least this long is compared with the sustained (power-capped) bf16 peak;
# a shorter one with the burst peak
SUSTAINED_REGION_S = 1.0
# the workloads reported beside the headline one, each as a compact record
SIDE_WORKLOADS = ("abot", "480p")


def config_record(cfg, world):
    """The `config` of the bench line: the workload and its sizes (both arms print the same)."""
    T = cfg["gh"] * cfg["gw"]
    Lq = cfg["C"] * T
    n_layers = cfg.get("layers", 1)
    return {"workload": cfg["workload"], "queries_per_call": Lq, "keys_per_call": cfg["W"] * T,
            "calls_per_step": 5 * n_layers, "layers": n_layers,
            "parallelism": f"replicas x{world} (no data-path collective)",
            "l2": f"inputs larger than L2 ({19 * Lq * cfg['H'] * 128 * 2 / 1e6:.0f} MB per step)"}


def peak_for_region(pk, region_s):
    """(peak TFLOP/s, which one) for a timed region of region_s seconds."""
    if region_s >= SUSTAINED_REGION_S:
        return pk["bf16_tflops_sustained"], "bf16_tflops_sustained"
    return pk["bf16_tflops"], "bf16_tflops"


def run_rkv(args):
    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    result = measure_workload(args, args.config, headline=True)
    if CONFIGS[args.config].get("layers", 1) == 1 and not args.no_side:
        result["workloads"] = {}
        for name in SIDE_WORKLOADS:
            if name != args.config:
                result["workloads"][name] = measure_workload(args, name, headline=False)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def measure_workload(args, name, headline):
    """One workload: the timed steps (inputs resident in HBM), and for the headline also the
    whole rollout, the end-to-end pass from host buffers, the HBM-bound kernels, the
    cross-attention and the CPU baseline; side workloads give a compact record."""
    import torch
    import torch.distributed as dist

    import rolling_kv_chunked_b200 as rkv
    import synth

    world, rank, local = rank_env()
    cfg = CONFIGS[name]
    H, C, W, S = cfg["H"], cfg["C"], cfg["W"], cfg["S"]
    T = cfg["gh"] * cfg["gw"]
    Lq = C * T
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    n_layers = cfg.get("layers", 1)
    h = rkv.RollingKV(n_layers, H, 128, T, W, S, cfg["mode"])
    h.set_rope_grid(cfg["gh"], cfg["gw"])

    def fill(t, *fields):
        synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), synth.stream_key(rank, 77, *fields), 0, sp)
        return t

    bf = dict(dtype=torch.bfloat16, device="cuda")
    # a pool of step input sets (inputs of one step are ~300 MB, larger than L2)
    pool_n = 2
    pool = []
    for i in range(pool_n):
        pool.append(dict(
            q=[fill(torch.empty((Lq, H, 128), **bf), i, c, 1) for c in range(5)],
            k=[fill(torch.empty((Lq, H, 128), **bf), i, c, 2) for c in range(5)],
            v=[fill(torch.empty((Lq, H, 128), **bf), i, c, 3) for c in range(5)],
            xt=fill(torch.empty((Lq, H * 128), **bf), i, 9, 4),
            eps=[fill(torch.empty((Lq, H * 128), **bf), i, c, 5) for c in range(3)],
        ))
    outs = [torch.empty((Lq, H, 128), **bf) for _ in range(5)]
    x0 = torch.empty((Lq, H * 128), **bf)
    xn = [torch.empty((Lq, H * 128), **bf) for _ in range(2)]
    state = {"f0": 0}

    def step(inp, o=None, x0_buf=None, st=None):
        """One chunk through every layer: four denoise reads with the fused x0 / renoise
        epilogue, then the commit."""
        o = outs if o is None else o
        x0_buf = x0 if x0_buf is None else x0_buf
        st = sp if st is None else st
        f0 = state["f0"]
        for layer in range(n_layers):
            xt = inp["xt"]
            for s in range(4):
                sn = SIGMAS[s + 1] if s < 3 else -1.0
                nxt = xn[s % 2] if sn >= 0 else None
                h.chunk_attention(layer, inp["q"][s], inp["k"][s], inp["v"][s], o[s], C, f0, False, stream=st,
                                  flow=dict(xt=xt, eps=inp["eps"][s] if sn >= 0 else None, sigma=SIGMAS[s],
                                            sigma_next=sn, x0_out=x0_buf, xt_next_out=nxt))
                if nxt is not None:
                    xt = nxt
            h.chunk_attention(layer, inp["q"][4], inp["k"][4], inp["v"][4], o[4], C, f0, True, stream=st)
        state["f0"] = f0 + C

    # reference frames (sinks) and roll the window to steady state
    if cfg["refs"]:
        kr = fill(torch.empty((cfg["refs"] * T, H, 128), **bf), 99, 0, 2)
        vr = fill(torch.empty((cfg["refs"] * T, H, 128), **bf), 99, 0, 3)
        for layer in range(n_layers):
            h.write_chunk(layer, kr, vr, cfg["refs"], 0, stream=sp)
        state["f0"] = cfg["refs"]
    prefill = math.ceil((W - S) / C) + 1
    for i in range(prefill):
        inp = pool[i % pool_n]
        for layer in range(n_layers):
            h.chunk_attention(layer, inp["q"][4], inp["k"][4], inp["v"][4], outs[4], C, state["f0"], True, stream=sp)
        state["f0"] += C
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        gpu_id = None
    clocks = ClockSampler(gpu_id)  # started before the warm-up, so that it samples from the first timed step
    for i in range(args.warmup):
        step(pool[i % pool_n])
    torch.cuda.synchronize()
    if h.poll_device_status(sp) != rkv.OK:
        raise RuntimeError("device wait expired during warm-up")

    # FLOPs of the attention launches in the timed region (unmasked visible keys), and our
    # kernel launches there: per call the RoPE pre-pass and the attention (plus a combine
    # launch when its last wave is split), and the commit's write-back once per step
    flops = 0.0
    launches = 0
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    f = state["f0"]
    for _ in range(args.steps):
        flops += n_layers * 5 * 4.0 * H * 128 * Lq * visible_keys(cfg, f, f)
        launches += n_layers * (5 * (1 + attention_launches(cfg, f, f, sms)) + 1)
        f += C

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark_start()
    h.timing_begin(5 * n_layers * args.steps)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        step(pool[i % pool_n])
    ev1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    kernel_ms = h.timing_end(5 * n_layers * args.steps)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    status = h.poll_device_status(sp)
    if status != rkv.OK:
        raise RuntimeError("device wait expired in the timed region")
    ms = reduce_max(ms, "cuda")
    tokens = 5 * n_layers * Lq * args.steps * world
    value = tokens / (ms / 1e3)

    pk, pk_kind = peaks()
    mean_kernel_ms = sum(kernel_ms) / max(1, len(kernel_ms))
    achieved = flops / (sum(kernel_ms) / 1e3) / 1e12 if kernel_ms else None
    region_s = ms / 1e3
    peak, peak_name = peak_for_region(pk, region_s)
    n_launch = 5 * n_layers * args.steps
    attn = {"achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": (achieved / peak) if achieved else None,
            "peak_source": f"{pk_kind} {peak_name} (timed region {region_s:.2f} s; sustained peak from "
                           f"{SUSTAINED_REGION_S:g} s up)",
            "frac_of_burst": (achieved / pk["bf16_tflops"]) if achieved else None,
            "frac_of_sustained": (achieved / pk["bf16_tflops_sustained"]) if achieved else None,
            "mean_kernel_ms": mean_kernel_ms,
            "median_kernel_ms": statistics.median(kernel_ms) if kernel_ms else None,
            "launches_timed": len(kernel_ms), "flops_per_launch": flops / max(1, n_launch)}
    if not headline:
        hbm = None if args.no_hbm else measure_hbm_kernels(torch, rkv, synth, cfg, rank)
        h.close()
        del pool, outs, x0, xn
        torch.cuda.empty_cache()
        traffic, traffic_src, traffic_alg = profiled_traffic(name)
        attn.update(traffic=traffic, traffic_source=traffic_src, traffic_algorithmic_bytes=traffic_alg)
        return {"workload": cfg["workload"], "value": value, "unit": UNIT, "steps": args.steps,
                "ms_per_step": ms / args.steps, "queries_per_call": Lq, "keys_per_call": W * T,
                "attention": attn, "hbm_kernels": hbm, "clocks": clk}

    # ---- a whole rollout from an empty cache: the reference frames, then every chunk of the
    # workload's video (4 reads + 1 commit each), warm-up chunks with short windows included
    rollout = None
    if n_layers == 1 and world == 1 and not args.no_rollout:
        h.reset()
        state["f0"] = 0
        r0 = torch.cuda.Event(enable_timing=True)
        r1 = torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        if cfg["refs"]:
            h.write_chunk(0, kr, vr, cfg["refs"], 0, stream=sp)
            state["f0"] = cfg["refs"]
        n_chunks = cfg["rollout_chunks"]
        for i in range(n_chunks):
            step(pool[i % pool_n])
        r1.record(stream)
        torch.cuda.synchronize()
        if h.poll_device_status(sp) != rkv.OK:
            raise RuntimeError("device wait expired in the rollout")
        r_ms = r0.elapsed_time(r1)
        rollout = {"chunks": n_chunks, "frames": n_chunks * C, "ms": r_ms,
                   "query_tokens_per_s": 5 * n_chunks * Lq / (r_ms / 1e3),
                   "frames_per_s": n_chunks * C / (r_ms / 1e3)}

    # ---- end to end through the C ABI with host buffers (copies inside the timed region)
    e2e = None
    # (one layer only: the stacked-layer shape reruns the same kernels, and its layers' inputs
    # would come from the previous layer on the device, not from the host)
    if not args.no_e2e and n_layers == 1:
        e2e = run_e2e(args, torch, dist, world, pool, step, tokens)
    hbm = None if args.no_hbm or n_layers > 1 else measure_hbm_kernels(torch, rkv, synth, cfg, rank)
    cross = None if args.no_hbm or n_layers > 1 else measure_cross_attention(torch, rkv, synth, cfg, rank)

    traffic, traffic_src, traffic_alg = profiled_traffic(name)
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_record(cfg, world),
        "roofline": {"bound": "tensor", **attn, "traffic": traffic, "traffic_source": traffic_src,
                     "traffic_algorithmic_bytes": traffic_alg, "kernel": "chunk_attention_kernel"},
        "frames_per_s_per_layer": C * n_layers * args.steps * world / (ms / 1e3),
        "rollout": rollout,
        "e2e": e2e,
        "hbm_kernels": hbm,
        "cross_attention": cross,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_seconds)
    h.close()
    del pool, outs, x0, xn
    torch.cuda.empty_cache()
    return result


def run_cfg(args):
    """Guided mode on one GPU: one step = one chunk = 40 x (conditional read, unconditional read
    with the fused guidance + x0 / renoise epilogue) + the commit of each branch (82 attention
    launches). Device-timed with inputs resident in HBM."""
    import torch

    import rolling_kv_chunked_b200 as rkv
    import synth

    world, rank, local = rank_env()
    if world > 1:
        raise SystemExit("the guided workload is measured on one GPU")
    torch.cuda.set_device(local)
    cfg = CFG_CONFIGS[args.config]
    H, C, W, S = cfg["H"], cfg["C"], cfg["W"], cfg["S"]
    T = cfg["gh"] * cfg["gw"]
    Lq = C * T
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    hs = [rkv.RollingKV(1, H, 128, T, W, S, cfg["mode"]) for _ in range(2)]
    for h in hs:
        h.set_rope_grid(cfg["gh"], cfg["gw"])

    def fill(t, *fields):
        synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), synth.stream_key(rank, 76, *fields), 0, sp)
        return t

    bf = dict(dtype=torch.bfloat16, device="cuda")
    n_sets = 5      # q/k/v sets per branch, cycled over the steps (each set 49 MB at this size)
    qkv = [[[fill(torch.empty((Lq, H, 128), **bf), b, i, t) for t in range(3)] for i in range(n_sets)]
           for b in range(2)]
    xt0 = fill(torch.empty((Lq, H * 128), **bf), 9, 0, 4)
    eps = [fill(torch.empty((Lq, H * 128), **bf), 9, i, 5) for i in range(2)]
    outs = [torch.empty((Lq, H, 128), **bf) for _ in range(2)]
    x0 = torch.empty((Lq, H * 128), **bf)
    xn = [torch.empty((Lq, H * 128), **bf) for _ in range(2)]
    sig = [1.0 - k / CFG_STEPS for k in range(CFG_STEPS)] + [-1.0]
    state = {"f0": 0}

    def step():
        f0 = state["f0"]
        xt = xt0
        for k in range(CFG_STEPS):
            a, b = qkv[0][k % (n_sets - 1)], qkv[1][k % (n_sets - 1)]
            sn = sig[k + 1]
            nxt = xn[k % 2] if sn >= 0 else None
            hs[0].chunk_attention(0, *a, outs[0], C, f0, False, stream=sp)
            hs[1].chunk_attention(0, *b, outs[1], C, f0, False, stream=sp,
                                  flow=dict(xt=xt, eps=eps[k % 2] if sn >= 0 else None, sigma=sig[k],
                                            sigma_next=sn, x0_out=x0, xt_next_out=nxt, v_cond=outs[0],
                                            cfg_scale=CFG_SCALE))
            if nxt is not None:
                xt = nxt
        for br in range(2):
            hs[br].chunk_attention(0, *qkv[br][n_sets - 1], outs[br], C, f0, True, stream=sp)
        state["f0"] = f0 + C

    if cfg["refs"]:
        for br in range(2):
            kr = fill(torch.empty((cfg["refs"] * T, H, 128), **bf), 99, br, 2)
            vr = fill(torch.empty((cfg["refs"] * T, H, 128), **bf), 99, br, 3)
            hs[br].write_chunk(0, kr, vr, cfg["refs"], 0, stream=sp)
        state["f0"] = cfg["refs"]
    for i in range(math.ceil((W - S) / C) + 1):
        for br in range(2):
            hs[br].chunk_attention(0, *qkv[br][n_sets - 1], outs[br], C, state["f0"], True, stream=sp)
        state["f0"] += C
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        gpu_id = None
    clocks = ClockSampler(gpu_id)  # started before the warm-up, so that it samples from the first timed step
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    calls = 2 * CFG_STEPS + 2
    flops, f = 0.0, state["f0"]
    for _ in range(args.steps):
        flops += calls * 4.0 * H * 128 * Lq * visible_keys(cfg, f, f)
        f += C
    torch.cuda.synchronize()
    clocks.mark_start()
    for h in hs:
        h.timing_begin(calls * args.steps)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    kernel_ms = hs[0].timing_end(calls * args.steps) + hs[1].timing_end(calls * args.steps)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    for h in hs:
        if h.poll_device_status(sp) != rkv.OK:
            raise RuntimeError("device wait expired in the timed region")
    tokens = calls * Lq * args.steps
    pk, pk_kind = peaks()
    achieved = flops / (sum(kernel_ms) / 1e3) / 1e12 if kernel_ms else None
    peak = pk["bf16_tflops_sustained"]

    # the standalone guided epilogue (K4 with guidance): 4 bf16 reads + 2 bf16 writes per element
    n = Lq * H * 128
    n_ep = max(2, -(-int(320e6) // (n * 2 * 6)))
    ep_sets = [[fill(torch.empty(n, **bf), 50 + i, j) for j in range(6)] for i in range(n_ep)]
    s_ = lambda i: ep_sets[i % n_ep]
    rkv.flow_cfg_x0_renoise(*s_(0)[:4], CFG_SCALE, 1.0, 0.975, s_(0)[4], s_(0)[5], stream=sp)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(20):
        rkv.flow_cfg_x0_renoise(*s_(i)[:4], CFG_SCALE, 1.0, 0.975, s_(i)[4], s_(i)[5], stream=sp)
    e1.record(stream)
    torch.cuda.synchronize()
    ep_gbs = 12 * n / (e0.elapsed_time(e1) / 20 / 1e3) / 1e9
    result = {
        "metric": METRIC, "value": tokens / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg["workload"], "queries_per_call": Lq, "keys_per_call": W * T,
                   "calls_per_step": calls, "parallelism": "single GPU",
                   "l2": "inputs larger than L2 (window K/V 227 MB per branch)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": (achieved / peak) if achieved else None, "traffic": None,
                     "kernel": "chunk_attention_kernel", "peak_source": f"{pk_kind} bf16_tflops_sustained",
                     "frac_of_burst": (achieved / pk["bf16_tflops"]) if achieved else None,
                     "mean_kernel_ms": sum(kernel_ms) / max(1, len(kernel_ms)), "launches_timed": len(kernel_ms),
                     "flops_per_launch": flops / max(1, calls * args.steps)},
        "e2e": None,
        "hbm_kernels": {"flow_cfg_x0_renoise": {"bytes_per_launch": 12 * n, "GB/s": ep_gbs,
                                                "frac_of_hbm": ep_gbs / pk["hbm_gbs"]},
                        "peak_hbm_gbs": pk["hbm_gbs"], "peak_source": pk_kind},
        "gpu_launches": (2 * CFG_STEPS * (1 + attention_launches(
            cfg, W, W, torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count))
            + 2 * 2) * args.steps,
        "clocks": clk,
    }
    for h in hs:
        h.close()
    print(json.dumps(result), flush=True)


def run_e2e(args, torch, dist, world, pool, step, tokens):
    """The same steps through the public API with every input in pinned host memory: each
    step copies its inputs host -> device and its results (the five attention outputs and
    the final x0) device -> host. Copies run on their own streams, double-buffered, so the
    transfers of one step overlap the kernels of the previous one."""
    Lq, H = pool[0]["q"][0].shape[0], pool[0]["q"][0].shape[1]
    bf = dict(dtype=torch.bfloat16, device="cuda")
    comp = torch.cuda.Stream()
    h2d_s = torch.cuda.Stream()
    d2h_s = torch.cuda.Stream()
    host_in = []
    for i in range(2):
        host_in.append({k: ([t.cpu().pin_memory() for t in v] if isinstance(v, list) else v.cpu().pin_memory())
                        for k, v in pool[i].items()})
    dev_in = pool                                            # two device input sets
    dev_out = [[torch.empty((Lq, H, 128), **bf) for _ in range(5)] for _ in range(2)]
    dev_x0 = [torch.empty((Lq, H * 128), **bf) for _ in range(2)]
    host_out = [[torch.empty((Lq, H, 128), dtype=torch.bfloat16).pin_memory() for _ in range(5)] for _ in range(2)]
    host_x0 = [torch.empty((Lq, H * 128), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * 2 for v in host_in[0].values() for t in (v if isinstance(v, list) else [v]))
    d2h = sum(t.numel() * 2 for t in host_out[0]) + host_x0[0].numel() * 2
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of set b landed
    ev_done = [torch.cuda.Event() for _ in range(2)]    # kernels of set b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]     # results of set b copied out

    def copy_set(dst, src):
        for key_, val in src.items():
            if isinstance(val, list):
                for d_, s_ in zip(dst[key_], val):
                    d_.copy_(s_, non_blocking=True)
            else:
                dst[key_].copy_(val, non_blocking=True)

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_done[b])           # set b's inputs are free again
                copy_set(dev_in[b], host_in[b])
                ev_in[b].record(h2d_s)
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_out[b])                 # set b's outputs were copied out
            step(dev_in[b], dev_out[b], dev_x0[b], comp.cuda_stream)
            ev_done[b].record(comp)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[b])
                for d_, s_ in zip(host_out[b], dev_out[b]):
                    d_.copy_(s_, non_blocking=True)
                host_x0[b].copy_(dev_x0[b], non_blocking=True)
                ev_out[b].record(d2h_s)

    run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    h2d_s.wait_event(e0)
    run(args.steps)
    comp.wait_stream(h2d_s)
    comp.wait_stream(d2h_s)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), "cuda")
    return {"value": tokens / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_ms / args.steps, "overlap": "h2d / kernels / d2h on three streams, double-buffered"}


def measure_hbm_kernels(torch, rkv, synth, cfg, rank, reps=20):
    """Achieved HBM bandwidth of the memory-bound kernels at the workload's sizes, timed with
    CUDA events on their stream; every launch touches a different buffer set and the sets
    together exceed the 126 MB L2, so each launch streams from HBM."""
    H, C, W, S = cfg["H"], cfg["C"], cfg["W"], cfg["S"]
    T = cfg["gh"] * cfg["gw"]
    Lq = C * T
    n = Lq * H * 128
    st = torch.cuda.current_stream()
    sp = st.cuda_stream
    bf = dict(dtype=torch.bfloat16, device="cuda")
    n_sets = max(2, -(-int(320e6) // (n * 2 * 5)))       # >= 320 MB cycled

    def fill(t, *f):
        synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), synth.stream_key(rank, 88, *f), 0, sp)
        return t

    def timed(fn):
        """Seconds per launch: `reps` launches captured in one CUDA graph and replayed, so that
        the host's per-call overhead does not leave the GPU idle between small launches (the
        launches, their arguments and their buffers are the same as when called directly)."""
        fn(0)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(st)
        with torch.cuda.stream(cap):
            graph.capture_begin()
            for i in range(reps):
                fn(i, cap.cuda_stream)
            graph.capture_end()
        st.wait_stream(cap)
        graph.replay()
        torch.cuda.synchronize()
        e0.record(st)
        graph.replay()
        e1.record(st)
        torch.cuda.synchronize()
        del graph
        return e0.elapsed_time(e1) / reps / 1e3

    res = {}
    # K4: x0 = xt - sigma v; xt' = (1 - sigma') x0 + sigma' eps; 3 reads + 2 writes of bf16
    sets = [[fill(torch.empty(n, **bf), i, j) for j in range(5)] for i in range(n_sets)]
    sec = timed(lambda i, s=sp: rkv.flow_x0_renoise(sets[i % n_sets][0], sets[i % n_sets][1], sets[i % n_sets][2],
                                                    1.0, 0.75, sets[i % n_sets][3], sets[i % n_sets][4], stream=s))
    res["flow_x0_renoise"] = {"bytes_per_launch": 10 * n, "GB/s": 10 * n / sec / 1e9}
    del sets
    # K3: in-place RoPE of a [Lq, H, 128] tensor, one read + one write
    bufs = [fill(torch.empty((Lq, H, 128), **bf), 50, i) for i in range(2 * n_sets)]
    hr = rkv.RollingKV(1, H, 128, T, W, S, cfg["mode"])
    hr.set_rope_grid(cfg["gh"], cfg["gw"])
    sec = timed(lambda i, s=sp: hr.rope_apply(bufs[i % len(bufs)], C, 0, C, stream=s))
    res["rope_apply"] = {"bytes_per_launch": 4 * n, "GB/s": 4 * n / sec / 1e9}
    # K1: the ring write-back (rkv_write_chunk): K and V read and written once; in absolute
    # mode the rotated copy of K is written as well
    hw = rkv.RollingKV(1, H, 128, T, W, S, cfg["mode"])
    hw.set_rope_grid(cfg["gh"], cfg["gw"])
    state = {"f": 0}

    def write(i, s=sp):
        hw.write_chunk(0, bufs[(2 * i) % len(bufs)], bufs[(2 * i + 1) % len(bufs)], C, state["f"], stream=s)
        state["f"] += C
    sec = timed(write)
    per = 8 * n + (4 * n if cfg["mode"] == 0 else 0)
    res["commit_write"] = {"bytes_per_launch": per, "GB/s": per / sec / 1e9}
    pk, kind = peaks()
    for v in res.values():
        v["frac_of_hbm"] = v["GB/s"] / pk["hbm_gbs"]
    res["peak_hbm_gbs"] = pk["hbm_gbs"]
    res["peak_source"] = kind
    hr.close()
    hw.close()
    return res


def measure_cross_attention(torch, rkv, synth, cfg, rank, n_text=512, reps=20):
    """The cross-attention over the cached text K/V at the workload's chunk size: the chunk's
    queries against n_text text tokens. Query / output sets are cycled so that the launches
    together touch more than the 126 MB L2."""
    H, C = cfg["H"], cfg["C"]
    T = cfg["gh"] * cfg["gw"]
    Lq = C * T
    st = torch.cuda.current_stream()
    sp = st.cuda_stream
    bf = dict(dtype=torch.bfloat16, device="cuda")

    def fill(t, *f):
        synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), synth.stream_key(rank, 89, *f), 0, sp)
        return t

    h = rkv.RollingKV(1, H, 128, T, cfg["W"], cfg["S"], cfg["mode"])
    h.set_text_kv(0, fill(torch.empty((n_text, H, 128), **bf), 1), fill(torch.empty((n_text, H, 128), **bf), 2))
    n_sets = max(2, -(-int(320e6) // (Lq * H * 128 * 2 * 2)))
    qs = [fill(torch.empty((Lq, H, 128), **bf), 3, i) for i in range(n_sets)]
    outs = [torch.empty((Lq, H, 128), **bf) for _ in range(n_sets)]
    h.cross_attention(0, qs[0], outs[0], stream=sp)
    torch.cuda.synchronize()
    h.timing_begin(reps)
    for i in range(reps):
        h.cross_attention(0, qs[i % n_sets], outs[i % n_sets], stream=sp)
    torch.cuda.synchronize()
    ms = h.timing_end(reps)
    if h.poll_device_status(sp) != rkv.OK:
        raise RuntimeError("device wait expired in the cross-attention launches")
    h.close()
    sec = sum(ms) / len(ms) / 1e3
    flops = 4.0 * H * 128 * Lq * n_text
    bytes_ = 2 * Lq * H * 128 * 2 + 2 * n_text * H * 128 * 2
    pk, kind = peaks()
    return {"queries": Lq, "text_tokens": n_text, "mean_kernel_ms": sec * 1e3,
            "TFLOP/s": flops / sec / 1e12, "frac_of_burst": flops / sec / 1e12 / pk["bf16_tflops"],
            "GB/s": bytes_ / sec / 1e9, "frac_of_hbm": bytes_ / sec / 1e9 / pk["hbm_gbs"],
            "flops_per_launch": flops, "bytes_per_launch": bytes_, "peak_source": kind}


# ---------------------------------------------------------------------- oracle arm
def _oracle_steady_layer(cfg):
    """An oracle layer holding a full steady-state window (one synthetic frame reused)."""
    import synth
    from oracle.layer import OracleLayer
    H, C, W, S = cfg["H"], cfg["C"], cfg["W"], cfg["S"]
    T = cfg["gh"] * cfg["gw"]
    orc = OracleLayer(H, 128, T, cfg["gh"], cfg["gw"], W, S, cfg["mode"])
    frame = synth.normal_bf16_bits(synth.stream_key(0, 78), 0, T * H * 128).reshape(T, H, 128)
    f = 0
    while f < W + C:
        orc.write_chunk(frame, frame, 1, f)
        f += 1
    q = synth.normal_bf16_bits(synth.stream_key(0, 79), 0, C * T * H * 128).reshape(C * T, H, 128)
    return orc, q, f


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(i.get("num_threads", 1) for i in threadpool_info()) or os.cpu_count()
    except Exception:
        return os.cpu_count()


# the oracle's sample of one call: this many query rows (evenly spaced over the chunk) of one
# head against the full steady-state window, scaled to all rows and heads
SAMPLE_ROWS = 1024


def _sample_rows(Lq):
    import numpy as np
    n = min(SAMPLE_ROWS, Lq)
    return np.unique(np.linspace(0, Lq - 1, n).round().astype(np.int64))


def cpu_baseline(cfg, budget_s=10.0):
    """The oracle as it stands, on a bounded sample: steady-state denoise reads of one head,
    SAMPLE_ROWS query rows against the full window, repeated for ~budget_s, scaled by
    H * Lq / rows."""
    orc, q, f0 = _oracle_steady_layer(cfg)
    C, H = cfg["C"], cfg["H"]
    T = cfg["gh"] * cfg["gw"]
    rows = _sample_rows(C * T)
    n, t0 = 0, time.perf_counter()
    while True:
        orc.chunk_attention(q, q, q, C, f0, False, heads=[0], rows=rows)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    per_call_s = el / n * H * (C * T) / len(rows)
    # the oracle's x0 / renoise step (K4) on an eighth of the workload's latent
    from oracle import flow as oflow
    import synth
    n_el = C * T * H * 128 // 8
    xt, v, eps = (synth.normal_bf16_bits(synth.stream_key(0, 93, i), 0, n_el) for i in range(3))
    t1 = time.perf_counter()
    oflow.x0_renoise_bf16(xt, v, eps, 1.0, 0.75)
    flow_s = time.perf_counter() - t1
    return {"value": C * T / per_call_s, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n} steady-state reads of 1 of {H} heads, {len(rows)} of {C * T} query rows vs "
                      f"{cfg['W'] * T} keys, numpy fp64, scaled by {H} x {C * T}/{len(rows)}",
            "flow_x0_renoise": {"GB/s": 10 * n_el / flow_s / 1e9, "elements": n_el,
                                "sample": "one call on an eighth of the latent, sigma 1.0 -> 0.75, numpy fp64"}}


def run_reference(args):
    world, rank, _ = rank_env()
    if rank != 0:
        return                     # the oracle arm runs on rank 0 only; other ranks exit 0
    cfg = {**CONFIGS, **CFG_CONFIGS}[args.config]
    orc, q, f0 = _oracle_steady_layer(cfg)
    C, H = cfg["C"], cfg["H"]
    T = cfg["gh"] * cfg["gw"]
    Lq = C * T
    rows = _sample_rows(Lq)
    for _ in range(args.warmup):
        orc.chunk_attention(q, q, q, C, f0, False, heads=[0], rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.chunk_attention(q, q, q, C, f0, False, heads=[0], rows=rows)
    el = time.perf_counter() - t0
    per_call_s = el / args.steps * H * Lq / len(rows)
    value = Lq / per_call_s
    sample = (f"each step: one steady-state read of 1 of {H} heads, {len(rows)} of {Lq} query rows vs "
              f"{cfg['W'] * T} keys, scaled by {H} x {Lq}/{len(rows)}")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_record(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_isolated(args):
    """A few launches of one kernel at the workload's sizes and nothing else, for profiler
    captures (``ncu -k <kernel> -s 1 -c 1 python bench.py --isolate ...``): ``attention``
    (steady-state reads, see run_isolated_attention), ``commit``
    (rkv_write_chunk: the ring write-back), ``rope`` (rkv_rope_apply of one chunk's
    [Lq, H, 128] tensor), ``flow`` (rkv_flow_x0_renoise on the [Lq, H*128] latent, renoise
    on) or ``cross`` (rkv_cross_attention of the chunk's queries over 512 text tokens).
    Launches rotate over buffer sets that together exceed the 126 MB L2. Prints one JSON line
    with the mean CUDA-event time per launch (not a benchmark line)."""
    import torch
    import rolling_kv_chunked_b200 as rkv
    import synth
    cfg = CONFIGS[args.config]
    H, C, W, S = cfg["H"], cfg["C"], cfg["W"], cfg["S"]
    T = cfg["gh"] * cfg["gw"]
    Lq = C * T
    n = Lq * H * 128
    st = torch.cuda.current_stream()
    sp = st.cuda_stream
    bf = dict(dtype=torch.bfloat16, device="cuda")

    def fill(t, *f):
        synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), synth.stream_key(0, 91, *f), 0, sp)
        return t

    if args.isolate == "attention":
        run_isolated_attention(args, torch, rkv, synth, cfg)
        return
    per_set = {"commit": 2, "rope": 1, "flow": 5, "cross": 2}[args.isolate]
    n_sets = max(2, -(-int(256e6) // (per_set * n * 2)))
    sets = [[fill(torch.empty((Lq, H, 128), **bf), i, j) for j in range(per_set)] for i in range(n_sets)]
    h = None
    if args.isolate in ("commit", "rope", "cross"):
        h = rkv.RollingKV(1, H, 128, T, W, S, cfg["mode"])
        h.set_rope_grid(cfg["gh"], cfg["gw"])
    if args.isolate == "commit":
        state = {"f": 0}

        def launch(b):
            h.write_chunk(0, b[0], b[1], C, state["f"], stream=sp)
            state["f"] += C
        work = {"bytes_per_launch": 8 * n + (4 * n if cfg["mode"] == 0 else 0)}
    elif args.isolate == "rope":
        def launch(b):
            h.rope_apply(b[0], C, 0, C, stream=sp)
        work = {"bytes_per_launch": 4 * n}
    elif args.isolate == "flow":
        def launch(b):
            lat = [x.view(Lq, H * 128) for x in b]
            rkv.flow_x0_renoise(lat[0], lat[1], lat[2], 1.0, 0.75, lat[3], lat[4], stream=sp)
        work = {"bytes_per_launch": 10 * n}
    else:
        n_text = 512
        h.set_text_kv(0, fill(torch.empty((n_text, H, 128), **bf), 1000), fill(torch.empty((n_text, H, 128), **bf), 1001),
                      stream=sp)

        def launch(b):
            h.cross_attention(0, b[0], b[1], stream=sp)
        work = {"flops_per_launch": 4.0 * H * 128 * Lq * n_text}
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.reps)]
    torch.cuda.synchronize()
    for i in range(args.reps):
        ev[2 * i].record(st)
        launch(sets[i % n_sets])
        ev[2 * i + 1].record(st)
    torch.cuda.synchronize()
    if h is not None:
        if h.poll_device_status(sp) != rkv.OK:
            raise RuntimeError("device wait expired")
        h.close()
    us = [ev[2 * i].elapsed_time(ev[2 * i + 1]) * 1e3 for i in range(args.reps)]
    print(json.dumps({"isolate": args.isolate, "config": args.config, "launches": args.reps,
                      "us_per_launch": us, **work}), flush=True)


def run_isolated_attention(args, torch, rkv, synth, cfg):
    """Steady-state attention reads of the workload and as little else as possible: the window
    is filled by rkv_write_chunk (two launches: the sinks, then the rest), then --reps denoise
    reads of the next chunk run (each the RoPE pre-pass plus one attention launch). Holds the
    layer's caches and one q / k / v set (~3.5 GB at 720p), for profiler captures
    (``ncu -k regex:chunk_attention -c 1``)."""
    H, C, W, S = cfg["H"], cfg["C"], cfg["W"], cfg["S"]
    T = cfg["gh"] * cfg["gw"]
    Lq = C * T
    st = torch.cuda.current_stream()
    sp = st.cuda_stream
    bf = dict(dtype=torch.bfloat16, device="cuda")
    h = rkv.RollingKV(1, H, 128, T, W, S, cfg["mode"])
    h.set_rope_grid(cfg["gh"], cfg["gw"])
    f = 0
    for n in (S, W - S):
        k = torch.empty((n * T, H, 128), **bf)
        v = torch.empty((n * T, H, 128), **bf)
        synth.fill_normal_bf16_cuda(k.data_ptr(), k.numel(), synth.stream_key(0, 92, f, 2), 0, sp)
        synth.fill_normal_bf16_cuda(v.data_ptr(), v.numel(), synth.stream_key(0, 92, f, 3), 0, sp)
        h.write_chunk(0, k, v, n, f, stream=sp)
        f += n
        del k, v
    qkv = []
    for tag in (1, 2, 3):
        t = torch.empty((Lq, H, 128), **bf)
        synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), synth.stream_key(0, 92, f, tag), 0, sp)
        qkv.append(t)
    out = torch.empty((Lq, H, 128), **bf)
    keys = visible_keys(cfg, f, f)
    torch.cuda.synchronize()
    h.timing_begin(args.reps)
    for _ in range(args.reps):
        h.chunk_attention(0, *qkv, out, C, f, False, stream=sp)
    ms = h.timing_end(args.reps)
    if h.poll_device_status(sp) != rkv.OK:
        raise RuntimeError("device wait expired")
    h.close()
    print(json.dumps({"isolate": "attention", "config": args.config, "launches": args.reps,
                      "us_per_launch": [x * 1e3 for x in ms], "queries": Lq, "keys": keys,
                      "flops_per_launch": 4.0 * H * 128 * Lq * keys,
                      "algorithmic_bytes_per_launch": algorithmic_attention_bytes(cfg, keys, flow=False)}),
          flush=True)


def algorithmic_attention_bytes(cfg, keys, flow):
    """Bytes one attention launch must move at least: Q, K and V of the visible window read
    once per head, O written; with the fused x0 / renoise epilogue also xt and eps read and x0,
    xt' written (four latent-sized streams)."""
    H = cfg["H"]
    Lq = cfg["C"] * cfg["gh"] * cfg["gw"]
    b = 2 * 128 * H * (Lq + 2 * keys + Lq)
    if flow:
        b += 4 * 2 * 128 * H * Lq
    return b


def record_traffic(csv_path, config_name, command):
    """Write profiles/chunk_attention_<workload>.traffic.json from an ncu CSV (metrics
    dram__bytes_read.sum, dram__bytes_write.sum, gpu__time_duration.sum) of one attention launch
    made with ``--isolate attention``, stamped with the sha256 of the kernel sources."""
    import csv
    scales = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "ns": 1e-9, "us": 1e-6, "ms": 1e-3,
              "nsecond": 1e-9, "usecond": 1e-6, "msecond": 1e-3, "second": 1}
    vals = {}
    with open(csv_path) as fh:
        rows = [l for l in fh if l.startswith('"')]
    if '"Metric Name"' in rows[0]:
        # one metric per row (ncu --csv --log-file of a --metrics capture)
        for row in csv.DictReader(rows):
            if "chunk_attention" in row["Kernel Name"]:
                v = float(row["Metric Value"].replace(",", ""))
                vals.setdefault(row["Metric Name"], v * scales.get(row["Metric Unit"], 1))
    else:
        # one launch per row after a row of units (ncu -i <report> --page raw --csv)
        table = list(csv.reader(rows))
        hdr, units = table[0], table[1]
        for row in table[2:]:
            if "chunk_attention" in row[hdr.index("Kernel Name")]:
                for h, u, v in zip(hdr, units, row):
                    try:
                        vals.setdefault(h, float(v.replace(",", "")) * scales.get(u, 1))
                    except ValueError:
                        pass
                break
    cfg = CONFIGS[config_name]
    T = cfg["gh"] * cfg["gw"]
    keys = cfg["W"] * T  # the isolated reads see the full window
    rec = {"kernel": "chunk_attention_kernel", "workload": config_name,
           "launch": "steady-state denoise read without the fused epilogue (bench.py --isolate attention)",
           "kernel_sources": [os.path.relpath(f, ROOT) for f in ATTN_SRCS],
           "kernel_sources_sha256": attention_source_sha256(),
           "dram_bytes_read": int(vals["dram__bytes_read.sum"]), "dram_bytes_write": int(vals["dram__bytes_write.sum"]),
           "dram_bytes_per_launch": int(vals["dram__bytes_read.sum"] + vals["dram__bytes_write.sum"]),
           "algorithmic_bytes_per_launch": algorithmic_attention_bytes(cfg, keys, flow=False),
           "duration_s_under_ncu": vals.get("gpu__time_duration.sum"), "command": command}
    rec["traffic_over_algorithmic"] = rec["dram_bytes_per_launch"] / rec["algorithmic_bytes_per_launch"]
    out = os.path.join(ROOT, "profiles", f"chunk_attention_{config_name}.traffic.json")
    with open(out, "w") as fh:
        json.dump(rec, fh, indent=1)
        fh.write("\n")
    print(out)


def relaunch_ranks(n, impl):
    """--gpus N without a launcher: start N ranks of this same command line under
    torch.distributed.run (one process per GPU, rendezvous on 127.0.0.1) and return its exit
    status. The GPU arm needs N visible GPUs; the reference arm runs on the host."""
    if impl == "rkv":
        import torch
        have = torch.cuda.device_count()
        if have < n:
            raise SystemExit(f"--gpus {n}: only {have} CUDA device(s) visible")
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="720p", choices=sorted(CONFIGS) + sorted(CFG_CONFIGS))
    ap.add_argument("--impl", default="rkv", choices=["rkv", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--no-hbm", action="store_true",
                    help="skip the side measurements (HBM-bound kernels, cross-attention)")
    ap.add_argument("--no-rollout", action="store_true", help="skip the whole-rollout pass")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the compact records of the other single-layer workloads")
    ap.add_argument("--isolate", choices=["attention", "commit", "rope", "flow", "cross"],
                    help="only launch this kernel --reps times at the config's sizes (for profiler captures)")
    ap.add_argument("--reps", type=int, default=3, help="launches of the --isolate kernel")
    ap.add_argument("--record-traffic", metavar="CSV",
                    help="write the workload's attention traffic record from this ncu CSV and exit")
    ap.add_argument("--record-command", default="", help="the ncu command the CSV came from (for the record)")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args.record_traffic, args.config, args.record_command)
        return
    if args.isolate:
        if args.config not in CONFIGS:
            ap.error("--isolate takes one of " + ", ".join(sorted(CONFIGS)))
        run_isolated(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch_ranks(args.gpus, args.impl))
    if int(os.environ.get("WORLD_SIZE", "1")) != args.gpus:
        ap.error(f"--gpus {args.gpus} does not match the {os.environ.get('WORLD_SIZE', '1')} ranks launched")
    if args.impl == "reference":
        run_reference(args)
    elif args.config in CFG_CONFIGS:
        run_cfg(args)
    else:
        run_rkv(args)


if __name__ == "__main__":
    main()
