#!/usr/bin/env python
"""Benchmark of the Monodratic mixer on B200: route+attend tokens/s at S=32768.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload scale32k] [--no-sweep] [--no-cpu-baseline] [--no-decode]
                    [--no-backward]

A step is one pass of the whole hot path over one batch: projection + RoPE,
block summaries + addresses, posting lists, probe/rerank, selected-set
attention and the output projection, each through its C-ABI entry point on
one stream.  CUDA events bracket every stage.  `value` is the metric the
workload is quoted on: tokens / route+attend time (summaries through
attention, Q/K/V resident in HBM).  L2 is flushed (256 MiB write) before every
step, outside the events.

With N GPUs (torchrun, one process per GPU) each rank runs its own replica of
the workload: the path shards by (batch, head) with no exchange, so there is no
data-path collective; `value` = all ranks' tokens / the slowest rank's time.

`--impl reference` times the CPU oracle (the reference arm: the plain fp64/fp32
statement of the method) on a bounded sample of the same workload.

Prints ONE JSON line on rank 0; everything else goes to stderr.
"""
from __future__ import annotations

import argparse
import json
import os
import math
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "route+attend tokens/s at S=32768 bf16 on 1 B200; % of HBM roofline"
UNIT = "tokens/s"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def bf16_sustained_peak():
    """The bf16 tensor-core peak for a kernel timed inside a long run: measured sustained, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1400.0, "fallback"


def describe(cfg) -> str:
    return (f"{cfg.name}: B={cfg.B} S={cfg.S} W={cfg.W} H={cfg.H} d={cfg.d} {cfg.dtype} Bs={cfg.Bs} L={cfg.L} "
            f"R={cfg.R} E={cfg.E} M={cfg.M} C={cfg.C} T={cfg.T} cap={cfg.cap}")


# ---------------------------------------------------------------------------
# algorithmic bytes (per call) of each stage: what the stage must read and
# write at least once, each tensor counted once per call
# ---------------------------------------------------------------------------
def algorithmic_bytes(cfg, npairs: int = 0, blocks: int = 0) -> dict:
    """npairs: selected (query, remote block) pairs; blocks: distinct (b, h, block) among them."""
    es = 2 if cfg.dtype == "bf16" else 4
    B, H, S, d, R, nb = cfg.B, cfg.H, cfg.S, cfg.d, cfg.R, cfg.nb
    qkv = B * H * S * d * es
    kbar = B * H * nb * d * 4
    addr = B * H * nb * 4
    post = B * H * nb * 4 * 2                 # sorted ids + their addresses (ranks are not read back)
    sel = B * H * S * R * 4
    cb = H * cfg.C * d * 4
    o = B * S * H * d * es
    part = npairs * (2 * d + 8)               # one bf16 partial row and its (max, sum) per pair
    return {
        "summaries": qkv + kbar + addr + cb,            # read K, write kbar + addr
        "lists": addr + 3 * B * H * nb * 4,             # read addr, write ids/addr/rank
        "queries": qkv + kbar + post + cb + sel,        # read Q, kbar, lists; write sel
        "attend": 3 * qkv + sel + o,                    # read Q, K, V, sel; write O
        # the attention's stages in this design: pairs grouped by block (sel read twice, pair ids written);
        # remote: each pair's query row, each selected block's K and V rows once, the pair ids; partials written;
        # local: Q, K, V once, sel, the partials read; O written
        "pairs": 2 * sel + 4 * npairs,
        "remote": npairs * d * es + blocks * 2 * cfg.Bs * d * es + 4 * npairs + part,
        "local": 3 * qkv + sel + part + o,
        # the metric's roofline: unique Q/K/V/O + 2x each routing table (written once, read once)
        "route_attend": 3 * qkv + o + 2 * kbar + 2 * addr + 2 * (B * H * nb * 5) + 2 * sel,
    }


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._th = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: no clock record
            log("clock sampler unavailable:", e)
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((sm, rs, pw))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._th = threading.Thread(target=self._run, daemon=True)
            self._th.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._th:
            self._th.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        sms = [s[0] for s in self.samples]
        reasons = set()
        for _, rs, _ in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(sms), "power_w_max": max(s[2] for s in self.samples)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch

    from learned_product_hash_proj_b200 import dist, mono, synth

    rank, local, world = dist.init("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = synth.config(args.workload)
    seed = dist.replica_seed(args.seed, rank)
    log(f"[rank {rank}] generating {describe(cfg)} (seed {seed})")
    inp = synth.make_inputs(cfg, seed)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    to = lambda a: torch.from_numpy(a).to(tdt).to(dev).contiguous()
    x, Wq, Wk, Wv, Wo = (to(inp[k]) for k in ("x", "Wq", "Wk", "Wv", "Wo"))
    cb = torch.from_numpy(inp["codebooks"]).to(dev).contiguous()
    plan = mono.Plan(cfg)
    ws = plan.workspace(dev)
    B, H, S, d, R, W = cfg.B, cfg.H, cfg.S, cfg.d, cfg.R, cfg.W
    Q = torch.empty((B, H, S, d), dtype=tdt, device=dev)
    K, V = torch.empty_like(Q), torch.empty_like(Q)
    sel = torch.empty((B, H, S, R), dtype=torch.int32, device=dev)
    O = torch.empty((B, S, H * d), dtype=tdt, device=dev)
    delta = torch.empty((B, S, W), dtype=tdt, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = ["project", "summaries", "lists", "queries", "pairs", "remote", "local", "out_project"]
    window = ("summaries", "lists", "queries", "pairs", "remote", "local")

    def step_window(ev):
        # the timed step: the whole window through mono_route and mono_attend, with no event inside it (events
        # between the stages would keep the probe from starting while the lists kernel still runs)
        flush.zero_()
        ev[0].record(stream)
        mono.project(plan, x, Wq, Wk, Wv, Q, K, V, ws, stream)
        ev[1].record(stream)
        mono.route(plan, Q, K, cb, sel, ws, stream=stream)
        mono.attend(plan, Q, K, V, sel, O, ws, stream)
        ev[2].record(stream)
        mono.out_project(plan, O, Wo, delta, ws, stream)
        ev[3].record(stream)

    def step(ev):
        # the breakdown step: every stage through its own entry point, an event after each
        flush.zero_()
        ev[0].record(stream)
        mono.project(plan, x, Wq, Wk, Wv, Q, K, V, ws, stream)
        ev[1].record(stream)
        mono.route_summaries(plan, K, cb, ws, stream)
        ev[2].record(stream)
        mono.route_lists(plan, ws, stream)
        ev[3].record(stream)
        mono.route_queries(plan, Q, cb, sel, ws, stream=stream)
        ev[4].record(stream)
        mono.attend_pairs(plan, sel, ws, stream)
        ev[5].record(stream)
        mono.attend_remote(plan, Q, K, V, ws, stream)
        ev[6].record(stream)
        mono.attend_local(plan, Q, K, V, sel, O, ws, stream)
        ev[7].record(stream)
        mono.out_project(plan, O, Wo, delta, ws, stream)
        ev[8].record(stream)

    mk = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for _ in range(args.warmup):
        step_window(mk(4))
        step(mk(len(names) + 1))
    torch.cuda.synchronize()
    st = mono.stats(plan, ws, stream)
    evs = [mk(4) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    dist.barrier()
    torch.cuda.synchronize()
    launches0 = mono.kernel_launches()
    with sampler:
        t_wall0 = time.perf_counter()
        for k in range(args.steps):
            step_window(evs[k])
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall0
    dist.barrier()
    launches = mono.kernel_launches() - launches0
    ra_ms = [ev[1].elapsed_time(ev[2]) for ev in evs]
    fwd_ms = [ev[0].elapsed_time(ev[3]) for ev in evs]
    # the stage breakdown, from as many separately timed steps (each stage's event time is its kernels' time)
    bevs = [mk(len(names) + 1) for _ in range(args.steps)]
    for k in range(args.steps):
        step(bevs[k])
    torch.cuda.synchronize()
    stage_ms = {n: [] for n in names}
    for ev in bevs:
        for i, n in enumerate(names):
            stage_ms[n].append(ev[i].elapsed_time(ev[i + 1]))
    mean = lambda v: sum(v) / len(v)
    # max over ranks of the per-rank means
    srt = sorted(ra_ms)
    pct = lambda q: srt[min(len(srt) - 1, int(math.ceil(q * len(srt))) - 1)]  # nearest-rank percentile
    lat = dist.reduce_max([statistics.median(ra_ms), pct(0.99), srt[-1]], device=dev)
    agg = dist.reduce_max([mean(ra_ms), mean(fwd_ms), t_wall] + [mean(stage_ms[n]) for n in names], device=dev)
    ra, fwd, wall = agg[0], agg[1], agg[2]
    stage = dict(zip(names, agg[3:]))
    stage_sum = sum(stage[n] for n in window)
    tokens = world * B * S
    value = tokens / (ra / 1e3)

    # roofline: the dominant kernel of the route+attend window (among the stages
    # that are one kernel each, so its event time is that kernel's time), plus the
    # window itself.  "pairs" is three small kernels and is reported as a stage.
    hbm, bf16_tf, peak_kind = peaks()
    npairs = int(st["remote_selected"])
    nblk = int(torch.unique(((torch.arange(B * H, device=dev).view(B, H, 1, 1) * cfg.nb + sel.long())
                             [sel >= 0])).numel())
    ab = algorithmic_bytes(cfg, npairs=npairs, blocks=nblk)
    single_kernel_stages = {"summaries": "k_summary_assign_w",
                            "lists": "k_posting_dense" if cfg.A <= 4096 else "k_posting_build",
                            "queries": probe_kernel(cfg),
                            "remote": "k_remote_tc", "local": "k_local_ws" if cfg.dtype == "bf16" else "k_attend_simt"}
    dom = max(single_kernel_stages, key=lambda n: stage[n])
    achieved = ab[dom] / (stage[dom] / 1e3) / 1e9
    window_gbs = ab["route_attend"] / (ra / 1e3) / 1e9
    traffic = load_traffic(dom, cfg)
    projections = projection_roofline(cfg, stage)

    # end to end through the public API with host buffers, as a serving loop runs it: step i's x goes from
    # pinned host memory to the device on a copy stream while step i-1 computes, and step i-1's delta comes back
    # on another while step i computes (device x and delta double-buffered; events order each buffer's reuse).
    # Every step's copies and its L2 flush are inside the timed region, which spans the whole loop.
    x_host = torch.from_numpy(inp["x"]).to(tdt).pin_memory()
    d_host = [torch.empty(delta.shape, dtype=tdt).pin_memory() for _ in range(2)]
    xb = [x, torch.empty_like(x)]
    db = [torch.empty_like(delta) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_run(n):
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[j])             # step i-2 no longer reads xb[j]
                xb[j].copy_(x_host, non_blocking=True)
                in_done[j].record(s_in)
            stream.wait_event(in_done[j])
            if i >= 2:
                stream.wait_event(out_done[j])                # step i-2's delta has left db[j]
            flush.zero_()
            mono.forward(plan, xb[j], Wq, Wk, Wv, Wo, cb, db[j], ws, stream=stream)
            comp_done[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[j])
                d_host[j].copy_(db[j], non_blocking=True)
                out_done[j].record(s_out)

    e2e_run(max(2, min(args.warmup, 3)))
    torch.cuda.synchronize()
    e2e_t0, e2e_t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_t0.record(s_in)
    stream.wait_event(e2e_t0)
    e2e_run(args.steps)
    e2e_t1.record(s_out)
    torch.cuda.synchronize()
    # the pipeline delivered the staged pass's result (same inputs, deterministic kernels)
    if not torch.equal(d_host[(args.steps - 1) % 2].to(dev), delta):
        raise RuntimeError("end-to-end pipeline: delta differs from the staged pass")
    e2e_ms = dist.reduce_max([e2e_t0.elapsed_time(e2e_t1) / args.steps], device=dev)[0]

    decode = None
    if not args.no_decode:
        try:
            decode = measure_decode(plan, cfg, K, V, inp, tdt, dev, stream, hbm)
        except mono.MonoError as e:   # the decode kernels score every address: C^M <= 4096
            decode = {"unavailable": str(e)}
    backward = measure_backward(plan, cfg, x, Wq, Wk, Wv, Wo, sel, ws, tdt, dev, stream) \
        if not args.no_backward else None

    sweep = None
    if not args.no_sweep and world == 1 and args.workload == "scale32k":
        sweep = s_sweep(args, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, inp, Q, K, V)

    clocks = sampler.summary()
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": fwd, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded N(0,1) x, N(0,1/W) weights, "
                                                              "unit-norm N(0,1) codewords; random-init)",
            "config": {"workload": describe(cfg), "B": B, "S": S, "W": W, "H": H, "d": d, "Bs": cfg.Bs,
                       "L": cfg.L, "R": R, "E": cfg.E, "M": cfg.M, "C": cfg.C, "T": cfg.T, "cap": cfg.cap,
                       "l2": "flushed before every step (256 MiB write, outside the stage events)",
                       "replicas": "one independent replica per GPU (no data-path collective)"},
            "route_attend_ms": ra, "forward_tokens_per_s": tokens / (fwd / 1e3),
            "route_attend_latency": {"median_ms": lat[0], "p99_ms": lat[1], "max_ms": lat[2], "steps": args.steps,
                                     "note": "per timed step; p99 is the nearest-rank percentile (with few steps, the "
                                             "largest); max over ranks"},
            "stage_ms": stage,
            "stage_note": "stage_ms from separately timed steps, each stage through its own entry point; "
                          f"their window sum ({stage_sum:.4f} ms) exceeds route_attend_ms where mono_route "
                          "overlaps the probe with the lists kernel",
            "roofline": {"bound": "hbm", "kernel": single_kernel_stages[dom], "stage": dom, "achieved": achieved,
                         "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": traffic, "algorithmic_bytes": ab[dom],
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"},
            "route_attend_roofline": {"bound": "hbm", "achieved": window_gbs, "peak": hbm, "unit": "GB/s",
                                      "frac": window_gbs / hbm, "algorithmic_bytes": ab["route_attend"]},
            "projections": projections,
            "proj_tensor_frac": projections["qkv"]["frac"],
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": UNIT, "api": "mono_forward",
                    "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                    "d2h_bytes_per_step": int(d_host[0].numel() * d_host[0].element_size()), "ms_per_step": e2e_ms,
                    "pipeline": "H2D of step i and D2H of step i-1 on two copy streams overlap step i's forward; "
                                "timed from the first copy-in to the last copy-out, L2 flush per step included"},
            "gpu_launches": int(launches),
            "clocks": clocks,
            "routing": {"overflow_total": st["overflow_total"], "mean_remote": st["mean_remote"],
                        "queries_lt_R": st["queries_lt_R"]},
            "timed_region_wall_s": wall,
        }
        if decode:
            out["decode"] = decode
        if backward:
            out["backward"] = backward
        if sweep:
            out["s_sweep"] = sweep
        if cpu:
            out["cpu_baseline"] = cpu
        print(json.dumps(out), flush=True)
    dist.finalize()


def measure_decode(plan, cfg, K, V, inp, tdt, dev, stream, hbm, n_steps=128):
    """Decode latency at the end of the context: the cache holds the step's K and V,
    prefilled to S - n_steps; n_steps timed decode steps (B sequences each) follow.
    One warm-up pass over the same positions, then the lists are rebuilt.  Timed
    twice: each step through the API from Python (eager), and the same n_steps
    captured once into a CUDA graph and replayed (device time without the host's
    per-call overhead)."""
    import torch

    from learned_product_hash_proj_b200 import mono
    S, B = cfg.S, cfg.B
    t0 = S - n_steps
    cache = mono.decode_cache(plan, device=dev)
    mono.decode_region(plan, cache, "K").copy_(K)
    mono.decode_region(plan, cache, "V").copy_(V)
    to = lambda a: torch.from_numpy(a).to(tdt).to(dev).contiguous()
    Wq, Wk, Wv, Wo = (to(inp[k]) for k in ("Wq", "Wk", "Wv", "Wo"))
    cb = torch.from_numpy(inp["codebooks"]).to(dev).contiguous()
    xs = [to(inp["x"][:, t, :]) for t in range(t0, S)]
    delta_t = torch.empty((B, cfg.W), dtype=tdt, device=dev)

    def run():
        mono.decode_prefill(plan, t0, cb, cache, stream)
        for i, t in enumerate(range(t0, S)):
            mono.decode_step(plan, t, xs[i], Wq, Wk, Wv, Wo, cb, delta_t, cache, stream=stream)

    run()
    torch.cuda.synchronize()
    mono.decode_prefill(plan, t0, cb, cache, stream)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for i, t in enumerate(range(t0, S)):
        mono.decode_step(plan, t, xs[i], Wq, Wk, Wv, Wo, cb, delta_t, cache, stream=stream)
    ev[1].record(stream)
    torch.cuda.synchronize()
    ms_eager = ev[0].elapsed_time(ev[1]) / n_steps
    # the same steps as one CUDA graph (captured on torch's capture stream)
    g = torch.cuda.CUDAGraph()
    mono.decode_prefill(plan, t0, cb, cache, stream)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i, t in enumerate(range(t0, S)):
            mono.decode_step(plan, t, xs[i], Wq, Wk, Wv, Wo, cb, delta_t, cache)
    mono.decode_prefill(plan, t0, cb, cache, stream)
    torch.cuda.synchronize()
    ev[0].record(stream)
    g.replay()
    ev[1].record(stream)
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / n_steps
    del g
    es = 2 if cfg.dtype == "bf16" else 4
    # bytes a step must read: the four weight matrices, and per (b, h) the K and V
    # rows of its R remote and L local blocks plus E kbar rows
    per_step = 4 * cfg.H * cfg.d * cfg.W * es + B * cfg.H * (
        (cfg.R + cfg.L) * cfg.Bs * cfg.d * es * 2 + cfg.E * cfg.d * 4)
    gbs = per_step / (ms / 1e3) / 1e9
    return {"tokens_per_s": B / (ms / 1e3), "ms_per_token": ms, "ms_per_token_eager": ms_eager, "batch": B,
            "context": t0, "steps": n_steps,
            "api": "mono_decode_step (5 kernels per step, 6 when a block completes); ms_per_token from a CUDA "
                   "graph of the steps, ms_per_token_eager from one Python call per step",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "algorithmic_bytes": per_step}}


# fp32 FMA peak from the unit counts: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def measure_backward(plan, cfg, x, Wq, Wk, Wv, Wo, sel, ws, tdt, dev, stream, steps=3):
    """mono_backward for the step's selection and a seeded upstream gradient: mean of `steps`
    timed calls after one warm-up.  Algorithmic flops: the forward recompute (projection and
    selected-set attention), the projection gradients (8 GEMMs of B*S x H*d x W) and the
    attention gradients (per query and selected key 5 products of d multiply-adds: the score,
    dO . v, and the dS k, dS q, P dO terms).  With bf16 storage the GEMMs and the forward
    attention run on the tensor cores; the attention gradients do too where the library's
    tensor-core backward takes the shape (Bs = 64, d = 64 with L <= 2 or d = 128 with L = 1),
    else they run on the fp32 lanes, and the roofline's target time is the sum of the two parts
    at their own peaks."""
    import torch

    from learned_product_hash_proj_b200 import mono
    B, S, W, H, d = cfg.B, cfg.S, cfg.W, cfg.H, cfg.d
    g = torch.Generator(device="cpu").manual_seed(11)
    ddelta = torch.randn((B, S, W), generator=g).to(tdt).to(dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dx = torch.empty((B, S, W), **f32)
    dWq, dWk, dWv = (torch.empty((H * d, W), **f32) for _ in range(3))
    dWo = torch.empty((W, H * d), **f32)
    bws = mono.backward_workspace(plan, device=dev)
    run = lambda: mono.backward(plan, x, Wq, Wk, Wv, Wo, sel, ddelta, dx, dWq, dWk, dWv, dWo, ws, bws, stream=stream)
    run()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for _ in range(steps):
        run()
    ev[1].record(stream)
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / steps
    nsel = int((sel >= 0).sum().item())
    keys = nsel * cfg.Bs + B * H * S * ((cfg.L - 1) * cfg.Bs + (cfg.Bs + 1) / 2)   # selected keys, all queries
    gemm = 2.0 * B * S * H * d * W
    fwd_attn = 2 * keys * 2 * d
    bwd_attn = 5 * keys * 2 * d
    flops = 3 * gemm + fwd_attn + 8 * gemm + bwd_attn
    nk = 128 + (cfg.L - 1) * cfg.Bs
    attn_tc = cfg.dtype == "bf16" and cfg.Bs == 64 and ((d == 64 and nk <= 192) or (d == 128 and nk <= 128))
    tensor = (11 * gemm + fwd_attn + (bwd_attn if attn_tc else 0.0)) if cfg.dtype == "bf16" else 0.0
    alu = flops - tensor
    tpeak, tsrc = bf16_sustained_peak()
    target_s = tensor / (tpeak * 1e12) + alu / (FP32_PEAK_TFLOPS * 1e12)
    tf = flops / (ms / 1e3) / 1e12
    eff_peak = flops / target_s / 1e12
    return {"ms": ms, "tokens_per_s": B * S / (ms / 1e3),
            "api": "mono_backward (forward recompute + gradients of x, Wq, Wk, Wv, Wo for a fixed selection)",
            "roofline": {"bound": "tensor" if alu == 0 else "tensor+alu", "achieved": tf, "peak": eff_peak,
                         "unit": "TFLOP/s",
                         "frac": tf / eff_peak, "target_ms": target_s * 1e3, "algorithmic_flops": flops,
                         "tensor_flops": tensor, "alu_flops": alu, "peak_tensor_tflops": tpeak,
                         "peak_alu_tflops": FP32_PEAK_TFLOPS,
                         "peak_source": f"{tsrc} bf16_tflops_sustained (MEASURED_PEAKS.json) for the tensor part; "
                                        "fp32 lanes x clock (148 x 128 x 2 x 1.965 GHz) for the rest"}}


def probe_kernel(cfg) -> str:
    """The probe kernel the library launches for this shape (its dispatch in csrc/route.cu)."""
    shape = (cfg.d, cfg.C, cfg.T, cfg.E, cfg.R)
    if cfg.M == 2 and ((cfg.dtype == "bf16" and shape in ((64, 16, 4, 5, 2), (128, 32, 8, 8, 4))) or
                       (cfg.dtype != "bf16" and shape in ((64, 16, 4, 5, 2), (64, 8, 4, 5, 2)))):
        return "k_probe_m2"
    if cfg.M == 4 and ((cfg.dtype == "bf16" and shape in ((128, 16, 16, 8, 4), (64, 16, 16, 5, 2), (64, 4, 8, 8, 4)))
                       or (cfg.dtype != "bf16" and shape == (64, 4, 8, 8, 4))):
        return "k_probe_bf"
    return "k_probe_rerank"


def projection_roofline(cfg, stage: dict) -> dict:
    """Tensor-pipe fraction of the projection GEMMs (outside the route+attend metric): algorithmic flops
    (2 M N K per GEMM: Q/K/V = 3 GEMMs of B*S x H*d x W, the output projection one of B*S x W x H*d) over the
    stage's event time, against the measured sustained bf16 peak (the GEMMs run inside a long step)."""
    tpeak, tsrc = bf16_sustained_peak()
    gemm = 2.0 * cfg.B * cfg.S * cfg.H * cfg.d * cfg.W
    out = {}
    for name, st, fl in (("qkv", "project", 3 * gemm), ("out", "out_project", gemm)):
        tf = fl / (stage[st] / 1e3) / 1e12
        out[name] = {"bound": "tensor", "achieved": tf, "peak": tpeak, "unit": "TFLOP/s", "frac": tf / tpeak,
                     "algorithmic_flops": fl, "ms": stage[st],
                     "kernel": ("k_gemm_tcp" if (cfg.H * cfg.d if name == "qkv" else cfg.W) % 256 == 0 else "k_gemm_tc")
                     if cfg.dtype == "bf16" else "k_gemm_simt"}
    out["peak_source"] = f"{tsrc} bf16_tflops_sustained (MEASURED_PEAKS.json)"
    if cfg.dtype != "bf16":
        out["note"] = "fp32 storage runs the SIMT GEMM; the bf16 tensor peak is a reference only"
    return out


def host_cpu() -> dict:
    """The host's CPU model and how many cores this process may use (for the CPU-baseline record)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count()
    return {"cpu_model": model, "nproc": usable}


def load_traffic(stage: str, cfg):
    """DRAM read+write bytes per launch of the stage's kernel, from the committed ncu summary
    (profiles/traffic.json), or None when the summary does not cover this workload."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t.get(cfg.name, {}).get(stage)
        return None if e is None else float(e["bytes_per_launch"])
    except Exception:
        return None


def s_sweep(args, dev):
    """route+attend time at S = 4K..32K and the fitted time-vs-S exponent."""
    import torch

    from learned_product_hash_proj_b200 import mono, synth
    pts = []
    for k in (4, 8, 16, 32):
        cfg = synth.config(f"scale{k}k")
        inp = synth.make_inputs(cfg, 7)
        tdt = torch.bfloat16
        to = lambda a: torch.from_numpy(a).to(tdt).to(dev).contiguous()
        x, Wq, Wk, Wv = (to(inp[n]) for n in ("x", "Wq", "Wk", "Wv"))
        cb = torch.from_numpy(inp["codebooks"]).to(dev).contiguous()
        plan = mono.Plan(cfg)
        ws = plan.workspace(dev)
        Q = torch.empty((1, cfg.H, cfg.S, cfg.d), dtype=tdt, device=dev)
        K, V = torch.empty_like(Q), torch.empty_like(Q)
        sel = torch.empty((1, cfg.H, cfg.S, cfg.R), dtype=torch.int32, device=dev)
        O = torch.empty((1, cfg.S, cfg.H * cfg.d), dtype=tdt, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        mono.project(plan, x, Wq, Wk, Wv, Q, K, V, ws)
        times = []
        for it in range(3 + 10):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            mono.route(plan, Q, K, cb, sel, ws)
            mono.attend(plan, Q, K, V, sel, O, ws)
            b.record()
            torch.cuda.synchronize()
            if it >= 3:
                times.append(a.elapsed_time(b))
        pts.append((cfg.S, statistics.median(times)))
        del ws, Q, K, V, O, sel, flush
    xs = np.log([p[0] for p in pts])
    ys = np.log([p[1] for p in pts])
    slope = float(np.polyfit(xs, ys, 1)[0])
    return {"S": [p[0] for p in pts], "route_attend_ms_median": [p[1] for p in pts], "exponent": slope}


# ---------------------------------------------------------------------------
# CPU baseline and the reference arm: the oracle, as it stands
# ---------------------------------------------------------------------------
def oracle_route_attend(cfg, Q1, K1, V1, cb1, qidx=None):
    """Oracle route+attend for one (batch, head) slice (arrays [1,1,S,d]); returns seconds."""
    import oracle
    one = cfg.with_(B=1, H=1)
    t0 = time.perf_counter()
    kbar, addr, _ = oracle.summary_assign(one, K1, cb1)
    oracle.posting(one, addr)
    t1 = time.perf_counter()
    sel, *_ = oracle.route_queries(one, Q1, kbar, cb1, addr, qidx=qidx)
    if qidx is None:
        sel_full = sel
    else:
        sel_full = np.full((1, 1, cfg.S, cfg.R), -1, np.int32)
        sel_full.reshape(-1, cfg.R)[qidx] = sel
    oracle.attend(one, Q1.astype(np.float64), K1.astype(np.float64), V1.astype(np.float64), sel_full, qidx=qidx)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def cpu_baseline(cfg, inp, Q, K, V, n_heads: int = 4):
    """The oracle's route+attend on the GPU's Q/K/V for `n_heads` heads of batch 0, extrapolated to the whole
    workload: each head's summaries and lists in full, and the route+attend of all its queries, or, where the
    oracle's sort of the whole address grid per query makes that slow (C^M > 256), of a seeded sample of about
    4e6 / C^M queries (at least 256), scaled by S / sample.  About 4-15 s of single-threaded work."""
    import oracle
    oracle.build()
    n_heads = min(n_heads, cfg.H)
    n_q = cfg.S if cfg.A <= 256 else min(cfg.S, max(256, int(4e6 // cfg.A)))
    qidx = None if n_q == cfg.S else np.sort(np.random.default_rng(5).choice(cfg.S, n_q, replace=False))
    t_tab = t_q = 0.0
    for h in range(n_heads):
        sl = [t[0:1, h:h + 1].float().cpu().numpy() for t in (Q, K, V)]
        cb1 = np.ascontiguousarray(inp["codebooks"][h:h + 1])
        a, b = oracle_route_attend(cfg, *sl, cb1, qidx=None if qidx is None else qidx.astype(np.int64))
        t_tab += a
        t_q += b
    per_slice = (t_tab + t_q * cfg.S / n_q) / n_heads
    est = per_slice * cfg.B * cfg.H
    q_txt = f"all {cfg.S} queries" if qidx is None else f"a seeded sample of {n_q} of its {cfg.S} queries"
    return {"value": cfg.B * cfg.S / est, "unit": UNIT, "cores": 1, "kind": "oracle", **host_cpu(),
            "sample": f"heads 0..{n_heads - 1} of {cfg.H} (batch 0): summaries and lists of each slice in full, "
                      f"route+attend of {q_txt}, on the GPU's Q/K/V; {t_tab + t_q:.1f} s single-threaded, "
                      f"extrapolated linearly to {cfg.B} x {cfg.H} slices x {cfg.S} queries"}


def run_reference(args):
    from learned_product_hash_proj_b200 import dist, synth
    rank, _, world = dist.env_rank()
    if rank != 0:
        return
    import oracle
    oracle.build()
    cfg = synth.config(args.workload)
    inp = synth.make_inputs(cfg.with_(B=1), args.seed)
    one = cfg.with_(B=1, H=1)
    h = 0
    sl = slice(h * cfg.d, (h + 1) * cfg.d)
    log("reference arm: oracle projection of head 0 (setup, untimed)")
    Q1, K1, V1 = oracle.project(one, inp["x"][:1], inp["Wq"][sl], inp["Wk"][sl], inp["Wv"][sl])
    Q1, K1, V1 = (oracle.round_storage(a, cfg.dtype) for a in (Q1, K1, V1))
    cb1 = np.ascontiguousarray(inp["codebooks"][h:h + 1])
    rng = np.random.default_rng(args.seed)
    n_q = min(cfg.S, 4096)
    qidx = np.sort(rng.choice(cfg.S, size=n_q, replace=False)).astype(np.int64)
    per_step = []
    for k in range(args.warmup + args.steps):
        a, b = oracle_route_attend(cfg, Q1, K1, V1, cb1, qidx=qidx)
        if k >= args.warmup:
            per_step.append((a, b))
    t_tables = statistics.mean(p[0] for p in per_step)
    t_queries = statistics.mean(p[1] for p in per_step)
    est = cfg.B * cfg.H * (t_tables + t_queries * cfg.S / n_q)
    value = cfg.B * cfg.S / est
    sample = (f"per step: summaries+lists of one (batch, head) slice plus route+attend of {n_q} of its {cfg.S} "
              f"queries; extrapolated linearly to {cfg.B * cfg.H} slices x {cfg.S} queries")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * statistics.mean(a + b for a, b in per_step), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": describe(cfg)},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                            **host_cpu()},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="scale32k")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode latency measurement")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass measurement")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        log("warm-up raised to 3 steps (timing rule)")
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
