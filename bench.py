"""Benchmark of the MoE routing hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    (N > 1: launched by torch.distributed.run, one process per GPU)

One step = one pass of the routing path over one batch of the throughput
workload (T=16384 tokens, d=7168, N=256 experts, K=8, sigmoid scores, 8 groups
keep 4, bias, weights x2.5):
  moe_route_tiles      gate GEMM (tcgen05) + sigmoid + group-limited top-K +
                       weights + per-tile expert histograms, all in the GEMM
                       epilogue (no scores in memory)
  moe_load_stats_tiles histogram, offsets, in-expert ranks, load stats
  moe_bias_update      sign-rule bias step
  moe_dispatch         bf16 rows into the expert-contiguous buffer (+ positions)
(--unfused: moe_route writing the scores, the selection kernel, moe_load_stats.)
Combine is timed in its own loop (identity experts: it gathers the
dispatched rows back) and reported under "stages".

Schedule: by default the steps are software-pipelined -- the routing of batch
i+1 runs on a high-priority stream beside the dispatch of batch i (see
expert_load_balancing_tcgen05_b200/step.py); the results are those of the
serial order.  --serial times the calls one after another instead.  The
per-stage times under "stages" always come from the serial schedule.

Metric: routed tokens/s = tokens of all ranks / max-over-ranks device time.
Inputs are synthetic (seeded, drawn on the device) and larger than L2, so no
flush is needed between steps.  Rank 0 prints one JSON line.

--impl reference runs the CPU oracle (the plain fp64 restatement the tests
use) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
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

METRIC = "routed tokens/s (gate+topK+hist+dispatch) T=16K N=256 K=8; % roofline"
UNIT = "tokens/s"
WORKLOAD_NAME = "metric"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), \
            "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload_config(wl):
    return {"workload": f"{wl.name}: T={wl.T} d={wl.d} N={wl.N} K={wl.K} sigmoid, {wl.n_groups} groups keep "
                        f"{wl.topk_groups}, group score top-{wl.group_topn} sum, bias U(-0.01,0.01), "
                        f"weights x{wl.scale}, bf16 x~N(0,1) W~N(0,1/d)",
            "T": wl.T, "d": wl.d, "N": wl.N, "K": wl.K,
            "l2": "inputs larger than L2 (x 235 MB, dispatch buffer 1.88 GB per rank); consecutive steps "
                  "alternate between two distinct token batches; no flush"}


# --------------------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        # inside the working tree (git-ignored), not the system temp directory
        fd, self.path = tempfile.mkstemp(prefix=".clocks_", suffix=".csv", dir=ROOT)
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        return rows

    @staticmethod
    def summarise(rows):
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for n, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        loaded = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded)}


# --------------------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------------------
def make_step(wl, rank, dev, world, pipelined, fused=None, gate_ctas=None):
    """The routing step on this rank's batches (inputs drawn on the device).
    Consecutive steps alternate between two distinct token batches in
    different buffers, so that overlapped steps never share rows of x in L2."""
    from expert_load_balancing_tcgen05_b200 import workloads as W
    from expert_load_balancing_tcgen05_b200.step import RoutingStep
    inp = W.make_inputs(wl, device=dev, seed=wl.seed + 100 * rank)
    x2 = W.make_inputs(wl, device=dev, seed=wl.seed + 100 * rank + 50)["x"]
    return RoutingStep(wl, [inp["x"], x2], inp["W"], inp["bias"].clone(), inp["off"], dev, world=world,
                       pipelined=pipelined, fused=fused, gate_max_ctas=gate_ctas if pipelined else None)


def routing_path(args):
    """None (the step's default: the fused path where the epilogue can select), or False with --unfused."""
    return False if args.unfused else None


def stage_bytes(wl, fused=False):
    """Algorithmic bytes / flops per launch (per batch of T tokens).  The
    fused path keeps the scores on chip: its gate writes the choices (and the
    tile histograms) instead of the scores, and there is no separate
    selection stage reading them back."""
    T, d, N, K = wl.T, wl.d, wl.N, wl.K
    A = T * K
    if fused:
        tiles = (T + 127) // 128 * 2 * N * 4
        return {
            "gate": {"bytes": T * d * 2 + N * d * 2 + A * 8 + tiles, "flops": 2 * T * d * N},
            "topk": {"bytes": 0},
            "hist": {"bytes": A * 4 * 2 + A * 4 + tiles + (N + 1) * 4 * 2},
            "dispatch": {"bytes": T * d * 2 + A * d * 2 + A * 12},
            "combine": {"bytes": A * d * 2 + A * 8 + T * d * 2},
        }
    return {
        "gate": {"bytes": T * d * 2 + N * d * 2 + T * N * 4, "flops": 2 * T * d * N},
        "topk": {"bytes": T * N * 4 + N * 4 + A * 8},
        "hist": {"bytes": A * 4 * 2 + A * 4 + (N + 1) * 4 * 2},   # idx read, slot+rank write, rank rw, offsets
        "dispatch": {"bytes": T * d * 2 + A * d * 2 + A * 12},     # x once, K row copies, slot/rank in, pos out
        "combine": {"bytes": A * d * 2 + A * 8 + T * d * 2},       # K rows in, pos/w in, token row out
    }


def pipeline_roofline_us(wl, hbm_gbs, tflops, overlapped=False, fused=False):
    """Serial schedule: the stages one after another, each at the slower of
    its HBM and tensor bounds.  Overlapped schedule (routing of the next
    batch beside the dispatch): all stages share HBM, so the bound is the
    step's total bytes over HBM bandwidth, or the gate's tensor time if that
    is longer."""
    b = stage_bytes(wl, fused)
    stages = ("gate", "topk", "hist", "dispatch")
    if overlapped:
        tb = sum(b[k]["bytes"] for k in stages) / (hbm_gbs * 1e9)
        tf = b["gate"]["flops"] / (tflops * 1e12)
        return max(tb, tf) * 1e6
    t = 0.0
    for k in stages:
        tb = b[k]["bytes"] / (hbm_gbs * 1e9)
        tf = b[k].get("flops", 0) / (tflops * 1e12)
        t += max(tb, tf)
    return t * 1e6


def _traffic_for(kernel_file: str, summary: str):
    """dram bytes per launch from a committed ncu summary, if the kernel
    source is unchanged since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "expert_load_balancing_tcgen05_b200", "csrc", kernel_file)
    if not (os.path.exists(p) and os.path.exists(src)):
        return None
    with open(p) as f:
        j = json.load(f)
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    if j.get("source_sha256") != h:
        return None
    return j.get("dram_bytes_per_launch")


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from expert_load_balancing_tcgen05_b200 import moe
    from expert_load_balancing_tcgen05_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = W.WORKLOADS[WORKLOAD_NAME]
    pipelined = not args.serial
    P = make_step(wl, rank, dev, world, pipelined, fused=routing_path(args), gate_ctas=args.gate_ctas)
    P_fused = P.fused
    hbm, tf_burst, tf_sust, peak_kind = _peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    # clocks are sampled from before the warm-up to after the timed region
    sampler = ClockSampler(local_rank)
    sampler.start()
    # warm-up (also ramps clocks) and a correctness status check
    w0 = time.time()
    n_warm = max(args.warmup, 3)
    for _ in range(n_warm):
        P.step()
    torch.cuda.synchronize()
    st = moe.moe_workspace_status(P.ws)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device-side status {st} after warm-up")
    # every rank runs the same number of steps (each holds one collective at
    # N > 1): loop counts come from the slowest rank's warm-up step time
    t_step = torch.tensor([(time.time() - w0) / n_warm], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t_step, op=dist.ReduceOp.MAX)
    t_step = max(float(t_step.item()), 1e-4)

    def soak(seconds):
        for _ in range(max(1, min(5000, int(seconds / t_step)))):
            P.step()
        torch.cuda.synchronize()

    # soak ~0.6 s so the sampler sees the loaded clock before and during timing
    soak(0.6)

    E = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    moe.moe_launch_count(reset=True)
    barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    P.fence()
    for i in range(args.steps):
        P.step(dispatch_events=E[i])
    stop.record()
    torch.cuda.synchronize()
    barrier()
    launches = moe.moe_launch_count()
    # keep the sampler running over a few more steps so short timed regions still get samples
    soak(0.4)
    clocks = sampler.summarise(sampler.stop())
    ms = start.elapsed_time(stop)
    t_disp = statistics.mean(a.elapsed_time(b) for a, b in E)
    del P
    torch.cuda.empty_cache()
    if args.timed_only:
        # a sweep point: the timed region only (no serial stages, combine or end-to-end leg)
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())
        return {"metric": METRIC, "value": wl.T * args.steps * world / (ms_max / 1e3), "unit": UNIT,
                "ms_per_step": ms_max / args.steps, "timed_only": True, "fused": not args.unfused,
                "gate_ctas": args.gate_ctas, "dispatch_ms_in_timed_region": t_disp, "clocks": clocks} \
            if rank == 0 else None

    # the serial schedule: per-stage times (route, load statistics + bias
    # step, dispatch), the combine loop and the end-to-end leg
    S = make_step(wl, rank, dev, world, pipelined=False, fused=routing_path(args))
    for _ in range(3):
        S.step()
    n_stage = max(3, min(args.steps, 50))
    SE = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_stage)]
    torch.cuda.synchronize()
    barrier()
    for i in range(n_stage):
        S.step(stage_events=SE[i])
    torch.cuda.synchronize()
    t_route = statistics.mean(e[0].elapsed_time(e[1]) for e in SE)
    t_stats = statistics.mean(e[1].elapsed_time(e[2]) for e in SE)
    t_disp_serial = statistics.mean(e[2].elapsed_time(e[3]) for e in SE)
    t_serial_step = statistics.mean(e[0].elapsed_time(e[3]) for e in SE)

    # combine: own loop (identity experts: gathers the dispatched rows back)
    out_rows = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        moe.moe_combine(S.rows, wl.T, wl.d, wl.K, S.pos, S.w, out_rows)
    cs, ce = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    cs.record()
    for _ in range(args.steps):
        moe.moe_combine(S.rows, wl.T, wl.d, wl.K, S.pos, S.w, out_rows)
    ce.record()
    torch.cuda.synchronize()
    t_comb = cs.elapsed_time(ce) / args.steps

    # max over ranks
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    tokens = wl.T * args.steps * world
    value = tokens / (ms_max / 1e3)

    # end to end through the public API with host buffers: every step copies
    # its tokens from pinned host memory (a copy stream, two device buffers,
    # so the copy of batch i+1 overlaps the work on batch i), runs the step
    # in the same schedule as the timed region, and reads its routing result
    # back (idx, weights, offsets, counts, stats); the dispatched rows stay on
    # the device for the expert GEMMs.
    del S
    torch.cuda.empty_cache()
    E2 = make_step(wl, rank, dev, world, pipelined, fused=routing_path(args), gate_ctas=args.gate_ctas)
    x_host = E2.x.cpu().pin_memory()
    x_dev = [torch.empty_like(E2.x) for _ in range(2)]
    res_host = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in E2.results(E2.sets[0])]
    h2d = x_host.numel() * x_host.element_size()
    d2h = sum(r.numel() * r.element_size() for r in res_host)
    copy_stream = torch.cuda.Stream(device=dev)
    main = torch.cuda.current_stream(dev)
    ev_copied = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]

    def e2e_loop(n):
        copy_stream.wait_stream(main)
        E2.fence()
        for i in range(n):
            bb = i % 2
            if i >= 2:
                copy_stream.wait_event(ev_free[bb])  # the step that read this buffer is done
            with torch.cuda.stream(copy_stream):
                x_dev[bb].copy_(x_host, non_blocking=True)
            ev_copied[bb].record(copy_stream)
            E2.step(x_dev[bb], ready=ev_copied[bb], host_out=res_host)
            ev_free[bb].record(main)

    e2e_steps = max(3, min(args.steps, 20))
    e2e_loop(2)
    torch.cuda.synchronize()
    barrier()
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es.record()
    e2e_loop(e2e_steps)
    ee.record()
    torch.cuda.synchronize()
    te = torch.tensor([es.elapsed_time(ee)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_value = wl.T * e2e_steps * world / (float(te.item()) / 1e3)

    b = stage_bytes(wl, fused=P_fused)
    disp_bytes = b["dispatch"]["bytes"]
    achieved = disp_bytes / (t_disp / 1e3) / 1e9
    traffic = _traffic_for("dispatch_combine.cu", "dispatch_metric_dram.json")
    roof_us = pipeline_roofline_us(wl, hbm, tf_burst, overlapped=pipelined, fused=P_fused)
    ms_step = ms_max / args.steps

    out = None
    if rank == 0:
        from expert_load_balancing_tcgen05_b200.step import PIPELINED_GATE_CTAS
        schedule = ("pipelined: the routing of batch i+1 (gate on "
                    f"{PIPELINED_GATE_CTAS} SMs, selection, load statistics, bias step) on a high-priority stream beside "
                    "the dispatch of batch i") if pipelined else "serial: one call after another on one stream"
        schedule += ("; routing through the fused path (selection and per-tile histograms in the gate's epilogue, "
                     "no scores in memory; statistics from the tile histograms)") if not args.unfused else \
            "; routing through the gate's scores epilogue and the selection kernel"
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(wl), "schedule": schedule,
                       "parallelism": (f"dp{world} (token shards; one all-reduce of the {wl.N} expert counts per "
                                       "step for the shared bias, in the routing stream)") if world > 1
                       else "dp1 (independent token batches)"},
            "roofline": {"bound": "hbm", "kernel": "dispatch_kernel", "achieved": achieved, "peak": hbm,
                         "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                         "bytes_per_launch": disp_bytes, "peak_kind": f"{peak_kind} hbm_gbs (copy)",
                         "timed": "average dispatch launch in the timed region" +
                                  (" (sharing the GPU with the next batch's routing)" if pipelined else ""),
                         "frac_alone": disp_bytes / (t_disp_serial / 1e3) / 1e9 / hbm},
            "pipeline_roofline": {"time_us": roof_us, "frac": roof_us / (ms_step * 1e3),
                                  "tokens_per_s_at_roofline": wl.T / (roof_us / 1e6),
                                  "rule": ("max(total bytes of gate/topK/hist/dispatch / HBM peak, gate flops / "
                                           "bf16 burst peak): the stages overlap") if pipelined else
                                          ("sum over gate/topK/hist/dispatch of max(flops/bf16 burst peak, "
                                           "bytes/HBM peak)")},
            "stages": {
                "serial_step_ms": t_serial_step,
                "route_ms": t_route, "load_stats_and_bias_ms": t_stats, "dispatch_ms": t_disp_serial,
                "dispatch_ms_in_timed_region": t_disp,
                "combine_ms": t_comb,
                "gate_topk_gbs_equiv": (b["gate"]["bytes"] + b["topk"]["bytes"]) / (t_route / 1e3) / 1e9,
                "routing_path": "fused (moe_route_tiles + moe_load_stats_tiles)" if P_fused else
                                "scores (moe_route + moe_load_stats)",
                "gate_tflops_lower_bound": b["gate"]["flops"] / (t_route / 1e3) / 1e12,
                "dispatch_gbs_serial": disp_bytes / (t_disp_serial / 1e3) / 1e9,
                "combine_gbs": b["combine"]["bytes"] / (t_comb / 1e3) / 1e9,
            },
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps,
                    "schedule": ("copy of batch i+1 from pinned host memory beside the work on batch i; " +
                                 ("pipelined step" if pipelined else "serial step"))},
            "gpu_launches": launches,
            "clocks": clocks,
        }
    return out


def cpu_baseline(seconds: float = 12.0):
    """The oracle, as it stands, on the host cores: fp64 gate + scores +
    selection + histogram/positions + dispatch rows for a sample of tokens of
    the throughput workload; tokens/s scaled from the sample."""
    import numpy as np
    import torch

    import oracle
    from expert_load_balancing_tcgen05_b200 import workloads as W
    wl = W.WORKLOADS[WORKLOAD_NAME]

    def run(n):
        sw = wl.with_(T=n)
        inp = W.make_inputs(sw, seed=wl.seed)
        x = inp["x"].float().numpy()
        Wg = inp["W"].float().numpy()
        b = inp["bias"].numpy()
        x16 = inp["x"].view(torch.int16).numpy()
        t0 = time.perf_counter()
        h = oracle.logits(x, Wg)
        s = oracle.scores(h, wl.fn)
        idx, w = oracle.select(s, b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
        counts, offsets, pos, rk, src = oracle.positions(idx, wl.N)
        oracle.load_stats(counts)
        oracle.bias_update(counts, n * wl.K, b, 0.001, 0)
        oracle.dispatch_rows(x16, pos)
        return time.perf_counter() - t0

    probe = 64
    tp = run(probe)
    n = int(max(probe, min(wl.T, probe * seconds / max(tp, 1e-3))))
    dt = run(n)
    return {"value": n / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} tokens of the {WORKLOAD_NAME} workload (T={wl.T} d={wl.d} N={wl.N} K={wl.K}): "
                      f"fp64 gate, scores, grouped top-K, histogram/positions, stats, bias step, dispatch rows; "
                      f"{dt:.1f} s wall"}


def run_reference(args):
    """The CPU oracle as the reference arm: W warm-up + K timed steps, each a
    bounded sample of the throughput workload."""
    import oracle
    from expert_load_balancing_tcgen05_b200 import workloads as W
    import torch
    wl = W.WORKLOADS[WORKLOAD_NAME]
    n = int(os.environ.get("REF_SAMPLE_TOKENS", "1024"))
    sw = wl.with_(T=n)
    inp = W.make_inputs(sw, seed=wl.seed)
    x = inp["x"].float().numpy()
    Wg = inp["W"].float().numpy()
    b = inp["bias"].numpy()
    x16 = inp["x"].view(torch.int16).numpy()

    def step():
        h = oracle.logits(x, Wg)
        s = oracle.scores(h, wl.fn)
        idx, w = oracle.select(s, b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
        counts, offsets, pos, rk, src = oracle.positions(idx, wl.N)
        oracle.load_stats(counts)
        oracle.bias_update(counts, n * wl.K, b, 0.001, 0)
        oracle.dispatch_rows(x16, pos)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = (f"{n} tokens per step of the {WORKLOAD_NAME} workload (T={wl.T} d={wl.d} N={wl.N} K={wl.K}), "
              f"fp64 oracle on the host cores")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**workload_config(wl), "sample_tokens": n},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_kernel_report(only=None):
    """Per-call device times of the library on every workload (3 warm-up
    calls, then 10 calls captured in a CUDA graph and replayed under CUDA
    events), each against its bound: HBM
    bytes over the copy bandwidth, or the gate's flops over the bf16 burst
    peak if longer (the measured peaks when present, else the fallback).  Prints a markdown table (not the
    benchmark's JSON line)."""
    import torch
    from expert_load_balancing_tcgen05_b200 import moe
    from expert_load_balancing_tcgen05_b200 import workloads as W
    hbm, tf_burst, _, peak_kind = _peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    def t_us(fn, n=10):
        # n calls captured in a CUDA graph and replayed: device time, without
        # the host's launch rate
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / n * 1e3

    rows = []

    def add(wl, call, us, nbytes, flops=0, note=""):
        bound = max(nbytes / (hbm * 1e9), flops / (tf_burst * 1e12)) * 1e6
        rows.append((wl.name, f"T={wl.T} d={wl.d} N={wl.N} K={wl.K}", call, us, bound, bound / us, note))

    names = ("tiny_softmax", "v3_router", "collapse", "softmax_dispatch", "prefill_replicas", "metric")
    for name in names:
        if only is not None and name != only:
            continue
        # a short idle gap first: after the large workloads' seconds of full-power
        # work the clocks take a moment to recover, which the next rows would see
        torch.cuda.synchronize()
        time.sleep(2.0)
        wl = W.WORKLOADS[name]
        T, d, N, K = wl.T, wl.d, wl.N, wl.K
        A = T * K
        es = 2 if wl.dtype == torch.bfloat16 else 4
        inp = W.make_inputs(wl, device=dev, seed=wl.seed, with_y=wl.combine)
        x, Wg, off, bias = inp["x"], inp["W"], inp["off"], inp["bias"]
        scores = torch.empty(T, N, device=dev)
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        w = torch.empty(T, K, device=dev)
        n_slots = wl.n_slots
        ws = moe.workspace(T, K, N, n_slots, device=dev)
        dt = moe.MOE_BF16 if wl.dtype == torch.bfloat16 else moe.MOE_F32
        cfg = moe.route_cfg(T, d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale, dt)
        route = lambda: moe.moe_route(cfg, x, Wg, off, bias, scores, idx, w, ws)
        add(wl, "moe_route (gate + selection)", t_us(route), T * d * es + N * d * es + T * N * 4 + A * 8,
            2 * T * d * N)
        sel = lambda: moe.moe_route(cfg, None, None, None, bias, scores, idx, w, ws)
        add(wl, "  selection alone (scores given)", t_us(sel), T * N * 4 + A * 8)
        fusable = wl.dtype == torch.bfloat16 and N in (64, 128, 256) and K <= 8 and \
            (wl.n_groups == 1 or (wl.fn == moe.MOE_SIGMOID and N // wl.n_groups == 32))
        tiles = None
        if fusable:
            tiles = torch.empty(moe.tile_counts_shape(T, N), dtype=torch.int32, device=dev)
            rt = lambda: moe.moe_route_tiles(cfg, x, Wg, off, bias, idx, w, tiles, ws)
            add(wl, "moe_route_tiles (gate + selection + tile histograms in the epilogue)", t_us(rt),
                T * d * es + N * d * es + A * 8 + tiles.numel() * 4, 2 * T * d * N)
        route()
        slot = torch.empty(T, K, dtype=torch.int32, device=dev)
        rank = torch.empty(T, K, dtype=torch.int32, device=dev)
        counts = torch.empty(n_slots, dtype=torch.int32, device=dev)
        offsets = torch.empty(n_slots + 1, dtype=torch.int32, device=dev)
        stats = moe.empty_stats(dev)
        rep = None
        if wl.n_replicas:
            moe.moe_load_stats(idx, T, K, N, None, N, slot, counts[:N], offsets[:N + 1], rank, None, wl.fn, stats,
                               ws)
            rep = torch.empty(N, dtype=torch.int32, device=dev)
            moe.moe_replica_plan(counts[:N], N, wl.n_replicas, rep)
            add(wl, "moe_replica_plan", t_us(lambda: moe.moe_replica_plan(counts[:N], N, wl.n_replicas, rep)),
                N * 8)
        ls = lambda: moe.moe_load_stats(idx, T, K, N, rep, n_slots, slot, counts, offsets, rank, None, wl.fn, stats,
                                        ws)
        add(wl, "moe_load_stats", t_us(ls), A * 12 + n_slots * 8, note="latency-bound (single-pass scan)")
        if tiles is not None:
            moe.moe_route_tiles(cfg, x, Wg, off, bias, idx, w, tiles, ws)
            lst = lambda: moe.moe_load_stats_tiles(idx, T, K, N, tiles, rep, n_slots, slot, counts, offsets, rank,
                                                   stats, ws)
            add(wl, "moe_load_stats_tiles", t_us(lst), A * 12 + tiles.numel() * 4 + n_slots * 8,
                note="latency-bound (single-pass scan)")
        ls()
        if wl.bias_steps or wl.has_bias:
            b2 = bias.clone() if bias is not None else torch.zeros(N, device=dev)
            add(wl, "moe_bias_update", t_us(lambda: moe.moe_bias_update(counts[:N], N, A, 0.001, 0, b2)), N * 8,
                note="one block")
        rows_b = torch.empty(A, d, dtype=wl.dtype, device=dev)
        pos = torch.empty(T, K, dtype=torch.int32, device=dev)
        disp = lambda: moe.moe_dispatch(x, T, d, K, slot, offsets, rank, rows_b, None, None, pos, None)
        add(wl, "moe_dispatch", t_us(disp), T * d * es + A * d * es + A * 12)
        if wl.fp8:
            q = torch.empty(A, d, dtype=torch.uint8, device=dev)
            sc = torch.empty(A, d // 128, device=dev)
            disp8 = lambda: moe.moe_dispatch(x, T, d, K, slot, offsets, rank, rows_b, q, sc, pos, None)
            add(wl, "moe_dispatch + FP8 copy", t_us(disp8), T * d * es + A * d * (es + 1) + A * d // 32 + A * 12)
            del q, sc
        disp()
        y = inp.get("y")
        if y is None:
            y = rows_b
        out = torch.empty(T, d, dtype=wl.dtype, device=dev)
        comb = lambda: moe.moe_combine(y, T, d, K, pos, w, out)
        add(wl, "moe_combine", t_us(comb), A * d * es + A * 8 + T * d * es)
        if name == "metric":
            C = moe.capacity_limit(T, K, N)
            ci, cw = torch.empty_like(idx), torch.empty_like(w)
            info = moe.empty_capacity_info(dev)
            cws = moe.capacity_workspace(T, K, N, dev)
            cap = lambda: moe.moe_route_capacity(cfg, scores, bias, C, ci, cw, info, cws)
            add(wl, "moe_route_capacity (from scores)", t_us(cap), T * N * 4 + A * 8 * 4,
                note="six launches, latency-bound")
            rb = lambda: moe.moe_route_balanced(T, K, N, wl.scale, ci, cw)
            add(wl, "moe_route_balanced", t_us(rb), A * 8)
        del inp, x, rows_b, y, out
        torch.cuda.empty_cache()

    print(f"| workload | shape | call | time (us) | bound (us) | fraction of bound | note |")
    print("|---|---|---|---|---|---|---|")
    for r in rows:
        print(f"| {r[0]} | {r[1]} | {r[2]} | {r[3]:.1f} | {r[4]:.1f} | {r[5]:.2f} | {r[6]} |")
    print(f"\nbounds: HBM {hbm} GB/s (copy), bf16 {tf_burst} TFLOP/s (burst): {peak_kind} peaks")


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_pipeline(wl, n, threads=None):
    """The oracle (as it stands) on the first n tokens of a workload: the
    stage set of the GPU pipeline -- fp64 gate, scores, selection,
    histogram/positions, stats, bias step, dispatch rows (+ the replica plan
    and the remap over the replica slots, + the FP8 copy, where the workload
    has them).  Returns (seconds, threads used)."""
    import torch
    import oracle
    from expert_load_balancing_tcgen05_b200 import workloads as W
    sw = wl.with_(T=n)
    inp = W.make_inputs(sw, seed=wl.seed)
    x = inp["x"].float().numpy()
    Wg = inp["W"].float().numpy()
    off = inp["off"].numpy() if inp["off"] is not None else None
    b = inp["bias"].numpy() if inp["bias"] is not None else None
    xb = inp["x"].view(torch.int16).numpy() if wl.dtype == torch.bfloat16 else inp["x"].numpy()
    old = oracle.num_threads()
    if threads is not None:
        oracle.set_num_threads(threads)
    used = oracle.num_threads()
    try:
        t0 = time.perf_counter()
        s = oracle.scores(oracle.logits(x, Wg, off), wl.fn)
        idx, w = oracle.select(s, b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
        slot, n_slots = idx, wl.N
        counts, offsets, pos, rk, src = oracle.positions(idx, wl.N)
        if wl.n_replicas:
            rs = oracle.replica_plan(counts, wl.n_replicas)
            slot, n_slots = oracle.apply_replicas(idx, rs), wl.n_slots
            counts, offsets, pos, rk, src = oracle.positions(slot, n_slots)
        oracle.load_stats(counts)
        if b is not None:
            oracle.bias_update(counts[:wl.N], n * wl.K, b, 0.001, 0)
        rows = oracle.dispatch_rows(xb, pos)
        if wl.fp8:
            oracle.fp8_rows(oracle.dispatch_rows(x, pos))
        del rows
        return time.perf_counter() - t0, used
    finally:
        oracle.set_num_threads(old)


def _oracle_rate(wl, seconds, threads=None):
    """tokens/s of the oracle pipeline on a sample sized for about `seconds`."""
    probe = min(wl.T, 64)
    tp, _ = _oracle_pipeline(wl, probe, threads)
    n = int(max(probe, min(wl.T, probe * seconds / max(tp, 1e-4))))
    dt, used = _oracle_pipeline(wl, n, threads)
    reps = 1
    while dt < 0.25 * seconds and n == wl.T:  # the whole workload is quick: repeat it
        reps *= 2
        dt = sum(_oracle_pipeline(wl, n, threads)[0] for _ in range(reps))
    return n * reps / dt, (f"{n} tokens" + (f" x {reps}" if reps > 1 else "")), dt, used


def run_report(oracle_seconds: float = 4.0):
    """Three markdown sections, each GPU number produced through the library's
    C ABI and checked in the same run against the oracle:
    1. the collapse workload's 100 sign-rule bias steps on fixed scores: per
       step std/mean, max/mean and load entropy from moe_stats;
    2. the prefill workload's per-slot loads and imbalance before and after
       the 32 replicas;
    3. per workload, the GPU pipeline (route, load statistics, bias step,
       dispatch) in routed tokens/s and GB/s against its roofline, beside the
       oracle on the host cores (all cores; one core for the two smallest
       workloads) on a bounded sample."""
    import numpy as np
    import torch
    import oracle
    from expert_load_balancing_tcgen05_b200 import moe
    from expert_load_balancing_tcgen05_b200 import workloads as W
    hbm, tf_burst, _, peak_kind = _peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    out = []
    P = out.append

    def route_scores(wl, inp, T=None):
        T = wl.T if T is None else T
        scores = torch.empty(T, wl.N, device=dev)
        idx = torch.empty(T, wl.K, dtype=torch.int32, device=dev)
        w = torch.empty(T, wl.K, device=dev)
        ws = moe.workspace(T, wl.K, wl.N, wl.n_slots, device=dev)
        cfg = moe.route_cfg(T, wl.d, wl.N, wl.K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm,
                            wl.scale, moe.MOE_BF16 if wl.dtype == torch.bfloat16 else moe.MOE_F32)
        moe.moe_route(cfg, inp["x"], inp["W"], inp["off"], inp["bias"], scores, idx, w, ws)
        torch.cuda.synchronize()
        assert moe.moe_workspace_status(ws) == moe.MOE_OK
        return cfg, scores, idx, w, ws

    def stats_match(st, ref):
        ok = st["status"] == 0 and st["total"] == int(ref["total"]) and st["max_load"] == int(ref["max"])
        for g in ("mean", "imbalance", "std_over_mean", "entropy_load_bits"):
            ok = ok and abs(st[g] - ref[g]) <= 1e-6 * abs(ref[g]) + 1e-12
        return ok

    # ---------------------------------------------------------------- 1. collapse
    wl = W.WORKLOADS["collapse"]
    T, N, K = wl.T, wl.N, wl.K
    inp = W.make_inputs(wl, device=dev)
    cfg, scores, idx, w, ws = route_scores(wl, inp)
    s_np = scores.cpu().numpy()
    bias = inp["bias"].clone()
    b_ref = inp["bias"].cpu().numpy().copy()
    counts = torch.empty(N, dtype=torch.int32, device=dev)
    offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
    rank = torch.empty(T, K, dtype=torch.int32, device=dev)
    stats = moe.empty_stats(dev)
    rows_c3 = []
    all_ok = True
    for step in range(wl.bias_steps + 1):
        moe.moe_route(cfg, None, None, None, bias, scores, idx, w, ws)
        moe.moe_load_stats(idx, T, K, N, None, N, None, counts, offsets, rank, None, wl.fn, stats, ws)
        if step < wl.bias_steps:
            moe.moe_bias_update(counts, N, T * K, 0.001, 0, bias)
        st = moe.read_stats(stats)
        ri, _ = oracle.select(s_np, b_ref, K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
        c_ref = oracle.histogram(ri, N)
        ok = bool(np.array_equal(counts.cpu().numpy(), c_ref)) and stats_match(st, oracle.load_stats(c_ref))
        all_ok = all_ok and ok
        celeb = int(sum(c_ref[e] for e in W.CELEBRITY_EXPERTS))
        rows_c3.append((step, st["max_load"], st["imbalance"], st["std_over_mean"], st["entropy_load_bits"], celeb, ok))
        if step < wl.bias_steps:
            b_ref = oracle.bias_update(c_ref, T * K, b_ref, 0.001, 0)
    bias_ok = bool(np.array_equal(bias.cpu().numpy(), b_ref))
    P(f"## 1. Collapse workload: 100 bias steps (T={T} d={wl.d} N={N} K={K}, sigmoid, 8 groups keep 4, "
      f"+2.0 logit offset on experts {list(W.CELEBRITY_EXPERTS)}, u = 0.001)\n")
    P("One gate pass (moe_route, tcgen05), then per step: moe_route from the fixed scores with the current bias "
      "-> moe_load_stats -> moe_bias_update (sign rule).  Row i is the routing made with the bias after i steps "
      "(row 100: the final bias).  'oracle' = the GPU counts equal the oracle's replay on the same scores and its "
      "stats agree within 1e-6.  Mean load = T*K/N = %d.  Monitoring bar of the deployment page: std <= 20%% of "
      "the mean.\n" % (T * K // N))
    P("| step | max load | max/mean | std/mean | H_load (bits) | load on the 5 celebrity experts | oracle |")
    P("|---|---|---|---|---|---|---|")
    for r in rows_c3:
        P(f"| {r[0]} | {r[1]} | {r[2]:.4f} | {r[3]:.4f} | {r[4]:.4f} | {r[5]} | {'yes' if r[6] else 'NO'} |")
    first_ok = next((r[0] for r in rows_c3 if r[3] <= 0.2), None)
    P(f"\nEvery step matches the oracle: {'yes' if all_ok else 'NO'}; final bias bit-exact: "
      f"{'yes' if bias_ok else 'NO'}.  log2 N = {np.log2(N):.4f} bits.  First step with std/mean <= 0.20: "
      f"{first_ok}.\n")
    del inp, scores, idx, w, ws, rank
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- 2. prefill replicas
    wl = W.WORKLOADS["prefill_replicas"]
    T, N, K, R = wl.T, wl.N, wl.K, wl.n_replicas
    inp = W.make_inputs(wl, device=dev)
    cfg, scores, idx, w, ws = route_scores(wl, inp)
    ri, _ = oracle.select(scores.cpu().numpy(), inp["bias"].cpu().numpy(), K, wl.n_groups, wl.topk_groups,
                          wl.group_topn, wl.renorm, wl.scale)
    sel_ok = bool(np.array_equal(idx.cpu().numpy(), ri))
    del scores
    slot = torch.empty(T, K, dtype=torch.int32, device=dev)
    rank = torch.empty(T, K, dtype=torch.int32, device=dev)
    c1 = torch.empty(N, dtype=torch.int32, device=dev)
    o1 = torch.empty(N + 1, dtype=torch.int32, device=dev)
    st1 = moe.empty_stats(dev)
    moe.moe_load_stats(idx, T, K, N, None, N, slot, c1, o1, rank, None, wl.fn, st1, ws)
    rs = torch.empty(N, dtype=torch.int32, device=dev)
    moe.moe_replica_plan(c1, N, R, rs)
    c2 = torch.empty(N + R, dtype=torch.int32, device=dev)
    o2 = torch.empty(N + R + 1, dtype=torch.int32, device=dev)
    st2 = moe.empty_stats(dev)
    moe.moe_load_stats(idx, T, K, N, rs, N + R, slot, c2, o2, rank, None, wl.fn, st2, ws)
    torch.cuda.synchronize()
    before, after = moe.read_stats(st1), moe.read_stats(st2)
    cb, ca, rsn = c1.cpu().numpy(), c2.cpu().numpy(), rs.cpu().numpy()
    cb_ref = oracle.histogram(ri, N)
    rs_ref = oracle.replica_plan(cb_ref, R)
    ca_ref, _, _, rk_ref, _ = oracle.positions(oracle.apply_replicas(ri, rs_ref), N + R)
    ok5 = (sel_ok and np.array_equal(cb, cb_ref) and np.array_equal(rsn, rs_ref) and np.array_equal(ca, ca_ref)
           and np.array_equal(rank.cpu().numpy(), rk_ref) and stats_match(before, oracle.load_stats(cb_ref))
           and stats_match(after, oracle.load_stats(ca_ref)))
    P(f"## 2. Prefill workload with redundant experts (T={T} d={wl.d} N={N} K={K}, Zipf(1.1) logit offsets "
      f"-1.1*ln(e+1), {R} replicas -> {N + R} slots)\n")
    P("moe_route (tcgen05 gate, selection in the epilogue) -> moe_load_stats over the 256 experts -> "
      "moe_replica_plan (32 hottest by count, ties to the lower index) -> moe_load_stats over the 288 slots (odd "
      "tokens of a replicated expert go to its replica).  Before replication the 32 replica slots are empty and "
      "max/mean is taken over the 256 experts (mean T*K/256); after, over the 288 slots (mean T*K/288).\n")
    P("| | slots | max load | mean | max/mean | std/mean | H_load (bits) |")
    P("|---|---|---|---|---|---|---|")
    for name, st in (("before", before), ("after", after)):
        P(f"| {name} | {st['n_slots']} | {st['max_load']} | {st['mean']:.2f} | {st['imbalance']:.4f} | "
          f"{st['std_over_mean']:.4f} | {st['entropy_load_bits']:.4f} |")
    P(f"\nGPU selection, histograms, replica plan, slot counts, ranks and stats equal the oracle's (on the GPU's "
      f"scores): {'yes' if ok5 else 'NO'}.\n")
    P("Per-slot loads (slot: before -> after; slots 256.. are the replicas, with the expert they copy):\n")
    P("| slot | expert | before | after |")
    P("|---|---|---|---|")
    owner = {int(rsn[e]): e for e in range(N) if rsn[e] >= 0}
    for sl in range(N + R):
        e = sl if sl < N else owner.get(sl, -1)
        P(f"| {sl} | {e} | {int(cb[sl]) if sl < N else 0} | {int(ca[sl])} |")
    P("")
    del inp, idx, w, ws, slot, rank
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- 3. per workload, GPU beside the oracle
    def t_us(fn, n=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / n * 1e3

    P("## 3. Routed tokens/s per workload: the GPU pipeline beside the oracle\n")
    P(f"GPU: route (gate + selection; '(fused)': selection and tile histograms in the gate's epilogue, "
      f"moe_route_tiles + moe_load_stats_tiles) -> load statistics (+ replica plan and the slot remap for the "
      f"prefill workload) -> bias step (workloads with a bias) -> dispatch (+ FP8 copy for the softmax-dispatch "
      f"workload), one stream, 10 pipelines captured in a CUDA graph and replayed under CUDA events.  Roofline = "
      f"sum over the stages of max(bytes / {hbm:.1f} GB/s, gate flops / {tf_burst:.1f} TFLOP/s) ({peak_kind} "
      f"peaks).  Oracle: the same stage set in plain C (fp64), on a bounded sample of each workload's tokens, on "
      f"the host: CPU '{_cpu_model()}', {os.cpu_count()} logical CPUs.\n")
    P("| workload | shape | GPU us/batch | GPU routed tokens/s | GPU GB/s (algorithmic) | fraction of roofline | "
      "oracle tokens/s (threads) | oracle sample | oracle 1 thread tokens/s | GPU / oracle |")
    P("|---|---|---|---|---|---|---|---|---|---|")
    for name in ("tiny_softmax", "v3_router", "collapse", "softmax_dispatch", "prefill_replicas", "metric"):
        wl = W.WORKLOADS[name]
        T, d, N, K = wl.T, wl.d, wl.N, wl.K
        A = T * K
        es = 2 if wl.dtype == torch.bfloat16 else 4
        inp = W.make_inputs(wl, device=dev, seed=wl.seed)
        x, Wg, off, bias = inp["x"], inp["W"], inp["off"], inp["bias"]
        scores = torch.empty(T, N, device=dev)
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        w = torch.empty(T, K, device=dev)
        ws = moe.workspace(T, K, N, wl.n_slots, device=dev)
        cfg = moe.route_cfg(T, d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale,
                            moe.MOE_BF16 if wl.dtype == torch.bfloat16 else moe.MOE_F32)
        slot = torch.empty(T, K, dtype=torch.int32, device=dev)
        rank = torch.empty(T, K, dtype=torch.int32, device=dev)
        counts = torch.empty(wl.n_slots, dtype=torch.int32, device=dev)
        offsets = torch.empty(wl.n_slots + 1, dtype=torch.int32, device=dev)
        stats = moe.empty_stats(dev)
        rs = torch.empty(N, dtype=torch.int32, device=dev) if wl.n_replicas else None
        b2 = bias.clone() if bias is not None else None
        rows = torch.empty(A, d, dtype=wl.dtype, device=dev)
        q = torch.empty(A, d, dtype=torch.uint8, device=dev) if wl.fp8 else None
        sc = torch.empty(A, d // 128, device=dev) if wl.fp8 else None
        pos = torch.empty(T, K, dtype=torch.int32, device=dev)

        from expert_load_balancing_tcgen05_b200.step import fused_routing_supported
        fused = fused_routing_supported(wl, x)
        tiles = torch.empty(moe.tile_counts_shape(T, N), dtype=torch.int32, device=dev) if fused else None

        def stats_call(rep, ns, cnt, offs):
            if fused:
                moe.moe_load_stats_tiles(idx, T, K, N, tiles, rep, ns, slot, cnt, offs, rank, stats, ws)
            else:
                moe.moe_load_stats(idx, T, K, N, rep, ns, slot, cnt, offs, rank, None, wl.fn, stats, ws)

        def pipeline():
            if fused:
                moe.moe_route_tiles(cfg, x, Wg, off, b2, idx, w, tiles, ws)
            else:
                moe.moe_route(cfg, x, Wg, off, b2, scores, idx, w, ws)
            if rs is not None:
                stats_call(None, N, counts[:N], offsets[:N + 1])
                moe.moe_replica_plan(counts[:N], N, wl.n_replicas, rs)
            stats_call(rs, wl.n_slots, counts, offsets)
            if b2 is not None:
                moe.moe_bias_update(counts[:N], N, A, 0.001, 0, b2)
            moe.moe_dispatch(x, T, d, K, slot, offsets, rank, rows, q, sc, pos, None)

        us = t_us(pipeline)
        # route bytes: the fused path never writes or re-reads the scores
        route_b = (T * d * es + N * d * es + A * 8 + tiles.numel() * 4) if fused else \
            (T * d * es + N * d * es + T * N * 4 + A * 8) + (T * N * 4 + A * 8)
        nbytes = route_b + A * 12 + (T * d * es + A * d * es + A * 12) + ((A * d + A * d // 32) if wl.fp8 else 0)
        # serial roofline: the gate at the slower of its HBM and tensor bounds, the rest at HBM speed
        gate_b = T * d * es + N * d * es + (A * 8 if fused else T * N * 4)
        roof = (max(gate_b / (hbm * 1e9), 2 * T * d * N / (tf_burst * 1e12)) + (nbytes - gate_b) / (hbm * 1e9)) * 1e6
        gpu_tps = T / (us / 1e6)
        del inp, x, Wg, scores, idx, w, ws, slot, rank, rows, q, sc, pos, tiles
        torch.cuda.empty_cache()
        o_tps, n, dt, used = _oracle_rate(wl, oracle_seconds)
        one = ""
        if name in ("tiny_softmax", "v3_router"):
            o1, n1, dt1, _ = _oracle_rate(wl, oracle_seconds, threads=1)
            one = f"{o1:,.0f} ({n1}, {dt1:.1f} s)"
        P(f"| {name}{' (fused)' if fused else ''} | T={T} d={d} N={N} K={K} | {us:.1f} | {gpu_tps:,.0f} | "
          f"{nbytes / (us / 1e6) / 1e9:,.0f} | "
          f"{roof / us:.2f} | {o_tps:,.0f} ({used}) | {n}, {dt:.1f} s | {one or '-'} | "
          f"{gpu_tps / o_tps:,.0f} |")
    P("")
    print("\n".join(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernels", action="store_true",
                    help="print per-call device times of every workload against their bounds (markdown)")
    ap.add_argument("--only", default=None,
                    help="with --kernels: report one workload only (tiny_softmax, v3_router, collapse, "
                         "softmax_dispatch, prefill_replicas, metric)")
    ap.add_argument("--report", action="store_true",
                    help="print the bias-balancing trajectory, the replica loads and per-workload GPU vs oracle "
                         "throughput (markdown)")
    ap.add_argument("--gate-ctas", type=int, default=None,
                    help="SM budget of the gate in the pipelined schedule (default: the step's own)")
    ap.add_argument("--timed-only", action="store_true",
                    help="print only the timed region's numbers (for sweeps; not the benchmark's full line)")
    ap.add_argument("--unfused", action="store_true",
                    help="route through the gate's scores epilogue and the selection kernel instead of the fused "
                         "path (selection and tile histograms in the gate's epilogue, the default)")
    ap.add_argument("--serial", action="store_true",
                    help="time the serial schedule (one call after another) instead of the pipelined one")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.kernels:
        run_kernel_report(args.only)
        return
    if args.report:
        run_report()
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline and not args.timed_only:
                out["cpu_baseline"] = cpu_baseline()
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
