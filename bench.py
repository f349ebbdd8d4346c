#!/usr/bin/env python
"""Benchmark of the Swimba layer forward pass (route -> mixed projection -> scan) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {swimba,reference}] [--workload NAME]

One step is one pass of the whole layer over one batch of the workload (default: the Mamba-1.4B-
like shape, B=8, L=4096, D=4096, N=16, R=128, E=8, top-2; its inputs are larger than the 126 MB
L2, so no flush is needed between steps). The reported value is tokens/s of the whole layer,
device-timed with CUDA events on the launching stream over exactly K steps (W untimed warm-up
steps before), the max over ranks. With N > 1 every rank runs its own copy of the workload (the
sequences are independent: weak scaling, no collective on the data path).

Also printed on the same JSON line: per-kernel times, the roofline of the dominant kernel, the
switch overhead against the E=1 dense layer of the same shape, an end-to-end figure through the
C ABI with host buffers (host<->device copies inside the timed region), the kernel-launch count,
SM clocks sampled during the timed region and a CPU baseline (the fp64 oracle on a bounded
sample, rank 0 only). ``--impl reference`` times that oracle alone as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from parameter_space_moe_swimba_b200 import synth  # noqa: E402
from parameter_space_moe_swimba_b200.configs import CONFIGS, dense_variant  # noqa: E402

METRIC = "Swimba scan tokens/s at 1 B200; % of HBM roofline; switch vs E=1 overhead"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="swimba", choices=["swimba", "reference"])
    ap.add_argument("--workload", default="mamba1p4b_like")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "sm_max_mhz": d.get("sm_max_mhz", 1965.0),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


# ------------------------------------------------------------------------------------------------
# algorithmic bytes per token (only the k active experts count)
# ------------------------------------------------------------------------------------------------

def io_bytes(cfg):
    return 2 if cfg.io_dtype == "bf16" else 4


def scan_bytes_per_token(cfg):
    """x, z read and out written (io), delta read (fp32), B_mix and C_mix read, idx and gates read."""
    D, N, k = cfg.d_inner, cfg.d_state, cfg.top_k
    return 3 * io_bytes(cfg) * D + 4 * D + 8 * N + 8 * k


def route_bytes_per_token(cfg):
    return io_bytes(cfg) * cfg.d_inner + 8 * cfg.top_k


def proj_bytes_per_token(cfg):
    """x read, delta written (fp32), B_mix and C_mix written, idx and gates read."""
    D, N, k = cfg.d_inner, cfg.d_state, cfg.top_k
    return io_bytes(cfg) * D + 4 * D + 8 * N + 8 * k


def proj_flops_per_token(cfg):
    D, N, R, k = cfg.d_inner, cfg.d_state, cfg.dt_rank, cfg.top_k
    return 2 * k * D * (R + 2 * N) + 2 * k * R * D


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        """Start sampling every 50 ms and wait (at most 3 s) until the first sample is written."""
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while self.mark() == 0 and time.time() - t0 < 3.0:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def _rows(self):
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and line.endswith("\n"):
                    rows.append(parts)
        return rows

    def mark(self):
        """Number of complete samples so far (brackets the timed region)."""
        if self.proc is None:
            return 0
        return len(self._rows())

    def stop(self, begin=0, end=None):
        """Summarise the samples taken between the marks ``begin`` and ``end`` (all if none fall there)."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = self._rows()
        os.unlink(self.path)
        inside = rows[begin:end]
        rows = inside if inside else rows
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------------------
# the CUDA path
# ------------------------------------------------------------------------------------------------

class GpuLayer:
    def __init__(self, S, cfg, x_host, z_host, device):
        import torch

        self.S, self.cfg, self.torch = S, cfg, torch
        self.dims = S.make_dims(cfg)
        self.w = S.upload_weights(synth.draw_weights(cfg), device)
        self.ws_struct = self.w.struct()
        self.x = S.to_device(x_host, cfg.io_dtype, device)
        self.z = S.to_device(z_host, cfg.io_dtype, device)
        io_t = torch.bfloat16 if cfg.io_dtype == "bf16" else torch.float32
        self.buf = S.LayerBuffers(self.dims, io_t, device)
        self.stream = torch.cuda.current_stream()

    def step(self, ev=None):
        S, d, b, w = self.S, self.dims, self.buf, self.ws_struct
        s = self.stream
        if ev is not None:
            ev[0].record(s)
        S.check(S.swimba_route(d, self.x, w.W_r, b.idx, b.gates, s), "route")
        if ev is not None:
            ev[1].record(s)
        S.check(S.swimba_mixed_proj(d, self.x, b.idx, b.gates, w, b.delta, b.B_mix, b.C_mix, b.ws, b.ws.numel(), s),
                "proj")
        if ev is not None:
            ev[2].record(s)
        S.check(S.swimba_scan_fwd(d, self.x, self.z, b.delta, b.B_mix, b.C_mix, b.idx, b.gates, w, None, b.out,
                                  b.h_final, None, b.ws, b.ws.numel(), s), "scan")
        if ev is not None:
            ev[3].record(s)


def max_over_ranks(value: float, dist, device) -> float:
    """The max of a per-rank number over all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Units all ranks processed, divided by the slowest rank's time (weak scaling)."""
    return units_per_rank_step * steps * world / (max_ms / 1e3)


def timed_steps(torch, layer, steps, warmup, dist=None):
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    launches0 = layer.S.swimba_kernel_launches()
    t0.record(layer.stream)
    for i in range(steps):
        layer.step(evs[i])
    t1.record(layer.stream)
    torch.cuda.synchronize()
    launches = layer.S.swimba_kernel_launches() - launches0
    if dist is not None:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    per = {"route": [], "proj": [], "scan": []}
    for e in evs:
        per["route"].append(e[0].elapsed_time(e[1]))
        per["proj"].append(e[1].elapsed_time(e[2]))
        per["scan"].append(e[2].elapsed_time(e[3]))
    return total_ms, {k: float(np.mean(v)) for k, v in per.items()}, launches


def e2e_steps(torch, S, layer, steps, warmup, x_host, z_host):
    """Host buffers in, host result out: H2D of x and z from pinned memory, the three library calls,
    D2H of out into pinned memory, every step, device-timed on the stream."""
    cfg = layer.cfg
    xh = S.to_device(x_host, cfg.io_dtype, "cpu", pin=True)
    zh = S.to_device(z_host, cfg.io_dtype, "cpu", pin=True)
    oh = torch.empty(layer.buf.out.shape, dtype=layer.buf.out.dtype, pin_memory=True)
    s = layer.stream

    def one():
        layer.x.copy_(xh, non_blocking=True)
        layer.z.copy_(zh, non_blocking=True)
        layer.step()
        oh.copy_(layer.buf.out, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for _ in range(steps):
        one()
    t1.record(s)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    h2d = xh.numel() * xh.element_size() + zh.numel() * zh.element_size()
    d2h = oh.numel() * oh.element_size()
    return ms, h2d, d2h


# ------------------------------------------------------------------------------------------------
# the fp64 oracle on the host (CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------------------

def oracle_sample(cfg, tokens):
    """One batch row, the first ``tokens`` tokens, every channel: the oracle's whole layer on it."""
    from oracle import swimba_oracle as O

    w = synth.draw_weights(cfg)
    x, z = synth.draw_activations(cfg.with_(seqlen=tokens), batch_rows=[0])
    W = {"W_r": w.W_r.astype(np.float64), "W_x": synth.widen(w.W_x, cfg.w_dtype),
         "W_dt": synth.widen(w.W_dt, cfg.w_dtype), "b_dt": w.b_dt.astype(np.float64), "A": w.A.astype(np.float64),
         "D_skip": w.D_skip.astype(np.float64)}
    x64, z64 = synth.widen(x, cfg.io_dtype), synth.widen(z, cfg.io_dtype)

    def run():
        O.layer_forward(x64, z64, W, cfg.top_k)

    return run


def time_oracle(cfg, tokens, reps=1):
    from threadpoolctl import threadpool_limits

    run = oracle_sample(cfg, tokens)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for _ in range(reps):
            run()
        dt = time.perf_counter() - t0
    return dt / reps


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    tokens = 256
    run = oracle_sample(cfg, tokens)
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):
        for _ in range(args.warmup):
            run()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            run()
        dt = time.perf_counter() - t0
    value = tokens * args.steps / dt
    sample = f"batch row 0, first {tokens} of {cfg.seqlen} tokens, all {cfg.d_inner} channels"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_block(cfg):
    return {"workload": cfg.name, "batch": cfg.batch, "seqlen": cfg.seqlen, "d_inner": cfg.d_inner,
            "d_state": cfg.d_state, "dt_rank": cfg.dt_rank, "n_experts": cfg.n_experts, "top_k": cfg.top_k,
            "io_dtype": cfg.io_dtype, "w_dtype": cfg.w_dtype,
            "l2": "inputs larger than the 126 MB L2 (x, z 268 MB each), no flush between steps"}


# ------------------------------------------------------------------------------------------------

def main():
    args = parse()
    cfg = CONFIGS[args.workload]
    if args.batch > 0:
        cfg = cfg.with_(batch=args.batch)
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = f"cuda:{local}"
    torch.cuda.set_device(local)

    from parameter_space_moe_swimba_b200 import swimba as S

    peaks = load_peaks()
    x_host, z_host = synth.draw_activations(cfg)
    layer = GpuLayer(S, cfg, x_host, z_host, device)

    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    m0 = clocks.mark()
    total_ms, per_kernel, launches = timed_steps(torch, layer, args.steps, args.warmup, dist)
    clk = clocks.stop(m0, clocks.mark())
    S.check(S.swimba_get_device_status(layer.buf.ws, layer.stream), "device status")

    max_ms = max_over_ranks(total_ms, dist, device)
    value = whole_job_rate(cfg.tokens, args.steps, world, max_ms)

    # switch overhead against the E=1 dense layer of the same shape (same inputs)
    dense = None
    if not args.no_dense:
        dcfg = dense_variant(cfg)
        dl = GpuLayer(S, dcfg, x_host, z_host, device)
        d_ms, d_per, _ = timed_steps(torch, dl, args.steps, args.warmup, None)
        dense = {"layer_ms": d_ms / args.steps, "scan_ms": d_per["scan"], "proj_ms": d_per["proj"],
                 "layer_overhead": (total_ms / args.steps) / (d_ms / args.steps) - 1.0,
                 "scan_overhead": per_kernel["scan"] / d_per["scan"] - 1.0}
        del dl

    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h = e2e_steps(torch, S, layer, args.steps, args.warmup, x_host, z_host)
        e2e = {"value": whole_job_rate(cfg.tokens, args.steps, world, max_over_ranks(e_ms, dist, device)), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    scan_bytes = scan_bytes_per_token(cfg) * cfg.tokens + 4 * cfg.batch * cfg.d_inner * cfg.d_state
    achieved = scan_bytes / (per_kernel["scan"] / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel": "scan_fwd",
                "algorithmic_bytes_per_launch": scan_bytes, "peak_source": peaks["source"]}
    kernels = {
        "route_us": 1e3 * per_kernel["route"], "proj_us": 1e3 * per_kernel["proj"], "scan_us": 1e3 * per_kernel["scan"],
        "route_gbs": route_bytes_per_token(cfg) * cfg.tokens / (per_kernel["route"] / 1e3) / 1e9,
        "proj_gbs": proj_bytes_per_token(cfg) * cfg.tokens / (per_kernel["proj"] / 1e3) / 1e9,
        "proj_tflops": proj_flops_per_token(cfg) * cfg.tokens / (per_kernel["proj"] / 1e3) / 1e12,
        "scan_gbs": achieved,
        "scan_exps_per_s": cfg.tokens * cfg.d_inner * cfg.d_state / (per_kernel["scan"] / 1e3),
    }

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok = 1024
        dt = time_oracle(cfg, tok)
        cpu = {"value": tok / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"batch row 0, first {tok} of {cfg.seqlen} tokens, all {cfg.d_inner} channels "
                         f"(fp64 numpy, 1 thread)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config_block(cfg),
            "roofline": roofline, "kernels": kernels, "switch_vs_dense_e1": dense, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk, "cpu_baseline": cpu,
            "compute": "bf16 x/W on tensor cores with fp32 accumulation; fp32 state and scan arithmetic",
        }
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
