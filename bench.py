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
    ap.add_argument("--seqlen", type=int, default=0, help="override the workload's sequence length (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--report", action="store_true",
                    help="per-workload table (one JSON line each): every workload, decode steps, E sweep")
    ap.add_argument("--report-ssd", action="store_true", help="only the SSD-form line")
    ap.add_argument("--report-decode", action="store_true",
                    help="only the decode line (--steps decode steps of the decode workload)")
    ap.add_argument("--report-separate", action="store_true",
                    help="only the separate-SSM comparison line (Teorema 2)")
    ap.add_argument("--report-bwd", action="store_true",
                    help="only the backward-pass line (scan, mixed projection and router gradients)")
    ap.add_argument("--report-block", action="store_true",
                    help="only the surrounding block's report lines (with --batch: the prefill line at that batch)")
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

def measured_traffic(cfg):
    """DRAM bytes per scan launch (dram__bytes_read.sum + dram__bytes_write.sum) from the committed
    ncu figure in profiles/scan_traffic.json, scaled to this workload's tokens when the capture was
    taken on a shorter sequence of the same shape (the scan's traffic grows with the tokens); None
    when the figure is for another shape or the scan kernel's source has changed since."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "scan_traffic.json")
    src = os.path.join(ROOT, "parameter_space_moe_swimba_b200", "csrc", "scan_fast.cu")
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256") != digest:
        return None
    shape = {k: getattr(cfg, k) for k in ("batch", "d_inner", "d_state", "n_experts", "top_k", "io_dtype")}
    if rec.get("shape") != shape:
        return None
    return int(rec["dram_bytes_per_launch"] * cfg.seqlen / rec["seqlen"])


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
    """Host buffers in, host result out, every step: H2D of x and z from pinned memory, the three
    library calls, D2H of out into pinned memory. A serving loop's pipeline: two device slots of
    x, z and layer buffers; step i's copies-in run on their own stream while step i-1 computes, and
    step i-1's D2H on a third stream while step i computes, so the two copy directions overlap each
    other and the kernels (the link is full duplex). Device-timed from the first copy's start to
    the last copy's end."""
    cfg = layer.cfg
    xh = S.to_device(x_host, cfg.io_dtype, "cpu", pin=True)
    zh = S.to_device(z_host, cfg.io_dtype, "cpu", pin=True)
    oh = torch.empty(layer.buf.out.shape, dtype=layer.buf.out.dtype, pin_memory=True)
    dev = layer.x.device
    io_t = layer.buf.out.dtype
    slots = [(layer.x, layer.z, layer.buf),
             (torch.empty_like(layer.x), torch.empty_like(layer.z), S.LayerBuffers(layer.dims, io_t, dev))]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_c = layer.stream
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_c = [torch.cuda.Event(), torch.cuda.Event()]
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]
    d, w = layer.dims, layer.ws_struct

    def step(i):
        k = i % 2
        x, z, b = slots[k]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_c[k])  # step i-2 has finished reading this slot's x and z
            x.copy_(xh, non_blocking=True)
            z.copy_(zh, non_blocking=True)
            ev_in[k].record(s_in)
        s_c.wait_event(ev_in[k])
        if i >= 2:
            s_c.wait_event(ev_out[k])  # step i-2's output has left this slot
        S.check(S.swimba_route(d, x, w.W_r, b.idx, b.gates, s_c), "route")
        S.check(S.swimba_mixed_proj(d, x, b.idx, b.gates, w, b.delta, b.B_mix, b.C_mix, b.ws, b.ws.numel(), s_c),
                "proj")
        S.check(S.swimba_scan_fwd(d, x, z, b.delta, b.B_mix, b.C_mix, b.idx, b.gates, w, None, b.out, b.h_final, None,
                                  b.ws, b.ws.numel(), s_c), "scan")
        ev_c[k].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[k])
            oh.copy_(b.out, non_blocking=True)
            ev_out[k].record(s_out)

    def run(n):
        for i in range(n):
            step(i)
        s_c.wait_stream(s_out)
        s_c.wait_stream(s_in)

    run(max(warmup, 2))
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    s_in.wait_stream(s_c)
    t0.record(s_in)
    run(steps)
    t1.record(s_c)
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
    W = _weights64(cfg, w)
    x64, z64 = synth.widen(x, cfg.io_dtype), synth.widen(z, cfg.io_dtype)

    def run():
        O.layer_forward(x64, z64, W, cfg.top_k)

    return run


def _weights64(cfg, w):
    return {"W_r": w.W_r.astype(np.float64), "W_x": synth.widen(w.W_x, cfg.w_dtype),
            "W_dt": synth.widen(w.W_dt, cfg.w_dtype), "b_dt": w.b_dt.astype(np.float64), "A": w.A.astype(np.float64),
            "D_skip": w.D_skip.astype(np.float64)}


# Worker side of the parallel oracle: each process draws the weights once, then runs the oracle's
# layer on one batch row and one block of channels per task (the recurrence of every (row,
# channel) is independent; the routing and projections of the row are computed by every task, as
# the oracle does them).
_ORACLE = {}


def _oracle_init(cfg, tokens):
    from threadpoolctl import threadpool_limits

    _ORACLE["limits"] = threadpool_limits(limits=1)
    _ORACLE["cfg"] = cfg.with_(seqlen=tokens)
    _ORACLE["W"] = _weights64(cfg, synth.draw_weights(cfg))
    _ORACLE["rows"] = {}


def _oracle_task(task):
    from oracle import swimba_oracle as O

    b, lo, hi = task
    cfg = _ORACLE["cfg"]
    rows = _ORACLE["rows"]
    if b not in rows:
        x, z = synth.draw_activations(cfg, batch_rows=[b])
        rows[b] = (synth.widen(x, cfg.io_dtype), synth.widen(z, cfg.io_dtype))
    x64, z64 = rows[b]
    t0 = time.perf_counter()
    O.layer_forward(x64, z64, _ORACLE["W"], cfg.top_k, channels=np.arange(lo, hi))
    return time.perf_counter() - t0


class OraclePool:
    """The fp64 oracle on every host core: a process pool (started with spawn, so it is safe to
    create after CUDA is initialised) over (batch row, channel block) tasks of one workload."""

    def __init__(self, cfg, tokens, rows):
        import multiprocessing as mp

        self.cfg, self.tokens, self.rows = cfg, tokens, rows
        # every worker holds the fp64 weights and one row's projections (a few hundred MB on the
        # bench workload), so the pool stops at 128 processes on hosts with more cores
        self.cores = min(os.cpu_count() or 1, 128)
        blocks = max(1, min(cfg.d_inner // 64, -(-self.cores // len(rows))))
        edges = [round(i * cfg.d_inner / blocks) for i in range(blocks + 1)]
        self.tasks = [(b, edges[i], edges[i + 1]) for b in rows for i in range(blocks)]
        self.procs = min(self.cores, len(self.tasks))
        self.pool = mp.get_context("spawn").Pool(self.procs, initializer=_oracle_init, initargs=(cfg, tokens))
        self.pool.map(_oracle_task, self.tasks)  # warm-up: every worker has drawn the rows it serves

    def run(self):
        """Wall seconds of one pass over every task (all rows, all channels)."""
        t0 = time.perf_counter()
        self.pool.map(_oracle_task, self.tasks)
        return time.perf_counter() - t0

    def sample(self):
        return (f"batch rows {self.rows[0]}..{self.rows[-1]}, first {self.tokens} of {self.cfg.seqlen} tokens, all "
                f"{self.cfg.d_inner} channels; fp64 numpy oracle, {len(self.tasks)} (row, channel block) tasks on "
                f"{self.procs} processes")

    def close(self):
        self.pool.terminate()
        self.pool.join()


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    tokens = 256
    pool = OraclePool(cfg, tokens, list(range(cfg.batch)))
    try:
        for _ in range(args.warmup):
            pool.run()
        dt = sum(pool.run() for _ in range(args.steps))
    finally:
        pool.close()
    value = tokens * cfg.batch * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.procs, "kind": "oracle",
                         "sample": pool.sample()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_block(cfg, world=1):
    return {"workload": cfg.name, "batch": cfg.batch, "global_batch": cfg.batch * world, "seqlen": cfg.seqlen,
            "d_inner": cfg.d_inner, "d_state": cfg.d_state, "dt_rank": cfg.dt_rank, "n_experts": cfg.n_experts,
            "top_k": cfg.top_k, "io_dtype": cfg.io_dtype, "w_dtype": cfg.w_dtype,
            "parallelism": f"dp{world}: the global batch of {cfg.batch * world} sequences sharded {cfg.batch} per "
                           "rank, no data-path collective",
            "l2": "inputs larger than the 126 MB L2 (x, z 268 MB each), no flush between steps"}


# ------------------------------------------------------------------------------------------------
# --report: every workload, the decode step and the E sweep (one JSON line each)
# ------------------------------------------------------------------------------------------------

class L2Flush:
    """Writes a buffer larger than the 126 MB L2 between timed runs (outside the timed events), then
    reads it back: the write evicts every line the timed kernels could reuse, the read makes the
    write-back of the buffer's own dirty lines happen here rather than inside the timed region, so
    the timed kernels start on an L2 of clean, unrelated lines."""

    def __init__(self, torch, device):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def __call__(self):
        self.buf.zero_()
        self.buf.max()


# A GPU-side pause after the L2 flush, so that the host has queued the whole timed sequence before
# the GPU reaches its first event: the events then time the kernels, not the host's launch calls.
HOST_LEAD_CYCLES = 400_000  # about 0.2 ms at 1.9-2.0 GHz


def _median_kernel_ms(torch, run, reps, warmup, flush, nev):
    for _ in range(warmup):
        flush()
        run(None)
    torch.cuda.synchronize()
    per = []
    for _ in range(reps):
        flush()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
        run(ev)
        torch.cuda.synchronize()
        per.append([ev[i].elapsed_time(ev[i + 1]) for i in range(nev - 1)])
    cols = list(zip(*per))
    return [statistics.median(c) for c in cols], statistics.median([sum(r) for r in per])


def report_workload(torch, S, cfg, peaks, flush, reps, warmup):
    x, z = synth.draw_activations(cfg)
    layer = GpuLayer(S, cfg, x, z, "cuda:0")
    (r_ms, p_ms, s_ms), tot = _median_kernel_ms(torch, layer.step, reps, warmup, flush, 4)
    T = cfg.tokens
    scan_bytes = scan_bytes_per_token(cfg) * T + 4 * cfg.batch * cfg.d_inner * cfg.d_state
    pf = proj_flops_per_token(cfg) * T
    pb = proj_bytes_per_token(cfg) * T
    tc_peak = peaks["bf16_tflops"] * 1e12
    proj_bound_s = max(pf / tc_peak, pb / (peaks["hbm_gbs"] * 1e9))
    exps = T * cfg.d_inner * cfg.d_state
    mufu_peak = 16 * 148 * peaks["sm_max_mhz"] * 1e6
    S.check(S.swimba_get_device_status(layer.buf.ws, layer.stream), "device status")
    return {
        "report": "workload", "workload": cfg.name, "tokens": T, "layer_us": 1e3 * tot,
        "tokens_per_s": T / (tot / 1e3),
        "route_us": 1e3 * r_ms, "route_gbs": route_bytes_per_token(cfg) * T / (r_ms / 1e3) / 1e9,
        "proj_us": 1e3 * p_ms, "proj_gbs": pb / (p_ms / 1e3) / 1e9, "proj_tflops": pf / (p_ms / 1e3) / 1e12,
        "proj_frac_of_tc_peak": pf / (p_ms / 1e3) / tc_peak,
        "proj_frac_of_min_tc_bw": proj_bound_s / (p_ms / 1e3),
        "scan_us": 1e3 * s_ms, "scan_gbs": scan_bytes / (s_ms / 1e3) / 1e9,
        "scan_frac_of_hbm": scan_bytes / (s_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "scan_frac_of_mufu": exps / (s_ms / 1e3) / mufu_peak,
        "median_of": reps, "l2": "flushed (256 MB written, then read) before every run",
    }


def report_bwd(torch, S, cfg, peaks, flush, reps, warmup):
    """The layer's backward pass on one workload: swimba_scan_bwd, swimba_proj_bwd (dx accumulated)
    and swimba_route_bwd (both gate-gradient parts, dx accumulated), after one forward call whose
    outputs (idx, gates, Δ, B_mix, C_mix) they read. CUDA events around each call, L2 flushed
    before every run; swimba_proj_bwd reads its per-expert sizes back to the host once, and the
    host's turn-around inside it is part of its time."""
    x, z = synth.draw_activations(cfg)
    layer = GpuLayer(S, cfg, x, z, "cuda:0")
    layer.step(None)
    dims, ws_w, buf = layer.dims, layer.ws_struct, layer.buf
    B, L, D, N, R, E, k = cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.dt_rank, cfg.n_experts, cfg.top_k
    T = B * L
    go = S.to_device(synth.draw_out_grad(cfg), cfg.io_dtype, "cuda:0")
    f = dict(dtype=torch.float32, device="cuda:0")
    dx, dz, ddelta = (torch.empty((B, L, D), **f) for _ in range(3))
    dB, dC = torch.empty((B, L, N), **f), torch.empty((B, L, N), **f)
    dg1, dg2 = torch.empty((B, L, k), **f), torch.empty((B, L, k), **f)
    dA, dD = torch.empty((E, D, N), **f), torch.empty((D,), **f)
    dWx, dWdt, db = torch.empty((E, D, R + 2 * N), **f), torch.empty((E, R, D), **f), torch.empty((E, D), **f)
    dWr = torch.empty((D, E), **f)
    ws1 = S.new_workspace(dims, S.SWIMBA_OP_SCAN_BWD, "cuda:0")
    ws2 = S.new_workspace(dims, S.SWIMBA_OP_PROJ_BWD, "cuda:0")
    ws3 = S.new_workspace(dims, S.SWIMBA_OP_ROUTE_BWD, "cuda:0")
    s = torch.cuda.current_stream()

    def run(ev):
        rec = (lambda i: ev[i].record(s)) if ev is not None else (lambda i: None)
        rec(0)
        S.check(S.swimba_scan_bwd(dims, layer.x, layer.z, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, ws_w,
                                  None, go, dx, dz, ddelta, dB, dC, dg1, dA, dD, None, ws1, ws1.numel(), s), "scan_bwd")
        rec(1)
        S.check(S.swimba_proj_bwd(dims, layer.x, buf.idx, buf.gates, ws_w, buf.delta, ddelta, dB, dC, dx, 1, dg2, dWx,
                                  dWdt, db, ws2, ws2.numel(), s), "proj_bwd")
        rec(2)
        S.check(S.swimba_route_bwd(dims, layer.x, ws_w.W_r, buf.idx, buf.gates, dg1, dg2, dx, 1, dWr, ws3, ws3.numel(),
                                   s), "route_bwd")
        rec(3)

    (s_ms, p_ms, r_ms), tot = _median_kernel_ms(torch, run, reps, warmup, flush, 4)
    for wsb in (ws1, ws2):
        S.check(S.swimba_get_device_status(wsb, s), "device status")
    P = T * k
    W = R + 2 * N
    proj_flops = 2 * P * (D * W + D * R + W * D + D * W + (R + 8) * D)
    # one exp2 per state element in each of: the checkpoint pass, the forward through each chunk, the
    # sub-block recompute and the adjoint
    exps = 4 * T * D * N
    mufu_peak = 16 * 148 * peaks["sm_max_mhz"] * 1e6
    return {
        "report": "backward", "workload": cfg.name, "tokens": T, "layer_bwd_us": 1e3 * tot,
        "tokens_per_s": T / (tot / 1e3),
        "scan_bwd_us": 1e3 * s_ms, "scan_bwd_exps_per_s": exps / (s_ms / 1e3),
        "scan_bwd_frac_of_mufu": exps / (s_ms / 1e3) / mufu_peak,
        "proj_bwd_us": 1e3 * p_ms, "proj_bwd_tflops": proj_flops / (p_ms / 1e3) / 1e12,
        "proj_bwd_frac_of_tc_peak": proj_flops / (p_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
        "route_bwd_us": 1e3 * r_ms, "median_of": reps, "l2": "flushed (256 MB written, then read) before every run",
        "peak_source": peaks["source"],
    }


def report_separate(torch, S, cfg, peaks, flush, reps, warmup):
    """Teorema 2 measured: the MoE of separate SSMs (one state trajectory per expert, the k active
    experts' states advanced per token) against Swimba's single mixed recurrence, on the same
    tokens and routing. Only the two scans are timed; the separate design's per-slot streams are
    made once beforehand by swimba_separate_proj."""
    x, z = synth.draw_activations(cfg)
    layer = GpuLayer(S, cfg, x, z, "cuda:0")
    layer.step()
    d, b, w = layer.dims, layer.buf, layer.ws_struct
    B, L, D, N, k, E = cfg.batch, cfg.seqlen, cfg.d_inner, cfg.d_state, cfg.top_k, cfg.n_experts
    f32 = dict(dtype=torch.float32, device="cuda:0")
    dj = torch.empty((B, L, k, D), **f32)
    bj = torch.empty((B, L, k, N), **f32)
    cj = torch.empty((B, L, k, N), **f32)
    S.check(S.swimba_separate_proj(d, layer.x, b.idx, b.gates, w, dj, bj, cj, layer.stream), "separate_proj")
    out = torch.empty_like(b.out)
    hf = torch.empty((E, B, D, N), **f32)
    wsb = S.new_workspace(d, S.SWIMBA_OP_SEPARATE, "cuda:0")
    s = layer.stream

    def run(ev):
        if ev is not None:
            ev[0].record(s)
        S.check(S.swimba_scan_fwd(d, layer.x, layer.z, b.delta, b.B_mix, b.C_mix, b.idx, b.gates, w, None, b.out,
                                  b.h_final, None, b.ws, b.ws.numel(), s), "scan")
        if ev is not None:
            ev[1].record(s)
        S.check(S.swimba_separate_scan(d, layer.x, layer.z, dj, bj, cj, b.idx, b.gates, w, None, out, hf, None, wsb,
                                       wsb.numel(), s), "separate_scan")
        if ev is not None:
            ev[2].record(s)

    (sw_ms, sep_ms), _ = _median_kernel_ms(torch, run, reps, warmup, flush, 3)
    S.check(S.swimba_get_device_status(wsb, s), "device status")
    T = cfg.tokens
    return {
        "report": "separate_ssm_moe", "workload": cfg.name, "tokens": T, "n_experts": E, "top_k": k,
        "swimba_scan_us": 1e3 * sw_ms, "separate_scan_us": 1e3 * sep_ms, "separate_over_swimba": sep_ms / sw_ms,
        "exponentials_per_token": {"swimba": D * N, "separate": k * D * N},
        "state_bytes_per_sequence": {"swimba": 4 * D * N, "separate": 4 * E * D * N},
        "median_of": reps, "l2": "flushed (256 MB written, then read) before every run",
    }


SSD_WORKLOAD = {"name": "swimba_ssd_nemotron_like", "batch": 8, "seqlen": 4096, "heads": 64, "head_dim": 64,
                "d_state": 128}


def report_ssd(torch, S, peaks, flush, reps, warmup, w=SSD_WORKLOAD):
    """Swimba on the Mamba-2 SSD form (swimba_ssd_scan): B=8, L=4096, 64 heads of 64 channels,
    state 128, one active expert per token. FLOPs counted as computed per (chunk of 128, head):
    C Bᵀ (2 Q² N), W X (2 Q² P), C S_inᵀ (2 Q N P), Bᵀ X_w (2 N Q P)."""
    B, L, H, P, N = w["batch"], w["seqlen"], w["heads"], w["head_dim"], w["d_state"]
    inp = synth.draw_ssd_inputs(B, L, H, P, N, seed=9)
    dims = S.swimba_ssd_dims(batch=B, seqlen=L, n_heads=H, head_dim=P, d_state=N, top_k=1)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda:0")
    X, Bm, C = (S.to_device(a, "bf16", "cuda:0") for a in (inp.X, inp.B, inp.C_mix))
    g, dl, A, Dk, S0 = t(inp.gates), t(inp.delta), t(inp.A), t(inp.D_skip), t(inp.S0)
    y = torch.empty((B, L, H, P), dtype=torch.float32, device="cuda:0")
    sf = torch.empty((B, H, P, N), dtype=torch.float32, device="cuda:0")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda:0")
    s = torch.cuda.current_stream()

    def run(ev):
        if ev is not None:
            ev[0].record(s)
        S.check(S.swimba_ssd_scan(dims, X, Bm, C, g, dl, A, Dk, S0, y, sf, ws, ws.numel(), s), "ssd_scan")
        if ev is not None:
            ev[1].record(s)

    (ms,), _ = _median_kernel_ms(torch, run, reps, warmup, flush, 2)
    S.check(S.swimba_get_device_status(ws, s), "device status")
    Q = 128
    chunks = -(-L // Q)
    flops = B * H * chunks * (2 * Q * Q * N + 2 * Q * Q * P + 2 * Q * N * P + 2 * N * Q * P)
    nbytes = B * L * (H * P * 2 + 2 * N * 2 + 4 + H * 4 + H * P * 4) + 2 * B * H * P * N * 4
    sec = ms / 1e3
    return {
        "report": "ssd", "workload": w["name"], "batch": B, "seqlen": L, "heads": H, "head_dim": P, "d_state": N,
        "top_k": 1, "tokens": B * L, "ssd_us": 1e3 * ms, "tokens_per_s": B * L / sec,
        "tflops": flops / sec / 1e12, "frac_of_tc_peak": flops / sec / 1e12 / peaks["bf16_tflops"],
        "gbs": nbytes / sec / 1e9, "frac_of_hbm": nbytes / sec / 1e9 / peaks["hbm_gbs"],
        "flops_per_launch": flops, "bytes_per_launch": nbytes,
        "median_of": reps, "l2": "flushed (256 MB written, then read) before every run",
    }


def report_decode(torch, S, cfg, peaks, flush, steps):
    """``steps`` decode steps (route -> mixed_proj -> step) on one cached state, L2 flushed before
    every step; the same x, z every step (draws of step 0)."""
    dims = S.make_dims(cfg)
    w = S.upload_weights(synth.draw_weights(cfg), "cuda:0")
    ws = w.struct()
    x, z = synth.draw_step_activations(cfg, 0)
    xd, zd = S.to_device(x, cfg.io_dtype, "cuda:0"), S.to_device(z, cfg.io_dtype, "cuda:0")
    h = torch.from_numpy(synth.draw_h0(cfg)).to("cuda:0")
    buf = S.LayerBuffers(dims, torch.bfloat16, "cuda:0")
    s = torch.cuda.current_stream()

    def run(ev):
        if ev is not None:
            ev[0].record(s)
        S.check(S.swimba_route(dims, xd, ws.W_r, buf.idx, buf.gates, s), "route")
        if ev is not None:
            ev[1].record(s)
        S.check(S.swimba_mixed_proj(dims, xd, buf.idx, buf.gates, ws, buf.delta, buf.B_mix, buf.C_mix, buf.ws,
                                    buf.ws.numel(), s), "proj")
        if ev is not None:
            ev[2].record(s)
        S.check(S.swimba_step(dims, xd, zd, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, ws, h, buf.out, s),
                "step")
        if ev is not None:
            ev[3].record(s)

    (r_ms, p_ms, st_ms), tot = _median_kernel_ms(torch, run, steps, 3, flush, 4)

    # the whole step captured once as a CUDA graph (the entry points allocate nothing and never
    # synchronise, so they capture) and replayed: what a serving loop launches per layer step
    cap = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cap, capture_error_mode="relaxed"):
        g = torch.cuda.current_stream()
        S.check(S.swimba_route(dims, xd, ws.W_r, buf.idx, buf.gates, g), "route")
        S.check(S.swimba_mixed_proj(dims, xd, buf.idx, buf.gates, ws, buf.delta, buf.B_mix, buf.C_mix, buf.ws,
                                    buf.ws.numel(), g), "proj")
        S.check(S.swimba_step(dims, xd, zd, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, ws, h, buf.out, g),
                "step")
    torch.cuda.synchronize()

    def replay(ev):
        if ev is not None:
            ev[0].record(s)
        graph.replay()
        if ev is not None:
            ev[1].record(s)

    (g_ms,), _ = _median_kernel_ms(torch, replay, steps, 3, flush, 2)
    S.check(S.swimba_get_device_status(buf.ws, s), "device status")
    del graph
    B, D, N = cfg.batch, cfg.d_inner, cfg.d_state
    step_bytes = scan_bytes_per_token(cfg) * B + 2 * 4 * B * D * N
    return {
        "report": "decode", "workload": cfg.name, "steps": steps, "layer_us_per_step": 1e3 * tot,
        "layer_us_per_step_graph": 1e3 * g_ms,
        "route_us": 1e3 * r_ms, "proj_us": 1e3 * p_ms, "step_us": 1e3 * st_ms,
        "step_gbs": step_bytes / (st_ms / 1e3) / 1e9, "step_frac_of_hbm": step_bytes / (st_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "l2": "flushed before every step", "inputs": "x, z of step 0 reused every step; the state evolves",
        "timing": "CUDA events around each call with the host queued ahead (a GPU pause after the flush); "
                  "the graph line replays the captured step",
    }


def _device_block(torch, S, cfg, d_model, d_conv, seqlen=None):
    bw = synth.draw_block_weights(cfg, d_model, d_conv)
    dims = S.swimba_block_dims(S.make_dims(cfg, seqlen=seqlen), d_model, d_conv)
    keep = {
        "lw": S.upload_weights(bw.layer, "cuda:0"),
        "W_in": S.to_device(bw.W_in, cfg.w_dtype, "cuda:0"),
        "W_out": S.to_device(bw.W_out, cfg.w_dtype, "cuda:0"),
        "conv_w": torch.from_numpy(bw.conv_w).to("cuda:0"),
        "conv_b": torch.from_numpy(bw.conv_b).to("cuda:0"),
    }
    w = S.swimba_block_weights(keep["W_in"].data_ptr(), keep["conv_w"].data_ptr(), keep["conv_b"].data_ptr(),
                               keep["W_out"].data_ptr(), keep["lw"].struct())
    ws = torch.zeros(S.swimba_block_workspace_size(dims), dtype=torch.uint8, device="cuda:0")
    return dims, w, ws, keep


def report_block(torch, S, cfg, d_model, d_conv, peaks, flush, reps, warmup):
    """The surrounding block (in-projection, causal conv + SiLU, the layer, out-projection +
    residual) over whole sequences, and its causal convolution timed alone on the same shape."""
    dims, w, ws, keep = _device_block(torch, S, cfg, d_model, d_conv)
    u = S.to_device(synth.draw_block_input(cfg, d_model), cfg.io_dtype, "cuda:0")
    out = torch.empty_like(u)
    T, D = cfg.tokens, cfg.d_inner
    x_pre = torch.randn(cfg.batch, cfg.seqlen, D, device="cuda:0").to(torch.bfloat16)
    x_conv = torch.empty_like(x_pre)
    s = torch.cuda.current_stream()

    def run(ev):
        if ev is not None:
            ev[0].record(s)
        S.check(S.swimba_block_fwd(dims, u, w, None, None, out, None, None, ws, ws.numel(), s), "block_fwd")
        if ev is not None:
            ev[1].record(s)
        S.check(S.swimba_conv1d_fwd(dims.layer, d_conv, x_pre, keep["conv_w"], keep["conv_b"], None, x_conv, None, s),
                "conv1d_fwd")
        if ev is not None:
            ev[2].record(s)

    (b_ms, c_ms), _ = _median_kernel_ms(torch, run, reps, warmup, flush, 3)
    S.check(S.swimba_get_device_status(ws, s), "device status")

    # the two projection GEMMs alone through swimba_block_gemm, and cuBLAS (torch.matmul) on the
    # same operands beside them for comparison
    W_in, W_out = keep["W_in"], keep["W_out"]
    u2 = u.view(T, d_model)
    xz = torch.empty(T, 2 * D, dtype=u.dtype, device="cuda:0")
    yb = torch.randn(T, D, device="cuda:0").to(u.dtype)
    o2 = torch.empty(T, d_model, dtype=u.dtype, device="cuda:0")
    gws = torch.zeros(256, dtype=torch.uint8, device="cuda:0")
    dt = S.dtype_code(cfg.io_dtype)

    def run_gemm(ev):
        rec = (lambda i: ev[i].record(s)) if ev is not None else (lambda i: None)
        rec(0)
        S.check(S.swimba_block_gemm(dt, T, 2 * D, d_model, u2, d_model, W_in, 2 * D, xz, 2 * D, None, 0, 2 * D, None,
                                    0, gws, 256, s), "block_gemm in")
        rec(1)
        S.check(S.swimba_block_gemm(dt, T, d_model, D, yb, D, W_out, d_model, o2, d_model, None, 0, d_model, u2,
                                    d_model, gws, 256, s), "block_gemm out")
        rec(2)
        torch.matmul(u2, W_in, out=xz)
        rec(3)
        torch.addmm(u2, yb, W_out, out=o2)
        rec(4)

    (gi_ms, go_ms, ci_ms, co_ms), _ = _median_kernel_ms(torch, run_gemm, reps, warmup, flush, 5)
    S.check(S.swimba_get_device_status(gws, s), "gemm device status")
    conv_bytes = 2 * T * D * 2
    in_flops, out_flops = 2 * T * d_model * 2 * D, 2 * T * D * d_model
    tc_peak = peaks["bf16_tflops"]
    return {
        "report": "block", "workload": cfg.name, "d_model": d_model, "d_conv": d_conv, "tokens": T,
        "block_us": 1e3 * b_ms, "tokens_per_s": T / (b_ms / 1e3),
        "projection_gemm_gflop": (in_flops + out_flops) / 1e9,
        "in_gemm_us": 1e3 * gi_ms, "in_gemm_tflops": in_flops / gi_ms / 1e9,
        "in_gemm_frac_of_tc_peak": in_flops / gi_ms / 1e9 / tc_peak,
        "out_gemm_us": 1e3 * go_ms, "out_gemm_tflops": out_flops / go_ms / 1e9,
        "out_gemm_frac_of_tc_peak": out_flops / go_ms / 1e9 / tc_peak,
        "cublas_in_gemm_us": 1e3 * ci_ms, "cublas_out_gemm_us": 1e3 * co_ms,
        "conv_us": 1e3 * c_ms, "conv_gbs": conv_bytes / (c_ms / 1e3) / 1e9,
        "conv_frac_of_hbm": conv_bytes / (c_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "median_of": reps, "l2": "flushed (256 MB written, then read) before every run",
    }


def report_block_decode(torch, S, cfg, d_model, d_conv, peaks, flush, steps):
    """``steps`` block decode steps on one cached (h, conv state), L2 flushed before every step."""
    dims, w, ws, keep = _device_block(torch, S, cfg, d_model, d_conv)
    u = S.to_device(synth.draw_block_input(cfg.with_(seqlen=1), d_model), cfg.io_dtype, "cuda:0")
    out = torch.empty_like(u)
    h = torch.from_numpy(synth.draw_h0(cfg)).to("cuda:0")
    cs = S.to_device(synth.draw_conv_state(cfg, d_conv), cfg.io_dtype, "cuda:0")
    s = torch.cuda.current_stream()

    def run(ev):
        if ev is not None:
            ev[0].record(s)
        S.check(S.swimba_block_step(dims, u, w, h, cs, out, ws, ws.numel(), s), "block_step")
        if ev is not None:
            ev[1].record(s)

    (b_ms,), _ = _median_kernel_ms(torch, run, steps, 3, flush, 2)
    S.check(S.swimba_get_device_status(ws, s), "device status")
    return {
        "report": "block_decode", "workload": cfg.name, "d_model": d_model, "d_conv": d_conv, "steps": steps,
        "block_us_per_step": 1e3 * b_ms, "tokens_per_s": cfg.batch / (b_ms / 1e3),
        "l2": "flushed before every step", "inputs": "u of step 0 reused every step; both states evolve",
    }


def run_report_block(args):
    import torch

    from parameter_space_moe_swimba_b200 import swimba as S

    torch.cuda.set_device(0)
    peaks = load_peaks()
    flush = L2Flush(torch, "cuda:0")
    cfg = CONFIGS["mamba1p4b_like"]
    if args.batch:
        cfg = cfg.with_(batch=args.batch)
    print(json.dumps(report_block(torch, S, cfg, 2048, 4, peaks, flush, 20, args.warmup)), flush=True)
    if not args.batch:
        print(json.dumps(report_block_decode(torch, S, CONFIGS["decode_b256"], 2048, 4, peaks, flush, 200)), flush=True)
    return 0


def run_report(args):
    import torch

    from parameter_space_moe_swimba_b200 import swimba as S

    torch.cuda.set_device(0)
    peaks = load_peaks()
    flush = L2Flush(torch, "cuda:0")
    reps = 20
    for name in ["tiny_fp32", "mamba130m_like", "mamba1p4b_like", "long_seq_65536"]:
        print(json.dumps(report_workload(torch, S, CONFIGS[name], peaks, flush, reps, args.warmup)), flush=True)
    print(json.dumps(report_decode(torch, S, CONFIGS["decode_b256"], peaks, flush, 1000)), flush=True)
    # the surrounding block at the Mamba-1.4B-like width (d_model = D / 2, 4 conv taps)
    print(json.dumps(report_block(torch, S, CONFIGS["mamba1p4b_like"], 2048, 4, peaks, flush, reps, args.warmup)),
          flush=True)
    print(json.dumps(report_block_decode(torch, S, CONFIGS["decode_b256"], 2048, 4, peaks, flush, 200)), flush=True)
    # Swimba on the Mamba-2 SSD form
    print(json.dumps(report_ssd(torch, S, peaks, flush, reps, args.warmup)), flush=True)
    # Theorem 2 against the design it is set against: one trajectory per expert
    print(json.dumps(report_separate(torch, S, CONFIGS["mamba1p4b_like"], peaks, flush, reps, args.warmup)),
          flush=True)
    # the layer's backward pass (scan, projection and router gradients)
    print(json.dumps(report_bwd(torch, S, CONFIGS["mamba1p4b_like"], peaks, flush, 10, args.warmup)), flush=True)
    # Theorem 2: the recurrence's cost does not grow with E (k = 2 fixed; E = 1 forces k = 1)
    base = CONFIGS["mamba1p4b_like"]
    for E in (1, 4, 8, 16):
        cfg = base.with_(name=f"mamba1p4b_like_E{E}", n_experts=E, top_k=min(2, E))
        row = report_workload(torch, S, cfg, peaks, flush, reps, args.warmup)
        row["report"] = "e_sweep"
        row["n_experts"], row["top_k"] = E, cfg.top_k
        print(json.dumps(row), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------

def main():
    args = parse()
    if args.report:
        return run_report(args)
    if args.report_block:
        return run_report_block(args)
    if args.report_ssd:
        import torch

        from parameter_space_moe_swimba_b200 import swimba as S

        torch.cuda.set_device(0)
        print(json.dumps(report_ssd(torch, S, load_peaks(), L2Flush(torch, "cuda:0"), 20, args.warmup)), flush=True)
        return 0
    if args.report_decode:
        import torch

        from parameter_space_moe_swimba_b200 import swimba as S

        torch.cuda.set_device(0)
        cfg = CONFIGS["decode_b256"]
        cfg = cfg.with_(batch=args.batch) if args.batch > 0 else cfg
        print(json.dumps(report_decode(torch, S, cfg, load_peaks(), L2Flush(torch, "cuda:0"), args.steps)), flush=True)
        return 0
    if args.report_bwd:
        import torch

        from parameter_space_moe_swimba_b200 import swimba as S

        torch.cuda.set_device(0)
        cfg = CONFIGS[args.workload]
        cfg = cfg.with_(batch=args.batch) if args.batch > 0 else cfg
        cfg = cfg.with_(seqlen=args.seqlen) if args.seqlen > 0 else cfg
        print(json.dumps(report_bwd(torch, S, cfg, load_peaks(), L2Flush(torch, "cuda:0"), 10, args.warmup)),
              flush=True)
        return 0
    if args.report_separate:
        import torch

        from parameter_space_moe_swimba_b200 import swimba as S

        torch.cuda.set_device(0)
        print(json.dumps(report_separate(torch, S, CONFIGS[args.workload], load_peaks(), L2Flush(torch, "cuda:0"), 20,
                                         args.warmup)), flush=True)
        return 0
    cfg = CONFIGS[args.workload]
    if args.batch > 0:
        cfg = cfg.with_(batch=args.batch)
    if args.seqlen > 0:
        cfg = cfg.with_(seqlen=args.seqlen)
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
    # the CPU baseline's process pool starts (spawned, warmed up) before the timed GPU work
    cpu_pool = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_pool = OraclePool(cfg, 1024, list(range(cfg.batch)))

    from parameter_space_moe_swimba_b200 import swimba as S

    peaks = load_peaks()
    # this rank's shard of the global batch (world x batch sequences; sequences are independent)
    from parameter_space_moe_swimba_b200.parallel import batch_shard

    b0, b1 = batch_shard(cfg.batch * world, world, rank)
    x_host, z_host = synth.draw_activations(cfg, batch_rows=range(b0, b1))
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
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipeline": "two device slots; each step's H2D, kernels and D2H on three streams, so step i+1's "
                           "copies-in and step i-1's copy-out overlap step i's kernels"}

    scan_bytes = scan_bytes_per_token(cfg) * cfg.tokens + 4 * cfg.batch * cfg.d_inner * cfg.d_state
    achieved = scan_bytes / (per_kernel["scan"] / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic(cfg), "kernel": "scan_fwd",
                "algorithmic_bytes_per_launch": scan_bytes, "peak_source": peaks["source"]}
    # the scan's arithmetic bound: one ex2 per (token, channel, state) and one tanh per (token,
    # channel) on the special-function unit, 16 per clock per SM at the maximum SM clock
    mufu_ops = cfg.tokens * cfg.d_inner * (cfg.d_state + 1)
    mufu_peak = 16 * 148 * peaks["sm_max_mhz"] * 1e6
    mufu_achieved = mufu_ops / (per_kernel["scan"] / 1e3)
    alu_roofline = {"bound": "alu", "unit": "MUFU ops/s", "achieved": mufu_achieved, "peak": mufu_peak,
                    "frac": mufu_achieved / mufu_peak, "kernel": "scan_fwd",
                    "peak_from": "16 MUFU ops per clock per SM x 148 SMs x max SM clock"}
    kernels = {
        "route_us": 1e3 * per_kernel["route"], "proj_us": 1e3 * per_kernel["proj"], "scan_us": 1e3 * per_kernel["scan"],
        "route_gbs": route_bytes_per_token(cfg) * cfg.tokens / (per_kernel["route"] / 1e3) / 1e9,
        "proj_gbs": proj_bytes_per_token(cfg) * cfg.tokens / (per_kernel["proj"] / 1e3) / 1e9,
        "proj_tflops": proj_flops_per_token(cfg) * cfg.tokens / (per_kernel["proj"] / 1e3) / 1e12,
        "scan_gbs": achieved,
        "scan_exps_per_s": cfg.tokens * cfg.d_inner * cfg.d_state / (per_kernel["scan"] / 1e3),
    }

    cpu = None
    if cpu_pool is not None:
        dt = cpu_pool.run()
        cpu = {"value": cpu_pool.tokens * len(cpu_pool.rows) / dt, "unit": UNIT, "cores": cpu_pool.procs,
               "kind": "oracle", "sample": cpu_pool.sample()}
        cpu_pool.close()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config_block(cfg, world),
            "roofline": roofline, "alu_roofline": alu_roofline, "kernels": kernels, "switch_vs_dense_e1": dense, "e2e": e2e,
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
