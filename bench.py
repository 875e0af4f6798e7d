#!/usr/bin/env python
"""Throughput of the W8A8 FP8 block-scaled linear layer on B200.

One JSON line on rank 0.  A *step* is one pass of the hot path over the decode
GEMV set: fp8bq_linear (dynamic group-128 activation quantization fused into
the call, block-scaled FP8 GEMM, BF16 out) for M in {1, 4, 8} tokens against
the fused QKV weight [9216, 7168] and the o_proj weight [7168, 7168] -- six
linear layers per step.  The weights are quantized once (the offline half of
the method) and every call of a step reads its own device copy: six copies per
shape, steps alternating between copies 0-2 and 3-5, so a copy is read again
only after two whole steps (more than 350 MB of other weights, well over the
126 MB L2) and every call streams its weights from HBM.

``value`` is algorithmic HBM bytes per second (weight codes + weight scales +
BF16 activations + BF16 outputs; one pass over each), timed with CUDA events
around CUDA-graph replays of the steps, max over ranks.  Alongside:

* ``roofline``   the decode GEMM kernel alone (pre-quantized activations),
                 algorithmic bytes / its average launch time vs measured HBM.
* ``prefill``    fp8bq_linear and the GEMM kernel on the prefill fused-QKV
                 shape X[8192, 7168] W[9216, 7168], TFLOP/s (2 M N K) vs the
                 measured dense-FP8 peak (measured BF16 x 2), L2 flushed
                 between iterations.
* ``quantize_act`` on [32768, 7168] (long-prefill activation), GB/s.
* ``workloads``  GEMM-kernel and linear throughput for every other shape.
* ``e2e``        the same decode steps through the public API from pinned host
                 buffers: H2D copy of X, the linear call, D2H copy of Y.
* ``cpu_baseline`` the CPU oracle (plain C, FP64 GEMM) on full decode steps;
                 each prefill row also carries one, timed on two row subsets
                 and extrapolated to the full M (labelled as such).

``--impl reference`` times the CPU oracle instead, on the same metric.
``--gpus N`` (under torchrun) runs N independent replicas, one per GPU: the
layer has no exchange step, so there is no collective on the data path.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "FP8 block-scaled GEMM TFLOPS (prefill) & HBM GB/s (decode), % of roofline, 1 B200"
FP8_OVER_BF16 = 2.0          # nominal dense ratio 4.5 / 2.25 PFLOP/s
# Nominal B200 figures, for the second fraction reported beside the measured
# one: HBM3e 7.7 TB/s (HGX), dense FP8 4.5 PFLOP/s.
NOMINAL_HBM_GBS = 7700.0
NOMINAL_FP8_TFLOPS = 4500.0
COPIES = 6                   # device copies of each decode weight (3 calls per shape per step)
STEP_VARIANTS = 2            # steps alternate between copies 0-2 and 3-5
# DRAM bytes (read + write) per decode GEMM launch, averaged over consecutive launches of the
# graph-replayed decode-GEMM step (per-call weight copies, L2 state carried from launch to
# launch), measured by ncu on `bench.py --only decode-graph`.  Valid only for the decode
# kernel source it was taken on: `kernel_sha` is the SHA-256 (first 16 hex digits) of
# gemm_decode.cuh + ptx.cuh; when the source differs, the traffic is reported as null.
DECODE_TRAFFIC = {"bytes_per_launch": 57746954, "kernel_sha": "bf3c4541ec7aa1fd",
                  "how": "ncu --cache-control none --clock-control none --metrics "
                         "dram__bytes_read.sum,dram__bytes_write.sum on the 24 graph-replayed "
                         "decode GEMM launches (4 steps of 6) of `bench.py --only decode-graph`: "
                         "57.30 MB read + 0.44 MB written per launch"}
DECODE_WORKLOAD = ("decode GEMV set: fp8bq_linear, M in {1,4,8} x {fused QKV W[9216,7168], "
                   "o_proj W[7168,7168]}, E4M3 128x128-blocked weights, X BF16 N(0,1) with "
                   "7 outlier channels x20")


# ----------------------------------------------------------------------------- helpers

def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def decode_kernel_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm_decode.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "fp8_block_scaled_09_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def weight_copy(step: int, call: int) -> int:
    """Device copy of its shape's weight that `call` (0..2 within its shape) of
    step `step` reads: steps alternate between copies 0-2 and 3-5."""
    return 3 * (step % STEP_VARIANTS) + call


def linear_bytes(g: W.Gemm) -> int:
    """Algorithmic bytes of one linear: W codes, W scales, BF16 X in, BF16 Y out."""
    return g.N * g.K + (g.N // 128) * (g.K // 128) * 4 + g.M * g.K * 2 + g.M * g.N * 2


def gemm_bytes(g: W.Gemm) -> int:
    """Algorithmic bytes of one GEMM launch: W and X codes, both scale sets, BF16 Y."""
    return (g.N * g.K + (g.N // 128) * (g.K // 128) * 4 + g.M * g.K + g.M * (g.K // 128) * 4
            + g.M * g.N * 2)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_device_index: int):
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._on = False
        self._thread = None
        self.error = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device_index).uuid)
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 -- clocks are reported as unavailable
            self.error = f"{type(e).__name__}: {e}"
            self._h = None

    def _run(self):
        nv = self._nvml
        while self._on:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, rs))
            except Exception as e:  # noqa: BLE001
                self.error = str(e)
                return
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._on = True
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._on = False
        if self._thread is not None:
            self._thread.join()
            # one sample right after the region, so short regions still get one
            try:
                self.samples.append((self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM),
                                     self._nvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)))
            except Exception:  # noqa: BLE001
                pass

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml", "error": self.error}
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "nvml, 2 ms polling during the timed regions"}


def max_over_ranks(v: float, world: int, device=None) -> float:
    """The largest value over all ranks (the timed region of the slowest replica)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, units_per_step: float, steps: int, ms_max: float,
                       scale: float = 1e-9) -> float:
    """Whole-job throughput of `world` replicas that each processed `units_per_step`
    per step for `steps` steps, timed by the slowest one (weak scaling)."""
    return world * units_per_step * steps / (ms_max * 1e-3) * scale


def events_ms(torch, fn, iters: int) -> float:
    s = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    for i in range(iters):
        fn(i)
    e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def flushed_ms(torch, fn, iters: int, warmup: int, flush) -> list[float]:
    """Per-iteration device times of fn with an L2 flush (untimed) before each.

    fn is captured once into a CUDA graph and replayed, and a short device-side
    sleep follows each flush, so the replay is already queued when the stream
    reaches the start event: the interval holds the kernels only, not the
    Python and driver time spent launching them.  The flush writes a buffer
    larger than L2 and then reads it back, so L2 holds clean lines when the
    timed kernels start (after a write alone, the kernels would pay for writing
    back ~126 MB of the flush's dirty lines)."""
    s = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(s)
    with torch.cuda.stream(side):
        fn()
    s.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    torch.cuda.synchronize()
    evs = []
    for i in range(warmup + iters):
        flush.zero_()
        flush.max()
        torch.cuda._sleep(100_000)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        graph.replay()
        e1.record(s)
        if i >= warmup:
            evs.append((e0, e1))
    torch.cuda.synchronize()
    del graph
    return [a.elapsed_time(b) for a, b in evs]


# ----------------------------------------------------------------------------- reference arm

def decode_host_inputs():
    """Host BF16 activations and weights of the decode set (seeded)."""
    xs = [g.make_x() for g in W.DECODE_SET]
    ws = {}
    for g in W.DECODE_SET:
        if g.N not in ws:
            ws[g.N] = g.make_w()
    return xs, ws


def oracle_decode_steps(oracle, xs, qws, steps: int, col_frac: float = 1.0):
    """Runs `steps` decode steps of the oracle; returns (seconds, algorithmic bytes)."""
    total_bytes = 0
    t0 = time.perf_counter()
    for _ in range(steps):
        for g, x in zip(W.DECODE_SET, xs):
            qw, sw = qws[g.N]
            nb = max(1, int(round(col_frac * (g.N // 128))))
            n = nb * 128
            oracle.linear_ref(x, qw[:n], sw[:nb])
            total_bytes += linear_bytes(W.scaled(g, N=n)) if n != g.N else linear_bytes(g)
    return time.perf_counter() - t0, total_bytes


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    import oracle
    oracle.build()
    xs, ws = decode_host_inputs()
    qws = {N: oracle.quantize_weight(w) for N, w in ws.items()}    # offline step, untimed
    # size each step so the whole run stays within about two minutes
    t_one, _ = oracle_decode_steps(oracle, xs, qws, 1)
    budget_s = 120.0
    frac = min(1.0, budget_s / max(1e-9, (args.steps + args.warmup) * t_one))
    oracle_decode_steps(oracle, xs, qws, args.warmup, frac)
    secs, nbytes = oracle_decode_steps(oracle, xs, qws, args.steps, frac)
    gbs = nbytes / secs / 1e9
    cores = len(os.sched_getaffinity(0))
    sample = (f"each step: the 6 decode linears on {frac:.3f} of the output columns "
              "(whole n-blocks), all rows and all K; oracle.linear_ref (plain C, OpenMP, "
              "binary32 quantizer + FP64 GEMM)")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy PCG64, BF16)",
        "config": {"workload": DECODE_WORKLOAD, "device": "host CPU"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm

def decode_device_set(torch, fp8bq, dev, xs_host, ws_host):
    """Device weights (COPIES per shape), activations, codes and workspaces of the
    decode set; each call records its index among the calls of its shape."""
    qw_rot, sw_rot = {}, {}
    for N, w in ws_host.items():
        qw, sw = fp8bq.quantize_weight(w.to(dev))
        qw_rot[N] = [qw] + [qw.clone() for _ in range(COPIES - 1)]
        sw_rot[N] = [sw] + [sw.clone() for _ in range(COPIES - 1)]
    calls, seen = [], {}
    for g, xh in zip(W.DECODE_SET, xs_host):
        x = xh.to(dev)
        qa, sa = fp8bq.quantize_act(x)
        calls.append({
            "g": g, "x": x, "qa": qa, "sa": sa, "call": seen.get(g.N, 0),
            "y": torch.empty((g.M, g.N), dtype=torch.bfloat16, device=dev),
            "ws_lin": fp8bq.new_workspace(fp8bq.OP_LINEAR, g.M, g.N, g.K, dev),
            "ws_gemm": fp8bq.new_workspace(fp8bq.OP_GEMM, g.M, g.N, g.K, dev),
            "x_host": xh,
        })
        seen[g.N] = seen.get(g.N, 0) + 1
    assert all(v * STEP_VARIANTS <= COPIES for v in seen.values())
    return qw_rot, sw_rot, calls


def decode_gemm_step(fp8bq, calls, qw_rot, sw_rot, r: int) -> None:
    """The decode GEMM kernel alone on every call of step r (pre-quantized activations)."""
    for c in calls:
        k = weight_copy(r, c["call"])
        N = c["g"].N
        fp8bq.gemm(c["qa"], c["sa"], qw_rot[N][k], sw_rot[N][k], out=c["y"],
                   workspace=c["ws_gemm"])


def capture_steps(torch, step_fn):
    """One CUDA graph per step variant (steps alternate between weight copies)."""
    graphs = []
    for r in range(STEP_VARIANTS):
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph):
            step_fn(r)
        graphs.append(gph)
    return graphs


def run_ours(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    import fp8_block_scaled_09_b200 as fp8bq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    fp8_peak_sus = peaks["bf16_tflops_sustained"] * FP8_OVER_BF16
    warmup = max(3, args.warmup)
    clocks = ClockSampler(local_rank)

    def barrier():
        if world > 1:
            dist.barrier()


    # ---------------------------------------------------------------- decode set
    xs_host, ws_host = decode_host_inputs()
    qw_rot, sw_rot, calls = decode_device_set(torch, fp8bq, dev, xs_host, ws_host)
    step_bytes = sum(linear_bytes(c["g"]) for c in calls)
    gemm_step_bytes = sum(gemm_bytes(c["g"]) for c in calls)

    def linear_step(r: int):
        for c in calls:
            k = weight_copy(r, c["call"])
            N = c["g"].N
            fp8bq.linear(c["x"], qw_rot[N][k], sw_rot[N][k], out=c["y"], workspace=c["ws_lin"])

    def gemm_step(r: int):
        decode_gemm_step(fp8bq, calls, qw_rot, sw_rot, r)

    # eager warm-up (also sets the library up on this device), launch counts per step
    n0 = fp8bq.launch_count()
    linear_step(0)
    kernels_per_step = fp8bq.launch_count() - n0
    n0 = fp8bq.launch_count()
    gemm_step(0)
    gemm_kernels_per_step = fp8bq.launch_count() - n0
    torch.cuda.synchronize()

    lin_graphs = capture_steps(torch, linear_step)
    gemm_graphs = capture_steps(torch, gemm_step)
    for i in range(warmup):
        lin_graphs[i % STEP_VARIANTS].replay()
    torch.cuda.synchronize()

    barrier()
    with clocks:
        ms = events_ms(torch, lambda i: lin_graphs[i % STEP_VARIANTS].replay(), args.steps)
    barrier()
    ms = max_over_ranks(ms, world, dev)
    value = replica_throughput(world, step_bytes, args.steps, ms)

    # dominant kernel: the decode GEMM alone
    for i in range(warmup):
        gemm_graphs[i % STEP_VARIANTS].replay()
    barrier()
    with clocks:
        gms = events_ms(torch, lambda i: gemm_graphs[i % STEP_VARIANTS].replay(), args.steps)
    barrier()
    gms = max_over_ranks(gms, world, dev)
    gemm_launches = args.steps * gemm_kernels_per_step
    gemm_gbs = gemm_step_bytes * args.steps / (gms * 1e-3) / 1e9
    sha = decode_kernel_sha()
    traffic = DECODE_TRAFFIC["bytes_per_launch"] if DECODE_TRAFFIC["kernel_sha"] == sha else None
    roofline = {"bound": "hbm", "achieved": gemm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gemm_gbs / peaks["hbm_gbs"], "frac_of_nominal": gemm_gbs / NOMINAL_HBM_GBS,
                "traffic": traffic,
                "traffic_source": DECODE_TRAFFIC["how"] if traffic is not None else
                                  f"null: no capture for this decode kernel source ({sha})",
                "kernel": "fp8bq::decode::gemm_decode_kernel<16> (cluster split)",
                "avg_launch_us": gms * 1e3 / gemm_launches,
                "algorithmic_bytes_per_launch": gemm_step_bytes / gemm_kernels_per_step,
                "peak_source": f"{peaks['source']} HBM copy bandwidth"}

    # ---------------------------------------------------------------- e2e through the API
    # The step's inputs live in one pinned host buffer and its outputs in another,
    # as a serving loop stages them: one host->device copy of every X, the six
    # fp8bq.linear calls on views of one device buffer, one device->host copy of
    # every Y.
    x_sizes = [c["g"].M * c["g"].K for c in calls]
    y_sizes = [c["g"].M * c["g"].N for c in calls]
    x_all_pin = torch.empty(sum(x_sizes), dtype=torch.bfloat16).pin_memory()
    y_all_pin = torch.empty(sum(y_sizes), dtype=torch.bfloat16).pin_memory()
    x_all = torch.empty(sum(x_sizes), dtype=torch.bfloat16, device=dev)
    y_all = torch.empty(sum(y_sizes), dtype=torch.bfloat16, device=dev)
    xo = yo = 0
    for c, nx, ny in zip(calls, x_sizes, y_sizes):
        x_all_pin[xo:xo + nx].copy_(c["x_host"].reshape(-1))
        c["x_e2e"] = x_all[xo:xo + nx].view(c["g"].M, c["g"].K)
        c["y_e2e"] = y_all[yo:yo + ny].view(c["g"].M, c["g"].N)
        xo += nx
        yo += ny

    def e2e_step(r: int):
        x_all.copy_(x_all_pin, non_blocking=True)
        for c in calls:
            k = weight_copy(r, c["call"])
            N = c["g"].N
            fp8bq.linear(c["x_e2e"], qw_rot[N][k], sw_rot[N][k], out=c["y_e2e"],
                         workspace=c["ws_lin"])
        y_all_pin.copy_(y_all, non_blocking=True)

    for i in range(warmup):
        e2e_step(i)
    barrier()
    with clocks:
        ems = events_ms(torch, lambda i: e2e_step(i), args.steps)
    barrier()
    ems = max_over_ranks(ems, world, dev)
    h2d = x_all.numel() * 2
    d2h = y_all.numel() * 2
    e2e = {"value": replica_throughput(world, step_bytes, args.steps, ems), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "how": "per step: one copy of every layer's X from a pinned host buffer, the six "
                  "fp8bq.linear calls, one copy of every Y to a pinned host buffer; eager "
                  "launches from Python, CUDA events on the stream"}

    extras = {}
    if not args.quick:
        extras = prefill_and_workloads(torch, fp8bq, dev, clocks, peaks, fp8_peak, fp8_peak_sus,
                                       args, cpu=rank == 0 and world == 1 and not args.no_cpu_baseline)

    status = fp8bq.last_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the benchmark")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(xs_host, ws_host)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic (seeded numpy PCG64, BF16; weights quantized on the GPU)",
            "config": {"workload": DECODE_WORKLOAD, "layers_per_step": len(calls),
                       "algorithmic_bytes_per_step": step_bytes,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs larger than L2: each call of a step reads its own weight "
                             f"copy ({COPIES} per shape); a copy is read again only after two "
                             "whole steps (> 350 MB of other weights)",
                       "timing": "CUDA events around CUDA-graph replays, max over ranks"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * kernels_per_step,
            "clocks": clocks.summary(),
            "peaks": peaks,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)


def oracle_prefill_baseline(g: W.Gemm, x_host, w_host) -> dict:
    """The CPU oracle's linear layer (quantize the activation rows, FP64 GEMM) on
    two evenly spaced row subsets of a prefill shape, all N and K, extrapolated to
    the full M with t(M) = a + b M fitted to the two timings (a: the per-call
    dequantization of W; b: one row).  The weight quantization is offline and
    untimed, as on the GPU."""
    import oracle
    oracle.build()
    qw, sw = oracle.quantize_weight(w_host)
    times = {}
    for r in (8, 24):
        rows = np.linspace(0, g.M - 1, r).round().astype(np.int64)
        t0 = time.perf_counter()
        oracle.linear_ref(x_host, qw, sw, rows=rows)
        times[r] = time.perf_counter() - t0
    b = max(1e-12, (times[24] - times[8]) / 16)
    a = max(0.0, times[8] - 8 * b)
    t_full = a + b * g.M
    return {"value": g.flops / t_full / 1e12, "unit": "TFLOP/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle", "extrapolated": True,
            "sample": f"oracle.linear_ref on 8 and 24 evenly spaced rows of {g.M} (all N, K): "
                      f"{times[8]:.2f} s and {times[24]:.2f} s; full M extrapolated as "
                      f"a + b M = {t_full:.1f} s"}


def prefill_and_workloads(torch, fp8bq, dev, clocks, peaks, fp8_peak, fp8_peak_sus, args,
                          cpu: bool = False):
    iters = max(5, min(20, args.steps))
    warm = 3
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {}

    def shape_result(g: W.Gemm, with_linear: bool):
        x_host = g.make_x()
        x = x_host.to(dev)
        qw, sw = fp8bq.quantize_weight(g.make_w().to(dev))
        qa, sa = fp8bq.quantize_act(x)
        y = torch.empty((g.M, g.N), dtype=torch.bfloat16, device=dev)
        wsg = fp8bq.new_workspace(fp8bq.OP_GEMM, g.M, g.N, g.K, dev)
        wsl = fp8bq.new_workspace(fp8bq.OP_LINEAR, g.M, g.N, g.K, dev)
        with clocks:
            tg = flushed_ms(torch, lambda: fp8bq.gemm(qa, sa, qw, sw, out=y, workspace=wsg),
                            iters, warm, flush)
            tl = flushed_ms(torch, lambda: fp8bq.linear(x, qw, sw, out=y, workspace=wsl),
                            iters, warm, flush) if with_linear else None
        r = {"name": g.name, "M": g.M, "N": g.N, "K": g.K}
        mg = statistics.fmean(tg)
        if g.M <= 128:
            # weight-streaming regime (decode kernel): bandwidth is the bound
            gbs = gemm_bytes(g) / (mg * 1e-3) / 1e9
            r.update({"gemm_us": mg * 1e3, "gemm_gbs": gbs, "gemm_frac_hbm": gbs / peaks["hbm_gbs"],
                      "gemm_tflops": g.flops / (mg * 1e-3) / 1e12})
            if tl:
                ml = statistics.fmean(tl)
                r.update({"linear_us": ml * 1e3,
                          "linear_gbs": linear_bytes(g) / (ml * 1e-3) / 1e9})
        else:
            tf = g.flops / (mg * 1e-3) / 1e12
            r.update({"gemm_us": mg * 1e3, "gemm_tflops": tf, "gemm_frac_fp8": tf / fp8_peak})
            if tl:
                ml = statistics.fmean(tl)
                r.update({"linear_us": ml * 1e3, "linear_tflops": g.flops / (ml * 1e-3) / 1e12})
            if cpu:
                r["cpu_baseline"] = oracle_prefill_baseline(g, x_host, g.make_w())
        del x, qw, sw, qa, sa, y
        return r

    pq = shape_result(W.PREFILL_QKV, True)
    out["prefill"] = {
        "workload": "prefill fused QKV: X[8192,7168] x W[9216,7168]^T, BF16 out",
        "metric": "TFLOP/s (2 M N K)", "linear_tflops": pq["linear_tflops"],
        "linear_us": pq["linear_us"], "gemm_tflops": pq["gemm_tflops"],
        "gemm_us": pq["gemm_us"], "cpu_baseline": pq.get("cpu_baseline"),
        "roofline": {"bound": "tensor", "achieved": pq["gemm_tflops"], "peak": fp8_peak,
                     "unit": "TFLOP/s", "frac": pq["gemm_tflops"] / fp8_peak,
                     "frac_of_sustained": pq["gemm_tflops"] / fp8_peak_sus,
                     "frac_of_nominal": pq["gemm_tflops"] / NOMINAL_FP8_TFLOPS, "traffic": None,
                     "kernel": "fp8bq::prefill::gemm_prefill_kernel<256, false, 32>",
                     "peak_source": f"{peaks['source']} cuBLAS BF16 x 2 (nominal FP8/BF16 ratio)"},
        "timing": f"mean of {iters} graph replays, CUDA events, L2 flushed (256 MB write + read) before each",
    }

    # standalone activation quantizer on the long-prefill activation
    g = W.LONG_O_PROJ
    x = g.make_x().to(dev)
    q = torch.empty((g.M, g.K), dtype=torch.uint8, device=dev)
    s = torch.empty((g.M, g.K // 128), dtype=torch.float32, device=dev)
    with clocks:
        tq = flushed_ms(torch, lambda: fp8bq.quantize_act(x, q, s), iters, warm, flush)
    mq = statistics.fmean(tq)
    qbytes = g.M * g.K * 2 + g.M * g.K + g.M * (g.K // 128) * 4
    out["quantize_act"] = {"shape": [g.M, g.K], "us": mq * 1e3, "gbs": qbytes / (mq * 1e-3) / 1e9,
                           "frac_hbm": qbytes / (mq * 1e-3) / 1e9 / peaks["hbm_gbs"],
                           "algorithmic_bytes": qbytes}
    del x, q, s

    mid = [shape_result(g, True) for g in W.MIDM_SET]
    q128 = next(r for r in mid if r["name"] == "qkv_m128")
    out["mid_m"] = {
        "workload": "mid-size batches (32 and 128 rows) on fused QKV [9216,7168] and o_proj "
                    "[7168,7168]: decode kernel with a 32- or 128-row token tile",
        "rows": mid,
        "roofline": {"bound": "hbm", "achieved": q128["gemm_gbs"], "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": q128["gemm_gbs"] / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "fp8bq::decode::gemm_decode_kernel<128> (qkv_m128)",
                     "algorithmic_bytes": gemm_bytes(W.by_name("qkv_m128"))},
        "timing": f"mean of {iters} graph replays, CUDA events, L2 flushed (256 MB write + read) before each",
    }

    # FP8 KV-cache write with unit scales: K and V of the fused QKV output
    kv_rows = []
    for T in (2048, 32768):
        gen = torch.Generator(device=dev).manual_seed(T)
        qkv = torch.randn((T, 9216), generator=gen, device=dev).mul_(3).to(torch.bfloat16)
        loc = torch.randperm(T, generator=gen, device=dev)
        kc = torch.empty((T, 1024), dtype=torch.uint8, device=dev)
        vc = torch.empty_like(kc)
        kk, vv = qkv[:, 7168:8192], qkv[:, 8192:]
        with clocks:
            tk = flushed_ms(torch, lambda: fp8bq.kv_write_e4m3(kk, vv, loc, kc, vc), iters, warm, flush)
        mk = statistics.fmean(tk)
        kbytes = T * (6 * 1024 + 8)
        kv_rows.append({"T": T, "width": 1024, "us": mk * 1e3, "gbs": kbytes / (mk * 1e-3) / 1e9,
                        "frac_hbm": kbytes / (mk * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "algorithmic_bytes": kbytes})
        del qkv, loc, kc, vc
    out["kv_write"] = {"rows": kv_rows,
                       "bytes": "per token: K and V read in BF16 (4 x 1024 B), written in E4M3 "
                                "(2 x 1024 B), slot index 8 B"}

    # SiLU-gated product quantized for the down projection (drafter MLP shape)
    Mg, Ig = 4096, 8192
    gen = torch.Generator(device=dev).manual_seed(4)
    gu = torch.randn((Mg, 2 * Ig), generator=gen, device=dev).mul_(2).to(torch.bfloat16)
    qh = torch.empty((Mg, Ig), dtype=torch.uint8, device=dev)
    sh = torch.empty((Mg, Ig // 128), dtype=torch.float32, device=dev)
    hb = torch.empty((Mg, Ig), dtype=torch.bfloat16, device=dev)

    def unfused():
        torch.mul(torch.nn.functional.silu(gu[:, :Ig]), gu[:, Ig:], out=hb)
        fp8bq.quantize_act(hb, qh, sh)

    with clocks:
        tf = flushed_ms(torch, lambda: fp8bq.silu_mul_quantize(gu, qh, sh), iters, warm, flush)
        tu = flushed_ms(torch, unfused, iters, warm, flush)
    mf, mu = statistics.fmean(tf), statistics.fmean(tu)
    sbytes = Mg * 2 * Ig * 2 + Mg * Ig + Mg * (Ig // 128) * 4
    out["silu_mul_quantize"] = {
        "shape": {"M": Mg, "I": Ig}, "us": mf * 1e3, "gbs": sbytes / (mf * 1e-3) / 1e9,
        "frac_hbm": sbytes / (mf * 1e-3) / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes": sbytes,
        "unfused_us": mu * 1e3,
        "unfused": "torch silu * up into BF16 h, then fp8bq.quantize_act(h): context only"}
    del gu, qh, sh, hb

    # gate/up GEMM -> codes of the down projection's input: the fused epilogue
    # (fp8bq_gemm_silu_mul_quantize) against the GEMM writing BF16 gate/up and
    # the SiLU kernel reading it back (drafter MLP shape, M = 4096, I = 8192)
    g = W.DRAFTER_GATE_UP
    I = g.N // 2
    xg = g.make_x().to(dev)
    qwg, swg = fp8bq.quantize_weight(g.make_w().to(dev))
    qag, sag = fp8bq.quantize_act(xg)
    gu = torch.empty((g.M, g.N), dtype=torch.bfloat16, device=dev)
    qh = torch.empty((g.M, I), dtype=torch.uint8, device=dev)
    sh = torch.empty((g.M, I // 128), dtype=torch.float32, device=dev)
    wsg = fp8bq.new_workspace(fp8bq.OP_GEMM, g.M, g.N, g.K, dev)

    def chain():
        fp8bq.gemm(qag, sag, qwg, swg, out=gu, workspace=wsg)
        fp8bq.silu_mul_quantize(gu, qh, sh)

    with clocks:
        tfu = flushed_ms(torch, lambda: fp8bq.gemm_silu_mul_quantize(qag, sag, qwg, swg, q=qh, s=sh),
                         iters, warm, flush)
        tch = flushed_ms(torch, chain, iters, warm, flush)
    mfu, mch = statistics.fmean(tfu), statistics.fmean(tch)
    out["gate_up_silu"] = {
        "workload": "drafter gate/up X[4096,7168] x W[16384,7168]^T -> E4M3 codes and scales of "
                    "h = silu(gate) * up [4096, 8192] (the down projection's input)",
        "fused_us": mfu * 1e3, "fused_tflops": g.flops / (mfu * 1e-3) / 1e12,
        "fused_frac_fp8": g.flops / (mfu * 1e-3) / 1e12 / fp8_peak,
        "chain_us": mch * 1e3,
        "chain": "fp8bq_gemm (BF16 gate/up to HBM) then fp8bq_silu_mul_quantize",
        "timing": f"mean of {iters} graph replays, CUDA events, L2 flushed before each"}
    del xg, qwg, swg, qag, sag, gu, qh, sh, wsg

    # NVFP4 weight-only GEMM (A16), decode shapes: back-to-back graph replays over 4
    # weight copies per shape (larger than L2), like the headline decode measurement
    nv_rows = []
    for name in ("qkv_m1", "o_proj_m1", "qkv_m8", "o_proj_m8"):
        gshape = W.by_name(name)
        w = gshape.make_w().to(dev)
        copies = [fp8bq.nvfp4_quantize_weight(w) for _ in range(4)]
        x = gshape.make_x().to(dev)
        y = torch.empty((gshape.M, gshape.N), dtype=torch.bfloat16, device=dev)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for c in copies:
                fp8bq.nvfp4_gemm_a16(x, *c, out=y)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for rep in range(2):
                for c in copies:
                    fp8bq.nvfp4_gemm_a16(x, *c, out=y)
        for _ in range(3):
            graph.replay()
        with clocks:
            t = events_ms(torch, lambda i: graph.replay(), iters)
        us = t / (iters * 8) * 1e3
        nbytes = (gshape.N * gshape.K // 2 + gshape.N * gshape.K // 16 + 4
                  + gshape.M * gshape.K * 2 + gshape.M * gshape.N * 2)
        nv_rows.append({"name": name, "M": gshape.M, "N": gshape.N, "K": gshape.K, "us": us,
                        "gbs": nbytes / (us * 1e-6) / 1e9,
                        "frac_hbm": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                        "algorithmic_bytes": nbytes})
        del graph, copies, w, x, y
    out["nvfp4_a16"] = {
        "workload": "NVFP4 weight-only GEMM, BF16 activations: decode QKV / o_proj at M = 1, 8",
        "rows": nv_rows,
        "bytes": "E2M1 codes N*K/2 + E4M3 block scales N*K/16 + global scale + X BF16 + Y BF16",
        "timing": "CUDA events around graph replays of 8 back-to-back launches over 4 weight copies"}

    rows = [pq]
    for g in (W.KPROJ_M16,) + W.DRAFTER_MLP + (W.LONG_O_PROJ,):
        rows.append(shape_result(g, True))
    out["workloads"] = rows
    return out


def cpu_baseline(xs_host, ws_host) -> dict:
    import oracle
    oracle.build()
    qws = {N: oracle.quantize_weight(w) for N, w in ws_host.items()}   # offline step, untimed
    secs, nbytes = oracle_decode_steps(oracle, xs_host, qws, 1)
    steps = 1
    while secs < 10.0 and steps < 16:
        s2, b2 = oracle_decode_steps(oracle, xs_host, qws, 1)
        secs += s2
        nbytes += b2
        steps += 1
    return {"value": nbytes / secs / 1e9, "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{steps} full decode steps (the same 6 linears, all columns), "
                      "oracle.linear_ref: plain C with OpenMP, FP64 GEMM accumulation"}


def run_profile_case(case: str) -> None:
    """A small, self-contained run of one kernel family (for ncu captures)."""
    import torch

    import fp8_block_scaled_09_b200 as fp8bq
    dev = torch.device("cuda", 0)
    t0 = time.perf_counter()
    if case == "quantize":
        g = W.LONG_O_PROJ
        x = g.make_x().to(dev)
        for _ in range(3):
            fp8bq.quantize_act(x)
    elif case == "kv":
        T = 32768
        qkv = torch.randn((T, 9216), device=dev).to(torch.bfloat16)
        loc = torch.randperm(T, device=dev)
        kc = torch.empty((T, 1024), dtype=torch.uint8, device=dev)
        vc = torch.empty_like(kc)
        for _ in range(3):
            fp8bq.kv_write_e4m3(qkv[:, 7168:8192], qkv[:, 8192:], loc, kc, vc)
    elif case == "nvfp4":
        gs = W.by_name("o_proj_m1")
        packed, sb, g = fp8bq.nvfp4_quantize_weight(gs.make_w().to(dev))
        x = gs.make_x().to(dev)
        for _ in range(3):
            fp8bq.nvfp4_gemm_a16(x, packed, sb, g)
    elif case == "silu":
        gu = torch.randn((4096, 16384), device=dev).mul_(2).to(torch.bfloat16)
        for _ in range(3):
            fp8bq.silu_mul_quantize(gu)
    elif case == "gateup":
        # the gate/up GEMM with the SiLU-gated quantization in its epilogue
        g = W.DRAFTER_GATE_UP
        qw, sw = fp8bq.quantize_weight(g.make_w().to(dev))
        qa, sa = fp8bq.quantize_act(g.make_x().to(dev))
        for _ in range(2):
            fp8bq.gemm_silu_mul_quantize(qa, sa, qw, sw)
    elif case == "decode-graph":
        # the bench's decode-GEMM step: per-call weight copies, CUDA-graph replays
        xs_host, ws_host = decode_host_inputs()
        qw_rot, sw_rot, calls = decode_device_set(torch, fp8bq, dev, xs_host, ws_host)
        decode_gemm_step(fp8bq, calls, qw_rot, sw_rot, 0)
        torch.cuda.synchronize()
        graphs = capture_steps(torch, lambda r: decode_gemm_step(fp8bq, calls, qw_rot, sw_rot, r))
        for i in range(4):
            graphs[i % STEP_VARIANTS].replay()
    else:
        gs = {"decode": W.DECODE_SET, "midm": W.MIDM_SET}.get(case, (W.PREFILL_QKV,))
        wq = {}
        for g in gs:
            if g.N not in wq:
                wq[g.N] = fp8bq.quantize_weight(g.make_w().to(dev))
        for g in gs:
            x = g.make_x().to(dev)
            qw, sw = wq[g.N]
            qa, sa = fp8bq.quantize_act(x)
            for _ in range(2):
                fp8bq.gemm(qa, sa, qw, sw)
                fp8bq.linear(x, qw, sw)
    torch.cuda.synchronize()
    status = fp8bq.last_device_status()
    print(json.dumps({"profile_case": case, "launches": fp8bq.launch_count(), "status": status,
                      "seconds": time.perf_counter() - t0}), flush=True)
    if status != 0:
        raise SystemExit(1)


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--quick", action="store_true", help="decode set only (no prefill/workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=("decode", "decode-graph", "midm", "prefill", "quantize",
                                       "kv", "silu", "gateup", "nvfp4"),
                    help="profiling case: run one kernel family a few times, print a short line")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")

    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.only:
        run_profile_case(args.only)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
