#!/usr/bin/env python3
"""Benchmark of the B200 exact-attention forward (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fa2|reference] [--workload NAME]

A step is one call of the forward over the whole workload (one kernel launch).
The default workload is B=8, H=16, N=2048, d=128, causal, bf16 Q/K/V drawn
i.i.d. N(0,1) from seed 0, scale 1/sqrt(128) (16k tokens, hidden 2048).  The
metric is forward TFLOP/s with FLOP = 4*B*H*N^2*d, halved when causal.

N > 1 (launched with torch.distributed.run): every rank runs the same
workload on its own GPU, i.e. its own shard of N x B sequences; the heads are
independent, so there is no collective on the data path (weak scaling).  The
value is the FLOPs of all ranks divided by the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on this host's cores instead,
each step on a bounded sample of heads of the same workload (rank 0 only).

The headline is timed as ``--repeats`` regions of exactly K steps, each
bracketed by a barrier and a synchronisation; the value is from the median
region.  On one GPU the line also carries ``grid``: every point of the
16k-token sweep (N = 512 .. 16384, d = 64 and 128, causal off and on, H =
2048/d, B = 16384/N, plus Q, K x 4 at d = 128, N >= 4096), each timed with
CUDA events over at least 10 launches, with its fraction of the measured
bf16 peak, the median SM clock while it ran, its exponential floor and the
tensor-pipe utilisation from an ncu capture of the same kernel source
(``profiles/tensor_pipe.txt``, null when the source has changed since).
``--profile-grid`` launches every grid point once and nothing else (for that
ncu capture).  The line also carries ``backward`` (fa2_bwd on the headline
workload) and ``decode`` (the split-K/V entry point on one query against
16384 keys at d = 128 and against 4096 keys at d = 64), timed the same way.

Decode workloads (``--workload decode_...`` / ``chunk_...``: Nq queries at the
end of an Nk-long sequence) run the split-K/V entry point instead; a step is
one call (range kernel + merge kernel) and the metric is effective HBM GB/s:
the bytes of Q, K, V read once and O, LSE written once, over the step time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOP/s (bf16, N=512–16k, d=64/128) and % of B200 dense BF16 peak"
DEFAULT_WORKLOAD = "B8_H16_N2048_d128_causal"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0
# ex2.approx throughput measured on the B200: 16 per clock per SM (about
# 8 cycles per warp instruction per sub-partition).
EX2_PER_CLK_PER_SM = 16
BWD_METRIC = "attn bwd TFLOP/s (bf16, FLOP = 2.5 x forward FLOP) and % of B200 dense BF16 peak"
DECODE_METRIC = "split-K/V attn fwd effective HBM GB/s (Q,K,V read once, O,LSE written once)"
KERNEL_SOURCES = ["exact_tiled_attention_45_b200/csrc/fa2_fwd.cu", "exact_tiled_attention_45_b200/csrc/sm100_ptx.cuh",
                  "exact_tiled_attention_45_b200/csrc/fa2_splitkv.cuh", "exact_tiled_attention_45_b200/csrc/fa2_bwd.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fa2", choices=["fa2", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the timed oracle sample")
    ap.add_argument("--splits", type=int, default=0, help="key ranges for decode workloads (0 = library choice)")
    ap.add_argument("--no-gemm", action="store_true", help="skip the library GEMM comparator")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd"],
                    help="bwd: time the backward (dQ, dK, dV) instead of the forward")
    ap.add_argument("--repeats", type=int, default=15, help="bracketed K-step regions of the headline (median)")
    ap.add_argument("--region-gap-ms", type=float, default=20.0, help="idle gap before each headline region")
    ap.add_argument("--no-grid", action="store_true", help="skip the sweep over the 16k-token grid")
    ap.add_argument("--grid-ms", type=float, default=5.0, help="target length of each grid point's timed regions")
    ap.add_argument("--sustained-ms", type=float, default=1000.0,
                    help="length of the sustained run of each d=128, N>=4096 grid point (0: skip)")
    ap.add_argument("--profile-grid", action="store_true",
                    help="launch the forward once per grid point and exit (for an ncu capture)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, src_hash: str):
    """DRAM bytes per launch from an ncu capture of this exact kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and not line.startswith("#") and parts[0] == src_hash and parts[1] == workload:
                    return float(parts[2])
    except OSError:
        pass
    return None


def recorded_tensor_pipe(src_hash: str):
    """Per-workload ncu figures of this exact kernel source:
    {workload: {"tensor_pipe_pct": elapsed %, "tensor_pipe_active_pct": active %, "traffic": bytes}}."""
    path = os.path.join(ROOT, "profiles", "tensor_pipe.txt")
    out = {}
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 5 and not line.startswith("#") and parts[0] == src_hash:
                    out[parts[1]] = {"tensor_pipe_pct": float(parts[2]), "tensor_pipe_active_pct": float(parts[3]),
                                     "traffic": float(parts[4])}
    except OSError:
        pass
    return out


GRID_TOKENS = 16384
GRID_HIDDEN = 2048


def grid_points():
    """(name, B, H, N, d, causal, qk_mult) of the 16k-token sweep."""
    pts = []
    for d in (64, 128):
        for causal in (False, True):
            for N in (512, 1024, 2048, 4096, 8192, 16384):
                pts.append((f"grid_N{N}_d{d}_{'causal' if causal else 'full'}", GRID_TOKENS // N, GRID_HIDDEN // d,
                            N, d, causal, 1.0))
    for causal in (False, True):
        for N in (4096, 8192, 16384):
            pts.append((f"grid_N{N}_d128_{'causal' if causal else 'full'}_x4", GRID_TOKENS // N, GRID_HIDDEN // 128,
                        N, 128, causal, 4.0))
    return pts


class GridInputs:
    """Device copies of the sweep's inputs, drawn once per head dimension.

    Every grid point of one d holds 16384 x 2048 elements per tensor, and
    make_qkv(B, H, N, d) draws the same flat sequence for every such shape,
    so one draw per d (viewed as [B, H, N, d]) gives each point exactly the
    inputs make_qkv would."""

    def __init__(self, dev):
        self.dev, self.d, self.qkv, self.x4 = dev, None, None, None

    def get(self, B, H, N, d, qk_mult):
        import torch
        from exact_tiled_attention_45_b200.inputs import make_qkv
        if self.d != d:
            self.qkv = self.x4 = None
            torch.cuda.empty_cache()
            self.qkv = [t.to(self.dev) for t in make_qkv(1, 1, GRID_TOKENS * (GRID_HIDDEN // d), d, seed=0)]
            self.o = torch.empty_like(self.qkv[0])
            self.lse = torch.empty(GRID_TOKENS * (GRID_HIDDEN // d), dtype=torch.float32, device=self.dev)
            self.d = d
        src = self.qkv
        if qk_mult != 1.0:
            if self.x4 is None:
                self.x4 = [self.qkv[0] * 4, self.qkv[1] * 4]
            src = [self.x4[0], self.x4[1], self.qkv[2]]
        shp = (B, H, N, d)
        return [t.view(shp) for t in src], self.o.view(shp), self.lse.view(B, H, N)


def run_grid(dev, stream, sampler, peaks, target_ms: float, src: str, sustained_ms: float = 1000.0):
    """Time every sweep point; returns the ``grid`` object of the bench line.

    Burst timing, like the headline: after a short idle gap, 5 regions of at
    least 10 back-to-back launches (and at least ``target_ms``), median.  For
    the d = 128, N >= 4096 points also a sustained run of ``sustained_ms``
    of back-to-back launches, against the measured sustained bf16 peak (the
    1 kW power cap lowers the SM clock under long full load)."""
    import torch
    import exact_tiled_attention_45_b200 as fa2
    from exact_tiled_attention_45_b200.inputs import Workload
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    rec = recorded_tensor_pipe(src)
    inputs = GridInputs(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    points = {}
    for name, B, H, N, d, causal, mult in grid_points():
        w = Workload(name, B, H, N, d, causal, mult)
        (q, k, v), o, lse = inputs.get(B, H, N, d, mult)

        def call():
            fa2.fwd(q, k, v, causal=causal, out=o, lse=lse, stream=stream)

        for _ in range(3):
            call()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        call()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        est = max(ev0.elapsed_time(ev1), 1e-3)
        reps = max(10, int(math.ceil(target_ms / est)))
        time.sleep(0.25)
        region_ms, t_start = [], time.time()
        for _ in range(5):
            ev0.record(stream)
            for _ in range(reps):
                call()
            ev1.record(stream)
            torch.cuda.synchronize(dev)
            region_ms.append(ev0.elapsed_time(ev1) / reps)
        t_end = time.time()
        ms = sorted(region_ms)[2]
        mhz = sampler.median_between(t_start, t_end)
        sustained = None
        if sustained_ms > 0 and d == 128 and N >= 4096 and mult == 1.0:
            n_sus = max(10, int(math.ceil(sustained_ms / est)))
            ts0 = time.time()
            ev0.record(stream)
            for _ in range(n_sus):
                call()
            ev1.record(stream)
            torch.cuda.synchronize(dev)
            sus_ms = ev0.elapsed_time(ev1) / n_sus
            sus_tf = w.flops / (sus_ms * 1e-3) / 1e12
            peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
            sustained = {"ms": round(sus_ms, 5), "tflops": round(sus_tf, 1), "launches": n_sus,
                         "seconds": round(time.time() - ts0, 2),
                         "sm_mhz": sampler.median_between(ts0, time.time()),
                         "frac_of_sustained_peak": round(sus_tf / peak_sus, 4),
                         "frac_of_burst_peak": round(sus_tf / peak, 4)}
        sm_hz = float(mhz or peaks.get("sm_max_mhz", 1965.0)) * 1e6
        tflops = w.flops / (ms * 1e-3) / 1e12
        r = rec.get(name, {})
        points[name] = {
            "B": B, "H": H, "N": N, "d": d, "causal": causal, "qk_mult": mult,
            "ms": round(ms, 5), "tflops": round(tflops, 1), "frac": round(tflops / peak, 4),
            "launches": 5 * reps, "sm_mhz": mhz, "sustained": sustained,
            "exp_bound_pct": round(100.0 * w.exps / (EX2_PER_CLK_PER_SM * sms * sm_hz) / (ms * 1e-3), 1),
            "tensor_pipe_pct": r.get("tensor_pipe_pct"), "tensor_pipe_active_pct": r.get("tensor_pipe_active_pct"),
            "traffic": r.get("traffic"), "algorithmic_bytes": w.io_bytes,
        }
    fa2.sync_status(stream)
    del inputs
    torch.cuda.empty_cache()
    target = [p for n, p in points.items() if p["d"] == 128 and p["N"] >= 4096 and p["qk_mult"] == 1.0]
    return {
        "points": points,
        "timing": ("burst: after a 250 ms idle gap, median of 5 CUDA-event regions of >= 10 back-to-back launches "
                   "(>= grid-ms each; inputs 201 MB > L2); sustained (d=128, N>=4096): one region of "
                   "back-to-back launches for sustained-ms"),
        "peak": peak, "peak_source": "measured bf16 burst",
        "tensor_pipe_source": "ncu sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed, one launch per "
                              "point, profiles/tensor_pipe.txt (null unless captured on this kernel source)",
        "d128_N_ge_4k": {"min_frac": min(p["frac"] for p in target), "max_frac": max(p["frac"] for p in target),
                          "target_frac": 0.60, "met": all(p["frac"] >= 0.60 for p in target),
                          "sustained_min_frac_of_sustained_peak": min(
                              (p["sustained"]["frac_of_sustained_peak"] for p in target if p["sustained"]),
                              default=None)},
    }


def burst_time(call, dev, stream, target_ms: float, sampler):
    """Median per-launch ms of 5 CUDA-event regions of >= 10 back-to-back
    launches (>= target_ms each) after a 250 ms idle gap; with the median SM
    clock inside them."""
    import torch
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    call()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    reps = max(10, int(math.ceil(target_ms / max(ev0.elapsed_time(ev1), 1e-3))))
    time.sleep(0.25)
    region_ms, t0 = [], time.time()
    for _ in range(5):
        ev0.record(stream)
        for _ in range(reps):
            call()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        region_ms.append(ev0.elapsed_time(ev1) / reps)
    return sorted(region_ms)[2], 5 * reps, sampler.median_between(t0, time.time())


DECODE_LINE_WORKLOADS = ("decode_B8_H16_Nk16384_d128", "decode_B32_H16_Nk4096_d64")


def decode_lines(dev, stream, sampler, peaks, src, target_ms: float):
    """The split-K/V entry point on the decode workloads (effective HBM GB/s)."""
    import torch
    import exact_tiled_attention_45_b200 as fa2
    from exact_tiled_attention_45_b200.inputs import WORKLOADS
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    out = {}
    for name in DECODE_LINE_WORKLOADS:
        w = WORKLOADS[name]
        q, k, v = (t.to(dev) for t in workload_inputs(w, 0))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        splits = fa2.splitkv_splits(w.B, w.H, w.Nq, w.Nk, w.d, 0)
        need = fa2.splitkv_workspace_bytes(w.B, w.H, w.Nq, w.Nk, w.d, 0)
        ws = torch.empty(need, dtype=torch.uint8, device=dev) if need else None

        def call():
            fa2.fwd_splitkv(q, k, v, causal=w.causal, out=o, lse=lse, workspace=ws, stream=stream)

        ms, launches, mhz = burst_time(call, dev, stream, target_ms, sampler)
        fa2.sync_status(stream)
        gbs = w.bytes / (ms * 1e-3) / 1e9
        out[name] = {"GB_s": round(gbs, 1), "frac_of_copy_bw": round(gbs / hbm, 4), "ms": round(ms, 5),
                     "n_splits": splits, "launches": launches, "sm_mhz": mhz, "algorithmic_bytes": w.bytes,
                     "traffic": recorded_traffic(name, src)}
        del q, k, v, o, lse, ws
        torch.cuda.empty_cache()
    return out


def backward_line(w, q, k, v, q_host, dev, stream, sampler, peaks, src, target_ms: float):
    """The backward (fa2_bwd) on the headline workload, TFLOP/s by the 2.5 x
    forward-FLOP convention."""
    import torch
    import exact_tiled_attention_45_b200 as fa2
    g = torch.Generator(device="cpu")
    g.manual_seed(1000)
    do = torch.randn(q_host.shape, generator=g, dtype=torch.float32).to(torch.bfloat16).to(dev)
    o, lse = fa2.fwd(q, k, v, causal=w.causal, stream=stream)
    ws = torch.empty(fa2.bwd_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def call():
        fa2.bwd(q, k, v, o, lse, do, causal=w.causal, dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)

    ms, launches, mhz = burst_time(call, dev, stream, target_ms, sampler)
    fa2.sync_status(stream)
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tf = 2.5 * w.flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "tflops": round(tf, 1), "frac": round(tf / peak, 4), "ms": round(ms, 5),
            "executed_tflops": round((4.0 if w.d > 128 else 3.5) * w.flops / (ms * 1e-3) / 1e12, 1),
            "launches": launches, "sm_mhz": mhz, "traffic": recorded_traffic(w.name + ":bwd", src),
            "convention": "2.5 x forward FLOP (five matmuls); the kernels execute seven"}


def profile_grid():
    """One forward launch per grid point, nothing else (the ncu capture)."""
    import torch
    import exact_tiled_attention_45_b200 as fa2
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    inputs = GridInputs(dev)
    for name, B, H, N, d, causal, mult in grid_points():
        (q, k, v), o, lse = inputs.get(B, H, N, d, mult)
        fa2.fwd(q, k, v, causal=causal, out=o, lse=lse, stream=stream)
        fa2.sync_status(stream)
        print(name, flush=True)
    return 0


def max_over_ranks(x: float, device) -> float:
    """Maximum of a per-rank scalar over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank: float, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's step time."""
    return flops_per_rank * world / (max_ms_per_step * 1e-3) / 1e12


def shard_seed(rank: int) -> int:
    """Each rank draws its own shard of sequences."""
    return int(rank)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, torch_device):
        self.samples, self.stamps, self.reasons, self.max_mhz = [], [], 0, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _sample(self):
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            self.stamps.append(time.time())
            self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
        except Exception:
            pass

    def median_between(self, t0: float, t1: float):
        """Median SM clock of the samples taken between two wall-clock times."""
        s = sorted(m for m, t in zip(list(self.samples), list(self.stamps)) if t0 <= t <= t1)
        return s[len(s) // 2] if s else None

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.005)

    def start(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self, windows=None):
        """Median SM clock and throttle reasons; with `windows` (pairs of wall
        times) only the samples taken inside them count for the median."""
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        s = sorted(self.samples)
        if windows:
            inside = sorted(m for m, t in zip(list(self.samples), list(self.stamps))
                            if any(a <= t <= b for a, b in windows))
            if inside:
                s = inside
        med = s[len(s) // 2] if s else None
        names = [k for k, bit in self.REASONS.items() if self.reasons & bit and k != "gpu_idle"]
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(s)}


def cpu_oracle_sample(w, budget_s: float, q, k, v):
    """Time the fp64 oracle on whole heads of the workload until the budget is spent."""
    import numpy as np
    import torch
    from oracle import attention_ref
    cores = torch.get_num_threads()
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    done, flops, t0 = 0, 0.0, time.perf_counter()
    per_head = w.flops / (w.B * w.H)
    for b, h in heads:
        attention_ref(q[b:b + 1, h:h + 1].double().numpy(), k[b:b + 1, h:h + 1].double().numpy(),
                      v[b:b + 1, h:h + 1].double().numpy(), causal=w.causal, scale=w.d ** -0.5)
        done += 1
        flops += per_head
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(cores), "kind": "oracle",
            "sample": f"{done} of {len(heads)} heads of {w.name} (fp64 NumPy, {dt:.1f} s)",
            "seconds": round(dt, 2)}, np


def is_decode(w) -> bool:
    return hasattr(w, "Nq")


def oracle_head(w, q, k, v, b, h):
    """The fp64 oracle on head (b, h) of the workload."""
    from oracle import attention_ref, attention_ref_rect
    fn = attention_ref_rect if is_decode(w) else attention_ref
    return fn(q[b:b + 1, h:h + 1].double().numpy(), k[b:b + 1, h:h + 1].double().numpy(),
              v[b:b + 1, h:h + 1].double().numpy(), causal=w.causal, scale=w.d ** -0.5)


def workload_inputs(w, seed):
    from exact_tiled_attention_45_b200.inputs import make_q_kv, make_qkv
    if is_decode(w):
        return make_q_kv(w.B, w.H, w.Nq, w.Nk, w.d, seed=seed, qk_mult=w.qk_mult)
    return make_qkv(w.B, w.H, w.N, w.d, seed=seed, qk_mult=w.qk_mult)


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import torch
    heads_per_step = 1
    q, k, v = workload_inputs(w, 0)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    bwd_pass = (not is_decode(w)) and args.pass_ == "bwd"
    if bwd_pass:
        from oracle import attention_bwd_ref
        g = torch.Generator(device="cpu")
        g.manual_seed(1000)
        do = torch.randn(q.shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
        per_head, unit, metric, scale_u = 2.5 * w.flops / (w.B * w.H), "TFLOP/s", BWD_METRIC, 1e12
    elif is_decode(w):
        per_head, unit, metric, scale_u = w.bytes / (w.B * w.H), "GB/s", DECODE_METRIC, 1e9
        heads_per_step = 16
    else:
        per_head, unit, metric, scale_u = w.flops / (w.B * w.H), "TFLOP/s", METRIC, 1e12

    def step(i):
        for t in range(heads_per_step):
            b, h = heads[(i * heads_per_step + t) % len(heads)]
            if bwd_pass:
                sl = (slice(b, b + 1), slice(h, h + 1))
                attention_bwd_ref(q[sl].double().numpy(), k[sl].double().numpy(), v[sl].double().numpy(),
                                  do[sl].double().numpy(), causal=w.causal, scale=w.d ** -0.5)
            else:
                oracle_head(w, q, k, v, b, h)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = per_head * heads_per_step * args.steps / dt / scale_u
    cores = torch.get_num_threads()
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(w.as_dict(), sample=f"{heads_per_step} head(s) of {w.B * w.H} per step"),
        "cpu_baseline": {"value": value, "unit": unit, "cores": int(cores), "kind": "oracle",
                         "sample": f"{heads_per_step} head(s) per step of {w.name}, fp64 NumPy on host cores"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def gemm_comparator(w, dev, reps: int = 20) -> dict:
    """Library bf16 GEMMs on the same GPU, beside the attention kernel.

    The pages put FlashAttention-2 "close to" GEMM efficiency; this measures
    what the vendor GEMM reaches here: a square 8192^3 matmul, and the two
    batched GEMMs of unfused attention at the workload's shapes
    (S = Q K^T, then O = P V, each over all B*H heads, with no softmax and
    no masking: 4*B*H*N^2*d FLOP).  Timed with CUDA events after warm-up.
    """
    import torch

    def timed(fn, flops):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        return flops * reps / (e0.elapsed_time(e1) * 1e-3) / 1e12

    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randn(8192, 8192, device=dev, dtype=torch.bfloat16, generator=g)
    b = torch.randn(8192, 8192, device=dev, dtype=torch.bfloat16, generator=g)
    out = {"square_8192_tflops": timed(lambda: a @ b, 2.0 * 8192 ** 3)}
    del a, b
    bh = w.B * w.H
    q = torch.randn(bh, w.N, w.d, device=dev, dtype=torch.bfloat16, generator=g)
    k = torch.randn(bh, w.N, w.d, device=dev, dtype=torch.bfloat16, generator=g)
    s = torch.empty(bh, w.N, w.N, device=dev, dtype=torch.bfloat16)
    o = torch.empty(bh, w.N, w.d, device=dev, dtype=torch.bfloat16)

    def unfused():
        torch.bmm(q, k.transpose(1, 2), out=s)
        torch.bmm(s, k, out=o)

    out["bmm_qk_pv_tflops"] = timed(unfused, 4.0 * bh * w.N * w.N * w.d)
    out["bmm_bytes_of_scores"] = bh * w.N * w.N * 2
    out["library"] = "torch.matmul / torch.bmm (cuBLAS), bf16 in, bf16 out, fp32 accumulation"
    del q, k, s, o
    torch.cuda.empty_cache()
    return out


def run_backward(args, w):
    """The backward (fa2_bwd: two kernels, three at d = 256) on the workload;
    TFLOP/s by the usual convention of 2.5 x the forward FLOP (five matmuls;
    the kernels execute seven, eight at d = 256, since dQ is computed without
    atomics)."""
    import torch
    import torch.distributed as dist
    import exact_tiled_attention_45_b200 as fa2

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    q_h, k_h, v_h = workload_inputs(w, shard_seed(rank))
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 + shard_seed(rank))
    do_h = torch.randn(q_h.shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    o, lse = fa2.fwd(q, k, v, causal=w.causal, stream=stream)
    ws = torch.empty(fa2.bwd_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    in_bytes = 5 * q.numel() * 2 + lse.numel() * 4
    out_bytes = 3 * q.numel() * 2
    flops = 2.5 * w.flops
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev) if in_bytes <= l2_bytes else None

    def call():
        fa2.bwd(q, k, v, o, lse, do, causal=w.causal, dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        call()
    fa2.sync_status(stream)
    sampler = ClockSampler(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    total_ms = 0.0
    if flush is None:
        ev0.record(stream)
        for _ in range(args.steps):
            call()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        total_ms = ev0.elapsed_time(ev1)
    else:
        for _ in range(args.steps):
            flush.zero_()
            ev0.record(stream)
            call()
            ev1.record(stream)
            ev1.synchronize()
            total_ms += ev0.elapsed_time(ev1)
    sampler.stop()
    barrier()
    fa2.sync_status(stream)
    step_ms = total_ms / args.steps
    max_ms = max_over_ranks(total_ms, dev) / args.steps
    value = flops * world / (max_ms * 1e-3) / 1e12

    e2e = None
    if not args.no_e2e:
        pinned = [t.pin_memory() for t in (q_h, k_h, v_h, do_h)]
        o_h, lse_h = o.cpu().pin_memory(), lse.cpu().pin_memory()
        outs = [torch.empty_like(q_h).pin_memory() for _ in range(3)]
        e2e_steps = max(3, min(args.steps, 10))

        def e2e_step():
            with torch.cuda.stream(stream):
                for dst, src in zip((q, k, v, do), pinned):
                    dst.copy_(src, non_blocking=True)
                o.copy_(o_h, non_blocking=True)
                lse.copy_(lse_h, non_blocking=True)
                call()
                for dst, src in zip(outs, (dq, dk, dv)):
                    dst.copy_(src, non_blocking=True)

        e2e_step()
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), dev) / e2e_steps
        e2e = {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes, "steps": e2e_steps,
               "path": "torch pinned copies + fa2.bwd on one stream"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (step_ms * 1e-3) / 1e12
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        from oracle import attention_bwd_ref
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        done, t0 = 0, time.perf_counter()
        for b, h in heads:
            sl = (slice(b, b + 1), slice(h, h + 1))
            attention_bwd_ref(q_h[sl].double().numpy(), k_h[sl].double().numpy(), v_h[sl].double().numpy(),
                              do_h[sl].double().numpy(), causal=w.causal, scale=w.d ** -0.5)
            done += 1
            if time.perf_counter() - t0 >= args.cpu_seconds:
                break
        dt = time.perf_counter() - t0
        cpu = {"value": flops / (w.B * w.H) * done / dt / 1e12, "unit": "TFLOP/s", "cores": torch.get_num_threads(),
               "kind": "oracle", "sample": f"{done} of {len(heads)} heads of {w.name}, backward (fp64 NumPy, {dt:.1f} s)"}
    line = {
        "metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(w.as_dict(), seed="rank", scale=f"1/sqrt({w.d})", pass_="bwd",
                       l2=("inputs larger than L2" if flush is None else "L2 flushed before every step"),
                       parallelism=("single GPU" if world == 1 else f"{world} ranks, independent heads, no collective")),
        # MMAs per tile pair: 7 (S and dP in both kernels), 8 at d = 256 (S^T in both dK/dV passes)
        "executed_tflops": (4.0 if w.d > 128 else 3.5) * w.flops / (step_ms * 1e-3) / 1e12,
        "pct_of_peak": {"measured_burst": 100.0 * achieved / peak, "peaks": peak_kind},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(w.name + ":bwd", source_hash()),
                     "peak_source": f"{peak_kind} bf16 burst",
                     "kernel": "fa2_bwd_dq_kernel + fa2_bwd_dkdv_kernel (one step, both timed)",
                     "src": source_hash()},
        "clocks": sampler.summary(),
        "gpu_launches": 2 * args.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_decode(args, w):
    """Split-K/V entry point on a decode workload; effective HBM GB/s."""
    import torch
    import torch.distributed as dist
    import exact_tiled_attention_45_b200 as fa2

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    q_h, k_h, v_h = workload_inputs(w, shard_seed(rank))
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    splits = fa2.splitkv_splits(w.B, w.H, w.Nq, w.Nk, w.d, args.splits)
    ws_bytes = fa2.splitkv_workspace_bytes(w.B, w.H, w.Nq, w.Nk, w.d, args.splits)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    in_bytes = (q.numel() + k.numel() + v.numel()) * 2
    out_bytes = o.numel() * 2 + lse.numel() * 4
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev) if in_bytes <= l2_bytes else None

    def call():
        fa2.fwd_splitkv(q, k, v, causal=w.causal, n_splits=args.splits, out=o, lse=lse, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        call()
    fa2.sync_status(stream)
    sampler = ClockSampler(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    if flush is None:
        ev0.record(stream)
        for _ in range(args.steps):
            call()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        total_ms = ev0.elapsed_time(ev1)
    else:
        total_ms = 0.0
        for _ in range(args.steps):
            flush.zero_()
            ev0.record(stream)
            call()
            ev1.record(stream)
            ev1.synchronize()
            total_ms += ev0.elapsed_time(ev1)
    sampler.stop()
    barrier()
    fa2.sync_status(stream)
    step_ms = total_ms / args.steps
    max_ms = max_over_ranks(total_ms, dev) / args.steps
    value = w.bytes * world / (max_ms * 1e-3) / 1e9

    # End to end: pinned host Q, K, V copied in, the call, O and LSE copied
    # back, all on the stream inside the timed region.
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        op = torch.empty_like(qp).pin_memory()
        lp = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32).pin_memory()
        e2e_steps = max(3, min(args.steps, 10))

        def e2e_step():
            with torch.cuda.stream(stream):
                q.copy_(qp, non_blocking=True)
                k.copy_(kp, non_blocking=True)
                v.copy_(vp, non_blocking=True)
                call()
                op.copy_(o, non_blocking=True)
                lp.copy_(lse, non_blocking=True)

        e2e_step()
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), dev) / e2e_steps
        e2e = {"value": w.bytes * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes, "steps": e2e_steps,
               "path": "torch pinned copies + fwd_splitkv on one stream"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # A long chunk of queries is a contraction again: above the ridge point
    # (FLOP per byte = peak FLOP/s / peak B/s) the tensor roofline applies.
    if w.flops / w.bytes > tf * 1e12 / (hbm * 1e9):
        roof = {"bound": "tensor", "achieved": w.flops / (step_ms * 1e-3) / 1e12, "peak": tf, "unit": "TFLOP/s",
                "peak_source": f"{peak_kind} bf16 burst"}
    else:
        roof = {"bound": "hbm", "achieved": w.bytes / (step_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                "peak_source": f"{peak_kind} copy bandwidth"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        import numpy as np  # noqa: F401
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        done, t0 = 0, time.perf_counter()
        for b, h in heads:
            oracle_head(w, q_h, k_h, v_h, b, h)
            done += 1
            if time.perf_counter() - t0 >= args.cpu_seconds:
                break
        dt = time.perf_counter() - t0
        cpu = {"value": w.bytes / (w.B * w.H) * done / dt / 1e9, "unit": "GB/s", "cores": torch.get_num_threads(),
               "kind": "oracle", "sample": f"{done} of {len(heads)} heads of {w.name} (fp64 NumPy, {dt:.1f} s)"}
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(w.as_dict(), seed="rank", scale=f"1/sqrt({w.d})", n_splits=splits,
                       l2=("inputs larger than L2" if flush is None else "L2 flushed before every step"),
                       parallelism=("single GPU" if world == 1 else f"{world} ranks, independent heads, no collective")),
        "tflops": w.flops / (step_ms * 1e-3) / 1e12,
        "roofline": dict(roof, traffic=recorded_traffic(w.name, source_hash()),
                         kernel=("fa2_splitkv_kernel (one range, no merge)" if splits == 1 else
                                 "fa2_splitkv_kernel + fa2_splitkv_combine_kernel (one step, both timed)"),
                         src=source_hash()),
        "clocks": sampler.summary(),
        "gpu_launches": (1 if splits == 1 else 2) * args.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    from exact_tiled_attention_45_b200.inputs import WORKLOADS
    if args.workload not in WORKLOADS:
        raise SystemExit(f"unknown workload {args.workload}; choose from {sorted(WORKLOADS)}")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.profile_grid:
        return profile_grid()
    if args.steps < 1 or args.warmup < 3 or args.repeats < 1:
        raise SystemExit("need --steps >= 1, --warmup >= 3 and --repeats >= 1")
    if is_decode(w):
        return run_decode(args, w)
    if args.pass_ == "bwd":
        return run_backward(args, w)

    import torch
    import torch.distributed as dist
    import exact_tiled_attention_45_b200 as fa2
    from exact_tiled_attention_45_b200.inputs import make_qkv

    world, rank, local = dist_env()
    if args.steps < 1 or args.warmup < 3:
        raise SystemExit("need --steps >= 1 and --warmup >= 3")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    # Each rank draws its own shard of sequences (seed = rank) and keeps it resident.
    q_h, k_h, v_h = make_qkv(w.B, w.H, w.N, w.d, seed=shard_seed(rank), qk_mult=w.qk_mult)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    in_bytes = 3 * q.numel() * 2
    out_bytes = o.numel() * 2 + lse.numel() * 4
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = None
    if in_bytes <= l2_bytes:
        flush = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev)

    def step():
        if flush is not None:
            flush.zero_()
        fa2.fwd(q, k, v, causal=w.causal, out=o, lse=lse, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    fa2.sync_status(stream)

    sampler = ClockSampler(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.start()
    # `repeats` regions of exactly K steps, each bracketed by a barrier and a
    # synchronisation on both sides; the value comes from the median region.
    # A short idle gap before each region makes every region one burst of K
    # steps (back-to-back regions would add up to a sustained load, which the
    # power cap throttles; the sweep below reports sustained figures too).
    region_ms, windows = [], []
    for _ in range(args.repeats):
        time.sleep(args.region_gap_ms * 1e-3)
        barrier()
        torch.cuda.synchronize(dev)
        t_win = time.time()
        if flush is None:
            ev0.record(stream)
            for _ in range(args.steps):
                step()
            ev1.record(stream)
            torch.cuda.synchronize(dev)
            region_ms.append(ev0.elapsed_time(ev1))
        else:
            # L2 is flushed before every step; only the kernels are timed.
            t = 0.0
            for _ in range(args.steps):
                flush.zero_()
                ev0.record(stream)
                fa2.fwd(q, k, v, causal=w.causal, out=o, lse=lse, stream=stream)
                ev1.record(stream)
                ev1.synchronize()
                t += ev0.elapsed_time(ev1)
            region_ms.append(t)
        windows.append((t_win, time.time()))
        barrier()
    sampler.stop()
    fa2.sync_status(stream)
    total_ms = sorted(region_ms)[len(region_ms) // 2]
    kernel_ms = total_ms / args.steps

    max_ms = max_over_ranks(total_ms, dev)
    ms_per_step = max_ms / args.steps
    total_flops = w.flops * world
    value = aggregate_tflops(w.flops, world, ms_per_step)

    # Per-launch distribution, from a second pass of the same launches with
    # an event pair around each (outside the bracketed timing above).
    step_times = []
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in pairs:
        if flush is not None:
            flush.zero_()
        a.record(stream)
        fa2.fwd(q, k, v, causal=w.causal, out=o, lse=lse, stream=stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    step_times = sorted(a.elapsed_time(b) for a, b in pairs)
    fa2.sync_status(stream)

    # End to end through the host-buffer entry point: pinned host inputs in,
    # host outputs back, copies inside the timed region.
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        op = torch.empty_like(qp).pin_memory()
        lp = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
        ws = torch.empty(fa2.workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
        e2e_steps = max(3, min(args.steps, 10))
        for _ in range(2):
            fa2.fwd_host(qp, kp, vp, causal=w.causal, out=op, lse=lp, workspace=ws, stream=stream)
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(e2e_steps):
            fa2.fwd_host(qp, kp, vp, causal=w.causal, out=op, lse=lp, workspace=ws, stream=stream)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), dev) / e2e_steps
        e2e = {"value": aggregate_tflops(w.flops, world, e2e_ms), "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes, "steps": e2e_steps}
        del qp, kp, vp, op, lp, ws

    peaks, peak_kind = load_peaks()
    src = source_hash()
    grid = decode = backward = None
    if not args.no_grid and world == 1:
        xsampler = ClockSampler(dev)
        xsampler.start()
        backward = backward_line(w, q, k, v, q_h, dev, stream, xsampler, peaks, src, args.grid_ms)
        del q, k, v, o, lse
        torch.cuda.empty_cache()
        decode = decode_lines(dev, stream, xsampler, peaks, src, args.grid_ms)
        xsampler.stop()
        torch.cuda.empty_cache()
        gsampler = ClockSampler(dev)
        gsampler.start()
        grid = run_grid(dev, stream, gsampler, peaks, args.grid_ms, src, args.sustained_ms)
        gsampler.stop()
        grid["clocks"] = gsampler.summary()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = w.flops / (kernel_ms * 1e-3) / 1e12
    traffic = recorded_traffic(w.name, src)

    def pct(p):
        return step_times[min(len(step_times) - 1, int(round(p / 100.0 * (len(step_times) - 1))))]

    clocks = sampler.summary(windows)
    clocks["basis"] = "samples inside the timed regions"
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    sm_hz = float(clocks.get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)) * 1e6
    exp_ms = w.exps / (EX2_PER_CLK_PER_SM * sms * sm_hz) * 1e3
    floors = {
        "hbm_ms": w.io_bytes / (hbm * 1e9) * 1e3, "hbm_bytes": w.io_bytes,
        "tensor_ms": w.flops / (peak * 1e12) * 1e3,
        "exp_ms": exp_ms, "exps": w.exps,
        "exp_basis": f"{EX2_PER_CLK_PER_SM} ex2/clk/SM x {sms} SMs x median SM clock (all exponentials on the MUFU)",
        "exp_bound_pct": 100.0 * exp_ms / kernel_ms,
    }
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu, _ = cpu_oracle_sample(w, args.cpu_seconds, q_h, k_h, v_h)
    gemm = None
    if not args.no_gemm and world == 1:
        gemm = gemm_comparator(w, dev)
        gemm["fa2_over_square_gemm"] = achieved / gemm["square_8192_tflops"]

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(w.as_dict(), seed="rank", scale=f"1/sqrt({w.d})",
                       l2=("inputs larger than L2" if flush is None else "L2 flushed before every step"),
                       parallelism=("single GPU" if world == 1 else f"{world} ranks, independent heads, no collective")),
        "pct_of_peak": {"measured_burst": 100.0 * achieved / peak, "measured_sustained": 100.0 * achieved / peak_sus,
                        "spec_2250": 100.0 * achieved / SPEC_BF16_TFLOPS, "peaks": peak_kind},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": f"{peak_kind} bf16 burst",
                     "kernel": "fa2_fwd_kernel", "src": src,
                     "tensor_pipe_pct": recorded_tensor_pipe(src).get(w.name, {}).get("tensor_pipe_pct")},
        "step_ms": {"median": pct(50), "p10": pct(10), "p90": pct(90), "n": len(step_times),
                    "pass": "second pass, one event pair per launch"},
        "regions_ms": [round(x, 4) for x in region_ms], "repeats": args.repeats,
        "floors": floors,
        "clocks": clocks,
        "gpu_launches": args.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gemm_comparator": gemm,
        "grid": grid,
        "backward": backward,
        "decode": decode,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
