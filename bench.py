#!/usr/bin/env python
"""Benchmark: device-timed attention forward on B200, one JSON line.

A step is one call of ``vitattn_forward`` over one batch of the workload:
the whole path (Q.K^T, online softmax, P.V, epilogue) in one kernel launch.
For a ragged multi-image workload (``--workload multi_image``) a step is one
call of ``vitattn_forward_varlen`` over the packed batch, and the flops are
4*H*D*sum(n_s^2) over its images.  For the prologue workload
(``--workload rope_batched``) a step is one ``vitattn_qkv_rope`` call (packed
QKV split + 2-D rope), and for ``rope_norm_batched`` one
``vitattn_qkv_norm_rope`` call (the same with a per-head q/k RMS norm first);
the metric is the algorithmic bytes per second against the measured HBM copy
bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

* ``value``: 4*B*H*N^2*D flops per step x steps x ranks / device time of the
  timed region (CUDA events on the launching stream, max over ranks), TFLOP/s.
* ``e2e``: the same metric through the host-buffer entry point
  ``vitattn_forward_host`` (pinned host -> device copies of q, k, v, the
  kernel, device -> host copy of out, all inside the timed region); for a
  ragged workload through the Python entry ``forward_varlen`` with the same
  copies issued on the same stream.
* ``roofline``: the kernel against the measured dense bf16 tensor peak.
* ``cpu_baseline``: the fp64 oracle on this host's cores, on a bounded sample
  of output rows of the same workload, scaled to the same metric.

With ``--gpus N`` (under torchrun) every rank runs the full workload on its
own GPU with no collective on the data path (the (b, h) units are
independent): weak scaling; ranks only meet for barriers and the max of the
timings.
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

import numpy as np  # noqa: E402

from vit_bidirectional_attention_b200 import ranks, synth  # noqa: E402

DEFAULT_WORKLOAD = "high_res"
METRIC = "attention fwd TFLOP/s (4·B·H·N²·D) and % of B200 dense BF16 tensor peak"
L2_BYTES = 126 * 1024 * 1024
L2_FLUSH_BYTES = 256 * 1024 * 1024  # written before each timed launch when the inputs fit in L2
FALLBACK_PEAK_TFLOPS = 1590.0  # the pool's earlier measurement, used only without MEASURED_PEAKS.json
DATASHEET_PEAK_TFLOPS = 2250.0
# the device sources each kernel is compiled from (its own file and what it includes)
_CSRC = "vit_bidirectional_attention_b200/csrc/"
KERNEL_SOURCES = {
    "fwd_kernel": [_CSRC + "fwd_kernel.cuh", _CSRC + "ptx.cuh"],
    "qkv_rope_kernel": [_CSRC + "rope_kernel.cuh"],
    "qkv_norm_rope_kernel": [_CSRC + "rope_kernel.cuh", _CSRC + "norm_rope_kernel.cuh"],
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for about 2 s of timed work)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(synth.WORKLOADS) + sorted(synth.RAGGED) + sorted(synth.PROLOGUE) + sorted(synth.LAYER))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def cpu_model() -> str:
    """The host CPU's model name (first entry of /proc/cpuinfo), for the CPU baseline."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def timed_launches(step, steps: int, stream, event_cls, flush=None, per_launch=None) -> float:
    """Device milliseconds of ``steps`` launches of ``step`` on ``stream``.

    Without ``flush``: one event pair around the back-to-back launches.  With
    ``flush`` (a callable that writes more than the L2's capacity on the same
    stream), the flush runs before every launch and only the launches are
    timed, each between its own pair of events; their sum is returned, and
    each launch's milliseconds are appended to ``per_launch`` if it is a list."""
    if flush is None:
        ev0, ev1 = event_cls(enable_timing=True), event_cls(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        ev1.synchronize()
        return ev0.elapsed_time(ev1)
    pairs = [(event_cls(enable_timing=True), event_cls(enable_timing=True)) for _ in range(steps)]
    for a, b in pairs:
        flush()
        a.record(stream)
        step()
        b.record(stream)
    pairs[-1][1].synchronize()
    times = [a.elapsed_time(b) for a, b in pairs]
    if per_launch is not None:
        per_launch.extend(times)
    return sum(times)


def kernel_of(workload: str) -> str:
    """The kernel a workload's step launches."""
    if workload in synth.PROLOGUE:
        return "qkv_norm_rope_kernel" if synth.PROLOGUE[workload].qk_norm else "qkv_rope_kernel"
    return "fwd_kernel"


def kernel_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "MEASURED_PEAKS.json"
    return None, "fallback"


def committed_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        data = json.load(f)
    entry = data.get(workload)
    if not entry or entry.get("kernel_hash") != kernel_hash(kernel_of(workload)):
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""

    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t_start = self.t_stop = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        import datetime

        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[1], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append({"t": ts, "sm": float(parts[2]), "max": float(parts[3]),
                             "reasons": parts[5:10]})
            except ValueError:
                continue
        window = "timed region"
        inside = [r for r in rows if self.t_start is not None and self.t_start <= r["t"] <= self.t_stop]
        if not inside:
            # timed region shorter than the sampling period: the samples
            # around it (warm-up and timed steps back to back) stand in
            inside, window = rows, "warm-up + timed region"
        if not inside:
            return None
        loaded = inside
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        active = set()
        for r in loaded:
            for n, flag in zip(names, r["reasons"][1:]):
                if flag.lower() == "active":
                    active.add(n)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in loaded),
                "reasons": sorted(active), "samples": len(loaded), "window": window}


def oracle_rows(w, q, k, v, rows):
    """The oracle on sampled output rows; returns the flops those rows cost."""
    import oracle

    if isinstance(w, synth.Workload) and w.causal:
        # the oracle's causal form on whole (b, h) slices: rows -> their (b, h), each computed once
        H = w.H
        bh = sorted({(int(r) // H // w.N, int(r) % H) for r in rows})
        for b, h in bh:
            oracle.attention_ext(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1], w.scale,
                                 w.dtype, causal=True)
        return 4.0 * w.D * w.N * (w.N + 1) / 2 * len(bh)
    if isinstance(w, synth.Workload) and w.Hkv:
        g = w.H // w.Hkv
        oracle.attention_rows(q, np.repeat(k, g, axis=2), np.repeat(v, g, axis=2), w.scale, w.dtype, rows)
        return 4.0 * w.N * w.D * len(rows)
    if isinstance(w, synth.RaggedWorkload):
        oracle.attention_varlen_rows(q, k, v, w.cu_seqlens, w.scale, w.dtype, rows)
        seg_len = np.diff(np.asarray(w.cu_seqlens))
        tok_seg = np.repeat(np.arange(len(seg_len)), seg_len)
        return float(4.0 * w.D * seg_len[tok_seg[np.asarray(rows) // w.H]].sum())
    oracle.attention_rows(q, k, v, w.scale, w.dtype, rows)
    return 4.0 * w.N * w.D * len(rows)


def total_rows_of(w):
    return (w.total if isinstance(w, synth.RaggedWorkload) else w.B * w.N) * w.H


def sample_rows_of(w, count, seed):
    if isinstance(w, synth.RaggedWorkload):
        return synth.sample_rows((1, w.total, w.H), count, seed)
    return synth.sample_rows(w, count, seed)


def cpu_baseline(w, q, k, v, seconds: float):
    """The fp64 oracle, as it stands, on a bounded sample of output rows."""
    import oracle

    total_rows = total_rows_of(w)
    n = min(64, total_rows)
    for attempt in range(6):
        rows = sample_rows_of(w, n, seed=w.seed + 11 + attempt)
        t0 = time.perf_counter()
        flops = oracle_rows(w, q, k, v, rows)
        dt = time.perf_counter() - t0
        if dt >= 0.8 * seconds or len(rows) >= total_rows:
            break
        n = int(min(total_rows, max(2 * n, 1.05 * len(rows) * seconds / max(dt, 1e-6))))
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"{len(rows)} of {total_rows} output rows (seeded), fp64, "
                      f"{dt:.1f} s on {oracle.num_threads()} threads"}


def dist_setup(args):
    import torch

    world, rank, local = ranks.env_world()
    if world > 1:
        torch.cuda.set_device(local)
        ranks.init("nccl", world, device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    ranks.barrier(world)


def max_over_ranks(x: float, world: int) -> float:
    return ranks.max_over_ranks(x, world, device="cuda")


def load_workload(name):
    """(workload, q, k, v): dense [B, N, H, D] or ragged [total, H, D] bit arrays."""
    if name in synth.RAGGED:
        w = synth.RAGGED[name]
        return (w,) + tuple(synth.make_qkv_ragged(w))
    w = synth.WORKLOADS[name]
    return (w,) + tuple(synth.make_qkv(w))


def shape_config(w):
    if isinstance(w, synth.RaggedWorkload):
        return {"images": len(w.seqlens), "seqlens": list(w.seqlens), "total_tokens": w.total,
                "H": w.H, "D": w.D}
    cfg = {"B": w.B, "N": w.N, "H": w.H, "D": w.D}
    if w.Hkv:
        cfg["Hkv"] = w.Hkv
    if w.causal:
        cfg["causal"] = "aligned (query i sees keys j <= i), with the f32 LSE output; flops count N(N+1)/2 pairs"
    return cfg


def run_reference(args):
    """The oracle as the reference arm: bounded samples on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle

    w, q, k, v = load_workload(args.workload)
    if args.steps is None:
        args.steps = 5
    total_rows = total_rows_of(w)
    per_step = max(1.0, min(2.0, 120.0 / max(1, args.steps + args.warmup)))
    rows_probe = sample_rows_of(w, min(64, total_rows), seed=w.seed + 17)
    t0 = time.perf_counter()
    oracle_rows(w, q, k, v, rows_probe)
    t_probe = max(time.perf_counter() - t0, 1e-6)
    n_rows = int(min(total_rows, max(32, len(rows_probe) * per_step / t_probe)))
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        rows = sample_rows_of(w, n_rows, seed=w.seed + 1000 + i)
        t0 = time.perf_counter()
        f = oracle_rows(w, q, k, v, rows)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
            flops.append(f)
    step_s = sum(times) / len(times)
    value = sum(flops) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(shape_config(w), workload=args.workload, input_dtype=synth.DTYPE_NAMES[w.dtype],
                       scale=w.scale, sample_rows_per_step=n_rows),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "cpu_model": cpu_model(),
                         "kind": "oracle",
                         "sample": f"{n_rows} of {total_rows} output rows per step (seeded)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


PROLOGUE_METRIC = "qkv split + 2-D rope prologue GB/s (algorithmic bytes / device time) and % of measured HBM copy bandwidth"
PROLOGUE_NORM_METRIC = ("qkv split + q/k RMS norm + 2-D rope prologue GB/s (algorithmic bytes / device time) and % of "
                        "measured HBM copy bandwidth")


def run_prologue(args):
    """The prologue workload: one vitattn_qkv_rope (or, with the q/k norm,
    vitattn_qkv_norm_rope) call per step."""
    w = synth.PROLOGUE[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    qkv, cs, sn = synth.make_prologue(w)
    qw, kw = synth.make_norm_weights(w.D, w.seed + 1000) if w.qk_norm else (None, None)
    metric = PROLOGUE_NORM_METRIC if w.qk_norm else PROLOGUE_METRIC
    entry = "vitattn_qkv_norm_rope" if w.qk_norm else "vitattn_qkv_rope"

    def cpu_leg(seconds, steps=1):
        # the oracle on a bounded, seeded sample of tokens; bytes scaled per token
        import oracle

        per_token = w.io_bytes / w.T
        n, dt = 64, 0.0
        for attempt in range(8):
            idx = np.random.Generator(np.random.PCG64(w.seed + attempt)).choice(w.T, min(n, w.T), replace=False)
            t0 = time.perf_counter()
            for _ in range(steps):
                if w.qk_norm:
                    oracle.qkv_norm_rope(qkv[idx], cs[idx], sn[idx], qw, kw, w.eps, w.dtype)
                else:
                    oracle.qkv_rope(qkv[idx], cs[idx], sn[idx], w.dtype)
            dt = (time.perf_counter() - t0) / steps
            if dt >= 0.5 * seconds or n >= w.T:
                break
            n = int(min(w.T, max(2 * n, n * seconds / max(dt, 1e-6))))
        return per_token * len(idx) / dt / 1e9, len(idx), dt

    peaks, _ = measured_peaks()
    peak = float(peaks["hbm_gbs"]) if peaks else 6650.0
    if args.impl == "reference":
        if rank != 0:
            return 0
        import oracle

        value, n, dt = cpu_leg(2.0, steps=max(1, args.steps or 1))
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world,
                "steps": args.steps or 1, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, "tokens": w.T, "H": w.H, "D": w.D, "sample_tokens": n},
                "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "cpu_model": cpu_model(), "kind": "oracle",
                                 "sample": f"{n} of {w.T} tokens (seeded), numpy fp64"},
                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch

    from vit_bidirectional_attention_b200 import vitattn

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local if world > 1 else 0)
    tdt = torch.bfloat16 if w.dtype == synth.BF16 else torch.float16
    hqkv = torch.from_numpy(qkv.view(np.int16).copy()).view(tdt)
    hcs, hsn = torch.from_numpy(cs), torch.from_numpy(sn)
    dqkv, dcs, dsn = (x.to(dev) for x in (hqkv, hcs, hsn))
    hqw, hkw = (torch.from_numpy(x) for x in (qw, kw)) if w.qk_norm else (None, None)
    dqw, dkw = (hqw.to(dev), hkw.to(dev)) if w.qk_norm else (None, None)
    q, k, v = (torch.empty((w.T, w.H, w.D), dtype=tdt, device=dev) for _ in range(3))
    stream = torch.cuda.Stream(dev)
    sh = stream.cuda_stream
    L = vitattn.lib()

    def step():
        if w.qk_norm:
            rc = L.vitattn_qkv_norm_rope(dqkv.data_ptr(), dcs.data_ptr(), dsn.data_ptr(), dqw.data_ptr(),
                                         dkw.data_ptr(), w.eps, q.data_ptr(), k.data_ptr(), v.data_ptr(), w.T, w.H,
                                         w.D, w.dtype, sh)
        else:
            rc = L.vitattn_qkv_rope(dqkv.data_ptr(), dcs.data_ptr(), dsn.data_ptr(), q.data_ptr(), k.data_ptr(),
                                    v.data_ptr(), w.T, w.H, w.D, w.dtype, sh)
        if rc:
            raise vitattn.VitAttnError(rc, entry)

    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    sampler.start()
    # exactly the requested warm-up steps, then untimed launches (reported apart) until the
    # clock sampler has run for a second
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    settle = 0
    t_w = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_w < 1.0:
            step()
            settle += 1
            if settle % 16 == 0:
                stream.synchronize()
    stream.synchronize()
    if args.steps is None:
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0.record(stream)
        for _ in range(5):
            step()
        w1.record(stream)
        w1.synchronize()
        steps = int(max(20, min(20000, 2000.0 / max(w0.elapsed_time(w1) / 5, 1e-3))))
        steps = int(max_over_ranks(float(steps), world))
    else:
        steps = args.steps
    barrier(world)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark("t_start")
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    ev1.synchronize()
    sampler.mark("t_stop")
    torch.cuda.synchronize(dev)
    barrier(world)
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world)
    clocks = sampler.stop()
    ms_step = ms_total / steps
    gbs = w.io_bytes * steps * world / (ms_total * 1e-3) / 1e9
    per_gpu = w.io_bytes / (ms_step * 1e-3) / 1e9

    # end to end through the Python entry, host copies on the same stream
    hqkv_p, hcs_p, hsn_p = (x.pin_memory() for x in (hqkv, hcs, hsn))
    hqw_p, hkw_p = (hqw.pin_memory(), hkw.pin_memory()) if w.qk_norm else (None, None)
    hq, hk, hv = (torch.empty((w.T, w.H, w.D), dtype=tdt).pin_memory() for _ in range(3))

    def e2e_step():
        dqkv.copy_(hqkv_p, non_blocking=True)
        dcs.copy_(hcs_p, non_blocking=True)
        dsn.copy_(hsn_p, non_blocking=True)
        if w.qk_norm:
            dqw.copy_(hqw_p, non_blocking=True)
            dkw.copy_(hkw_p, non_blocking=True)
            oq, ok, ov = vitattn.qkv_norm_rope(dqkv, dcs, dsn, dqw, dkw, w.eps, stream=stream)
        else:
            oq, ok, ov = vitattn.qkv_rope(dqkv, dcs, dsn, stream=stream)
        hq.copy_(oq, non_blocking=True)
        hk.copy_(ok, non_blocking=True)
        hv.copy_(ov, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_step()
    stream.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, args.e2e_steps)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
    e1.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    result = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            import oracle

            value, n, dt = cpu_leg(args.cpu_seconds)
            cpu = {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "cpu_model": cpu_model(), "kind": "oracle",
                   "sample": f"{n} of {w.T} tokens (seeded), numpy fp64, {dt:.1f} s"}
        in_bytes = 3 * w.T * w.H * w.D * 2 + 2 * w.T * w.D * 4 + (8 * w.D if w.qk_norm else 0)
        result = {
            "metric": metric, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "clock_settle_launches": {
                "launches": settle,
                "why": "untimed launches after the warm-up, until the nvidia-smi clock sampler (200 ms period) "
                       "has run for 1 s, so that the clocks line reflects the GPU under load"},
            "vs_baseline": None, "dtype": synth.DTYPE_NAMES[w.dtype],
            "data": "synthetic (seeded normals; 2-D rope tables of the patch grid)",
            "config": {"workload": w.name, "images": w.images, "grid": list(w.grid), "tokens": w.T, "H": w.H,
                       "D": w.D, "qk_norm": w.qk_norm, "global_batch": w.images * world,
                       "l2": f"{w.io_bytes / 2**20:.0f} MiB moved per step > 126 MiB L2, no flush",
                       "bytes_per_step": w.io_bytes},
            "roofline": {"bound": "hbm", "achieved": per_gpu, "peak": peak, "unit": "GB/s", "frac": per_gpu / peak,
                         "traffic": committed_traffic(w.name),
                         "peak_source": "measured copy bandwidth, MEASURED_PEAKS.json" if peaks else "fallback",
                         "kernel": "vitattn::" + kernel_of(w.name), "algorithmic_bytes_per_launch": w.io_bytes},
            "e2e": {"value": w.io_bytes * n_e2e * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": 3 * w.T * w.H * w.D * 2,
                    "ms_per_step": e2e_ms / n_e2e, "entry": entry[len("vitattn_"):] + " + stream copies"},
            "gpu_launches": steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
    ranks.finish(world)
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


def run_layer(args):
    """A ViT layer's attention step from its packed QKV projection: the
    prologue then the attention, one step each.  ``layer_batched`` copies v
    through the full prologue; ``layer_packed_batched`` rotates q and k only
    and lets the attention read v from the projection.  value: attention
    TFLOP/s over the whole step; the line also gives each kernel's share and
    the algorithmic bytes moved per step."""
    w = synth.LAYER[args.workload]
    if args.impl == "reference":
        print(json.dumps({"impl": "reference", "unavailable":
                          "layer workloads compare two device paths; the oracle arm runs on the attention workloads"}))
        return 0
    import torch

    from vit_bidirectional_attention_b200 import vitattn

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local if world > 1 else 0)
    pw = synth.PrologueWorkload(w.name, w.images, w.grid, w.H, w.D, w.dtype, index=w.index)
    qkv, cs, sn = synth.make_prologue(pw)
    tdt = torch.bfloat16 if w.dtype == synth.BF16 else torch.float16
    dqkv = torch.from_numpy(qkv.view(np.int16).copy()).view(tdt).to(dev)
    dcs, dsn = torch.from_numpy(cs).to(dev), torch.from_numpy(sn).to(dev)
    q, k, v, out = (torch.empty((w.T, w.H, w.D), dtype=tdt, device=dev) for _ in range(4))
    stream = torch.cuda.Stream(dev)
    sh = stream.cuda_stream
    L = vitattn.lib()
    hd = w.H * w.D
    v_src = dqkv.data_ptr() + 2 * hd * 2  # v's columns of the projection

    def prologue():
        if w.packed:
            rc = L.vitattn_qk_rope(dqkv.data_ptr(), dcs.data_ptr(), dsn.data_ptr(), q.data_ptr(), k.data_ptr(), w.T,
                                   w.H, w.D, w.dtype, sh)
        else:
            rc = L.vitattn_qkv_rope(dqkv.data_ptr(), dcs.data_ptr(), dsn.data_ptr(), q.data_ptr(), k.data_ptr(),
                                    v.data_ptr(), w.T, w.H, w.D, w.dtype, sh)
        if rc:
            raise vitattn.VitAttnError(rc, "prologue")

    def attention():
        if w.packed:
            rc = L.vitattn_forward_strided(q.data_ptr(), k.data_ptr(), v_src, out.data_ptr(), w.images, w.N, w.H, w.D,
                                           hd, hd, 3 * hd, w.scale, w.dtype, sh)
        else:
            rc = L.vitattn_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.images, w.N, w.H, w.D,
                                   w.scale, w.dtype, sh)
        if rc:
            raise vitattn.VitAttnError(rc, "attention")

    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            prologue()
            attention()
    stream.synchronize()
    settle = 0
    t_w = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_w < 1.0:
            prologue()
            attention()
            settle += 1
            if settle % 16 == 0:
                stream.synchronize()
    stream.synchronize()
    steps = args.steps or 200
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.mark("t_start")
    with torch.cuda.stream(stream):
        for e in ev:
            e[0].record(stream)
            prologue()
            e[1].record(stream)
            attention()
            e[2].record(stream)
    stream.synchronize()
    sampler.mark("t_stop")
    barrier(world)
    clocks = sampler.stop()
    pro_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    att_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    ms_step = max_over_ranks(ev[0][0].elapsed_time(ev[-1][2]), world) / steps
    peaks, _ = measured_peaks()
    peak = float(peaks["bf16_tflops"]) if peaks else FALLBACK_PEAK_TFLOPS
    if rank == 0:
        per_gpu = w.flops / (ms_step * 1e-3) / 1e12
        print(json.dumps({
            "metric": METRIC, "value": w.flops * world / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": synth.DTYPE_NAMES[w.dtype],
            "data": "synthetic (seeded normals; 2-D rope tables of the patch grid)",
            "clock_settle_launches": {"launches": 2 * settle, "why": "untimed steps after the warm-up until the "
                                      "nvidia-smi clock sampler has run for 1 s"},
            "config": {"workload": w.name, "images": w.images, "grid": list(w.grid), "N": w.N, "H": w.H, "D": w.D,
                       "packed": w.packed, "global_batch": w.images * world,
                       "l2": f"{w.io_bytes / 2**20:.0f} MiB moved per step > 126 MiB L2, no flush"},
            "layer": {"prologue_ms": pro_ms, "attention_ms": att_ms,
                      "prologue_bytes": w.prologue_bytes, "attention_bytes": w.attention_bytes,
                      "bytes_per_step": w.io_bytes,
                      "prologue_gbs": w.prologue_bytes / (pro_ms * 1e-3) / 1e9,
                      "attention_tflops": w.flops / (att_ms * 1e-3) / 1e12},
            "roofline": {"bound": "tensor", "achieved": per_gpu, "peak": peak, "unit": "TFLOP/s", "frac": per_gpu / peak,
                         "traffic": None, "kernel": "prologue + vitattn::fwd_kernel",
                         "note": "whole layer step; the attention kernel alone is layer.attention_tflops"},
            "gpu_launches": 2 * steps,
            "clocks": clocks,
            "cpu_baseline": None,
        }), flush=True)
    ranks.finish(world)
    return 0


def main():
    args = parse()
    if args.workload in synth.PROLOGUE:
        return run_prologue(args)
    if args.workload in synth.LAYER:
        return run_layer(args)
    if args.impl == "reference":
        return run_reference(args)
    import numpy as np
    import torch

    from vit_bidirectional_attention_b200 import vitattn

    world, rank, local = dist_setup(args)
    w, q, k, v = load_workload(args.workload)
    ragged = isinstance(w, synth.RaggedWorkload)
    gqa = not ragged and bool(w.Hkv)
    causal = not ragged and w.causal
    dlse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda") if causal else None
    tdt = torch.bfloat16 if w.dtype == synth.BF16 else torch.float16
    dev = torch.device("cuda", local if world > 1 else 0)

    def host(bits):
        return torch.from_numpy(bits.view(np.int16).copy()).view(tdt)

    hq, hk, hv = (host(x) for x in (q, k, v))
    dq, dk, dv = (x.to(dev) for x in (hq, hk, hv))
    dout = torch.empty_like(dq)  # [.., H, D] like q (k, v may have fewer heads)
    stream = torch.cuda.Stream(dev)
    sh = stream.cuda_stream
    L = vitattn.lib()

    if ragged:
        import ctypes

        cu_arr = (ctypes.c_int32 * len(w.cu_seqlens))(*w.cu_seqlens)
        cu_ptr, n_seqs = ctypes.cast(cu_arr, ctypes.c_void_p), len(w.seqlens)

        def step():
            rc = L.vitattn_forward_varlen(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), cu_ptr,
                                          n_seqs, w.H, w.D, w.scale, w.dtype, sh)
            if rc:
                raise vitattn.VitAttnError(rc, "vitattn_forward_varlen")
    elif causal:
        def step():
            rc = L.vitattn_forward_ext(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), dlse.data_ptr(),
                                       w.B, w.N, w.N, w.H, w.D, w.scale, 1, w.dtype, sh)
            if rc:
                raise vitattn.VitAttnError(rc, "vitattn_forward_ext")
    elif gqa:
        def step():
            rc = L.vitattn_forward_gqa(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), w.B, w.N,
                                       w.H, w.Hkv, w.D, w.scale, w.dtype, sh)
            if rc:
                raise vitattn.VitAttnError(rc, "vitattn_forward_gqa")
    else:
        def step():
            rc = L.vitattn_forward(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), w.B,
                                   w.N, w.H, w.D, w.scale, w.dtype, sh)
            if rc:
                raise vitattn.VitAttnError(rc, "vitattn_forward")

    # correctness gate on this exact launch configuration before timing
    with torch.cuda.stream(stream):
        if ragged:
            rc = vitattn.forward_varlen_ptr(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(),
                                            w.cu_seqlens, w.H, w.D, w.scale, w.dtype, sh, checked=True)
        elif gqa:
            rc = vitattn.forward_gqa_ptr(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), w.B, w.N,
                                         w.H, w.Hkv, w.D, w.scale, w.dtype, sh, checked=True)
        elif causal:
            rc = vitattn.forward_ext_ptr(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(),
                                         dlse.data_ptr(), w.B, w.N, w.N, w.H, w.D, w.scale, True, w.dtype, sh,
                                         checked=True)
        else:
            rc = vitattn.forward_ptr(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), w.B,
                                     w.N, w.H, w.D, w.scale, w.dtype, sh, checked=True)
    if rc:
        raise vitattn.VitAttnError(rc, "checked forward")

    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    sampler.start()
    # exactly the requested warm-up steps, then (untimed, reported apart) more launches until the
    # clock sampler has run for a second: nvidia-smi samples every 200 ms, and a short timed
    # region alone would hold too few samples to show the clocks under load
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step()
            if (i + 1) % 16 == 0:
                stream.synchronize()
    stream.synchronize()
    t_w = time.perf_counter()
    settle_done = 0
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_w < 1.0:
            step()
            settle_done += 1
            if settle_done % 16 == 0:
                stream.synchronize()
    stream.synchronize()
    if args.steps is None:
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0.record(stream)
        for _ in range(5):
            step()
        w1.record(stream)
        w1.synchronize()
        est_ms = max(w0.elapsed_time(w1) / 5, 1e-3)
        steps = int(max(20, min(20000, 2000.0 / est_ms)))
        steps = int(max_over_ranks(float(steps), world))
    else:
        steps = args.steps
    args.steps = steps
    flush = None
    if w.io_bytes <= L2_BYTES:  # inputs would stay in L2 between launches: evict them before each one
        flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

        def flush():
            flush_buf.fill_(0)
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.mark("t_start")
    launch_ms = []
    with torch.cuda.stream(stream):
        ms_local = timed_launches(step, args.steps, stream, torch.cuda.Event, flush, launch_ms)
    sampler.mark("t_stop")
    torch.cuda.synchronize(dev)
    barrier(world)
    ms_total = max_over_ranks(ms_local, world)
    clocks = sampler.stop()
    ms_step = ms_total / args.steps
    tflops = ranks.job_throughput(w.flops, args.steps, world, ms_total)
    per_gpu_tflops = w.flops / (ms_step * 1e-3) / 1e12

    # end to end through the host-buffer entry point
    hq_p, hk_p, hv_p = (x.pin_memory() for x in (hq, hk, hv))
    hout_p = torch.empty_like(hq).pin_memory()  # like q
    e2e_steps = max(1, args.e2e_steps)

    if ragged or gqa or causal:
        hlse_p = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory() if causal else None

        def e2e_step():
            for d, h in ((dq, hq_p), (dk, hk_p), (dv, hv_p)):
                d.copy_(h, non_blocking=True)
            if ragged:
                vitattn.forward_varlen(dq, dk, dv, w.cu_seqlens, out=dout, scale=w.scale, stream=stream)
            elif gqa:
                vitattn.forward_gqa(dq, dk, dv, out=dout, scale=w.scale, stream=stream)
            else:
                _, lse = vitattn.forward_ext(dq, dk, dv, out=dout, scale=w.scale, causal=True, with_lse=True,
                                             stream=stream)
                hlse_p.copy_(lse, non_blocking=True)
            hout_p.copy_(dout, non_blocking=True)
    else:
        def e2e_step():
            rc = L.vitattn_forward_host(hq_p.data_ptr(), hk_p.data_ptr(), hv_p.data_ptr(),
                                        hout_p.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                        dout.data_ptr(), w.B, w.N, w.H, w.D, w.scale, w.dtype, sh)
            if rc:
                raise vitattn.VitAttnError(rc, "vitattn_forward_host")

    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_step()
    stream.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
    e1.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = ranks.job_throughput(w.flops, e2e_steps, world, e2e_ms)

    peaks, peak_src = measured_peaks()
    if peaks:
        peak = float(peaks["bf16_tflops"])
        peak_note = "measured burst dense bf16 (cuBLAS 8192^3), MEASURED_PEAKS.json"
    else:
        peak = FALLBACK_PEAK_TFLOPS
        peak_note = "fallback 1.59 PFLOP/s (an earlier B200 measurement)"
    if w.dtype == synth.F16:
        peak_note += "; f16 runs at the bf16 rate (same nominal dense figure)"

    result = None
    if rank == 0:
        cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline(w, q, k, v, args.cpu_seconds)
        traffic = committed_traffic(args.workload)
        result = {
            "metric": METRIC,
            "value": tflops,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "clock_settle_launches": {
                "launches": settle_done,
                "why": "untimed launches after the warm-up, until the nvidia-smi clock sampler (200 ms period) "
                       "has run for 1 s, so that the clocks line reflects the GPU under load"},
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": synth.DTYPE_NAMES[w.dtype],
            "data": "synthetic (seeded normals with the workload's shape and distribution)",
            "config": dict(shape_config(w), **{
                "workload": args.workload,
                "scale": w.scale, "global_batch": (len(w.seqlens) if ragged else w.B) * world,
                "parallelism": f"independent ({'image' if ragged else 'b'},h) units per GPU x{world}",
                "l2": (f"inputs {w.io_bytes / 2**20:.0f} MiB > 126 MiB L2, no flush"
                       if flush is None else
                       f"inputs {w.io_bytes / 2**20:.1f} MiB fit in L2: {L2_FLUSH_BYTES >> 20} MiB written "
                       "before each timed launch, launch times summed from per-launch events"),
                "flops_per_step": w.flops,
            }),
            "pct_of_datasheet_peak": 100.0 * per_gpu_tflops / DATASHEET_PEAK_TFLOPS,
            "roofline": {
                "bound": "tensor",
                "achieved": per_gpu_tflops,
                "peak": peak,
                "unit": "TFLOP/s",
                "frac": per_gpu_tflops / peak,
                "frac_of_datasheet": per_gpu_tflops / DATASHEET_PEAK_TFLOPS,
                "traffic": traffic,
                "peak_source": peak_note if peaks else "fallback",
                "kernel": "vitattn::fwd_kernel",
                "algorithmic_flops_per_launch": w.flops,
                "algorithmic_bytes_per_launch": w.io_bytes,
                "achieved_hbm_gbs": w.io_bytes / (ms_step * 1e-3) / 1e9,
            },
            "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": sum(x.numel() for x in (hq, hk, hv)) * 2,
                    "d2h_bytes_per_step": hq.numel() * 2 + (w.B * w.H * w.N * 4 if causal else 0),
                    "ms_per_step": e2e_ms / e2e_steps,
                    "entry": ("forward_varlen + stream copies" if ragged else
                              "forward_gqa + stream copies" if gqa else
                              "forward_ext (causal, lse) + stream copies" if causal else "vitattn_forward_host")},
            "gpu_launches": args.steps * vitattn.launches_per_call(),
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        if launch_ms:  # each launch timed on its own after the L2 flush
            srt = sorted(launch_ms)
            result["launch_us"] = {"median": 1e3 * srt[len(srt) // 2], "min": 1e3 * srt[0],
                                   "note": "one event pair per launch after the flush; the ~6 us launch floor of "
                                           "that pattern is included"}
    ranks.finish(world)
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
