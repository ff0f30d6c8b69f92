"""The benchmark's host side without a GPU: the reference arm (the fp64
oracle on the host cores) prints one JSON line with the contract's keys,
ranks other than 0 of a multi-rank launch exit quietly, and the committed
traffic figures are keyed by the source of the kernel they were taken on."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from vit_bidirectional_attention_b200 import build, synth  # noqa: E402


def run_bench(*args, env=None):
    e = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        e.pop(k, None)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          timeout=300, cwd=ROOT, env=e)


@pytest.mark.parametrize("workload,unit", [("tiny", "TFLOP/s"), ("multi_image", "TFLOP/s"),
                                           ("batched_gqa", "TFLOP/s"), ("batched_causal", "TFLOP/s"),
                                           ("rope_norm_batched", "GB/s")])
def test_reference_arm_prints_one_contract_line(workload, unit):
    r = run_bench("--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "3",
                  "--cpu-seconds", "0.2")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["higher_is_better"] is True
    assert d["config"]["workload"] == workload and d["dtype"] == "f64"
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == d["value"] and cpu["sample"]
    assert cpu["cpu_model"] and cpu["cpu_model"] != "unknown"
    assert d["e2e"] == {"value": d["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    r = run_bench("--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
                  env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_every_workload_maps_to_a_kernel_with_sources():
    names = list(synth.WORKLOADS) + list(synth.RAGGED) + list(synth.PROLOGUE)
    for w in names:
        k = bench.kernel_of(w)
        assert k in bench.KERNEL_SOURCES
        for rel in bench.KERNEL_SOURCES[k]:
            assert os.path.exists(os.path.join(ROOT, rel)), rel
    assert bench.kernel_of("rope_batched") == "qkv_rope_kernel"
    assert bench.kernel_of("rope_norm_batched") == "qkv_norm_rope_kernel"
    assert bench.kernel_of("batched") == "fwd_kernel"


def test_traffic_entries_apply_only_to_the_source_they_were_taken_on():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    for workload, entry in table.items():
        kernel = bench.kernel_of(workload)
        assert len(entry["kernel_hash"]) == 16 and entry["dram_bytes_per_launch"] > 0
        assert os.path.exists(os.path.join(ROOT, entry["source"]))
        want = entry["dram_bytes_per_launch"] if entry["kernel_hash"] == bench.kernel_hash(kernel) else None
        assert bench.committed_traffic(workload) == want
    h = hashlib.sha256()
    for rel in bench.KERNEL_SOURCES["fwd_kernel"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    assert bench.kernel_hash("fwd_kernel") == h.hexdigest()[:16]
    assert bench.committed_traffic("no_such_workload") is None


def test_each_kernel_hash_covers_the_headers_it_includes():
    """A kernel's hash must change when any file it is compiled from changes:
    every csrc header a kernel's own file includes is in its source list."""
    csrc = os.path.join(ROOT, "vit_bidirectional_attention_b200", "csrc")
    for kernel, rels in bench.KERNEL_SOURCES.items():
        names = {os.path.basename(r) for r in rels}
        for rel in rels:
            for line in open(os.path.join(ROOT, rel)):
                if line.startswith('#include "'):
                    inc = line.split('"')[1]
                    if os.path.exists(os.path.join(csrc, inc)):
                        assert inc in names, f"{kernel}: {rel} includes {inc}"


def test_library_rebuild_tracks_every_kernel_header():
    csrc = os.path.join(ROOT, "vit_bidirectional_attention_b200", "csrc")
    headers = {os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith(".cuh")}
    assert headers <= set(build.DEPS)
    assert os.path.join(ROOT, "include", "vitattn.h") in build.DEPS


class FakeClock:
    """A device timeline: launches advance it; events read it when recorded."""

    def __init__(self):
        self.now = 0.0
        self.log = []


def fake_event_cls(clock):
    class Event:
        def __init__(self, enable_timing=False):
            assert enable_timing
            self.t = None

        def record(self, stream):
            assert stream == "s"
            self.t = clock.now
            clock.log.append("event")

        def synchronize(self):
            assert self.t is not None

        def elapsed_time(self, other):
            return other.t - self.t

    return Event


@pytest.mark.parametrize("steps", [1, 7])
def test_timed_launches_without_flush_times_the_whole_region(steps):
    clock = FakeClock()

    def step():
        clock.now += 2.0
        clock.log.append("kernel")

    ms = bench.timed_launches(step, steps, "s", fake_event_cls(clock))
    assert ms == 2.0 * steps
    assert clock.log == ["event"] + ["kernel"] * steps + ["event"]


@pytest.mark.parametrize("steps", [1, 7])
def test_timed_launches_with_flush_times_only_the_launches(steps):
    """The flush runs before every launch and its time is left out: only the
    kernels' own intervals are summed."""
    clock = FakeClock()

    def step():
        clock.now += 2.0
        clock.log.append("kernel")

    def flush():
        clock.now += 40.0
        clock.log.append("flush")

    per = []
    ms = bench.timed_launches(step, steps, "s", fake_event_cls(clock), flush=flush, per_launch=per)
    assert ms == 2.0 * steps
    assert per == [2.0] * steps
    assert clock.log == ["flush", "event", "kernel", "event"] * steps


def test_flush_buffer_exceeds_l2():
    assert bench.L2_FLUSH_BYTES > bench.L2_BYTES
    small = [n for n, w in synth.WORKLOADS.items() if w.io_bytes <= bench.L2_BYTES]
    assert set(small) >= {"tiny", "small_vit", "doc_page"}
    assert "batched" not in small and "high_res" not in small
