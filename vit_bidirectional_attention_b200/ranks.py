"""Multi-GPU plumbing for the benchmark: one process per GPU, no data-path
collective.

The attention of every (batch, head) pair is independent of every other, so
N GPUs each run a whole workload on their own inputs (weak scaling: the
per-GPU work is fixed as N grows).  Ranks meet only to line up the timed
region (barriers) and to take the slowest rank's device time; the job's
throughput is the work of all ranks divided by that time.
"""
from __future__ import annotations

import datetime
import os


def env_world():
    """(world_size, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, world: int, device=None, timeout_s: float = 120.0) -> None:
    """Join the process group (no-op for a single rank)."""
    if world <= 1:
        return
    import torch.distributed as dist

    kwargs = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kwargs["device_id"] = device
    dist.init_process_group(backend, **kwargs)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """The largest value of x over all ranks (the slowest rank's time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank did `steps` steps of `flops_per_step`
    within the slowest rank's `max_ms` milliseconds."""
    if max_ms <= 0 or steps <= 0:
        raise ValueError("timed region must be positive")
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


def finish(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
