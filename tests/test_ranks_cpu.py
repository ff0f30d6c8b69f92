"""The multi-rank benchmark plumbing on CPU: two gloo ranks, no GPU.

Each rank owns whole (batch, head) units, so the only cross-rank steps are
barriers and the max of the ranks' timings; throughput counts the work of
every rank over the slowest rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from vit_bidirectional_attention_b200 import ranks


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, local = ranks.env_world()
    assert (w, r, local) == (world, rank, rank)
    ranks.init("gloo", w, timeout_s=60)
    ranks.barrier(w)
    ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    mx = ranks.max_over_ranks(ms, w)
    tput = ranks.job_throughput(1e12, 4, w, mx)
    out[rank] = (mx, tput)
    ranks.finish(w)


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1]
    mx, tput = out[0]
    assert mx == 15.0
    # 2 ranks x 4 steps x 1 TFLOP in 15 ms
    assert tput == pytest.approx(2 * 4 * 1.0 / 0.015)


def test_single_rank_needs_no_group():
    assert ranks.max_over_ranks(3.5, 1) == 3.5
    assert ranks.job_throughput(2e12, 10, 1, 1000.0) == pytest.approx(20.0)
    with pytest.raises(ValueError):
        ranks.job_throughput(1.0, 0, 1, 1.0)
