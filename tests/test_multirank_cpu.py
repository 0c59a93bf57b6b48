"""The benchmark's multi-rank host logic on CPU: two gloo ranks (127.0.0.1) agree on the
slowest rank's time and on the whole-job throughput.  The mixer itself needs no
collective (ranks hold independent sequences), so this is all the multi-GPU path adds."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 100.0 + 50.0 * rank                      # rank 1 is the slow one
        mx = bench.max_over_ranks(my_ms, dist, "cpu")
        gbs = bench.job_gbs(bytes_per_rank_step=10**9, steps=10, world=world, max_ms=mx)
        q.put((rank, mx, gbs))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [150.0, 150.0]
    # 2 ranks x 1e9 bytes x 10 steps in 150 ms -> 133.33 GB/s for the whole job
    assert all(abs(r[2] - 2 * 1e9 * 10 / 0.150 / 1e9) < 1e-9 for r in res)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_gbs(10**9, 1, 1, 1000.0) == pytest.approx(1.0)
