"""The bench's rank logic on CPU with the gloo backend and two ranks: the job time is
the slowest rank's, the reported value is every rank's work over that time, and every
rank takes the same collective steps (no GPU, no CUDA)."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 1.0 + 0.5 * rank               # rank 1 is the slow one
        t = bench.max_over_ranks(elapsed, world)  # the same collective on every rank
        dist.barrier()
        out[rank] = (t, bench.job_throughput(100.0, world, 4, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo_two_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == pytest.approx(1.5)
    # 2 ranks x 4 steps x 100 units over the slowest rank's 1.5 s
    assert res[0][1] == res[1][1] == pytest.approx(800.0 / 1.5)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.job_throughput(10.0, 1, 3, 2.0) == pytest.approx(15.0)
