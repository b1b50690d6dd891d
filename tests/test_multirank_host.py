"""The bench's rank logic on CPU with the gloo backend: the job time is the slowest
rank's, the reported value is the job's work over that time, one call's heads are split
into contiguous slices (one per rank, uneven counts included), and per-head statistics
and pair counts are gathered in head order (no GPU, no CUDA)."""
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


@pytest.mark.parametrize("heads,world", [(40, 1), (40, 2), (40, 8), (24, 8), (16, 3), (5, 5), (7, 4)])
def test_head_slices_cover_every_head_once(heads, world):
    slices = [bench.head_slice(heads, world, r) for r in range(world)]
    assert slices[0][0] == 0 and slices[-1][1] == heads
    assert all(a[1] == b[0] for a, b in zip(slices, slices[1:]))       # contiguous, in rank order
    sizes = [hi - lo for lo, hi in slices]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_head_slice_rejects_more_ranks_than_heads():
    with pytest.raises(ValueError):
        bench.head_slice(4, 5, 0)


def _slice_worker(rank, world, port, heads, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = bench.head_slice(heads, world, rank)
        stats = [(float(h), 10.0 * h) for h in range(lo, hi)]     # per-head (mean, p99) of this slice
        gathered = bench.gather_head_stats(stats, world)
        pairs = bench.sum_over_ranks(float(hi - lo) * 1000.0, world)
        t = bench.max_over_ranks(0.1 * (hi - lo), world)
        out[rank] = (gathered, pairs, t)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,heads", [(2, 40), (3, 8)])
def test_head_split_bookkeeping_gloo(world, heads):
    """Every rank ends with all heads' statistics in head order, the summed pair count,
    and the slowest slice's time (3 ranks over 8 heads: slices of 2, 3 and 3)."""
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_slice_worker, args=(world, port, heads, out), nprocs=world, join=True)
        res = dict(out)
    want = [(float(h), 10.0 * h) for h in range(heads)]
    biggest = max(hi - lo for lo, hi in (bench.head_slice(heads, world, r) for r in range(world)))
    for r in range(world):
        gathered, pairs, t = res[r]
        assert [tuple(x) for x in gathered] == want
        assert pairs == pytest.approx(heads * 1000.0)
        assert t == pytest.approx(0.1 * biggest)
