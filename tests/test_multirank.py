"""The bench's multi-rank path on CPU: two gloo ranks run the same
collective sequence (barrier, max of the device time over ranks) that
`bench.py --gpus N` runs over NCCL, and the whole-job throughput is every
rank's work over the slowest rank's time (weak scaling, no collective on
the data path)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = bench.Ranks(world, torch.device("cpu"))
        r.barrier()
        ms = 10.0 + 5.0 * rank                  # rank 1 is the slowest
        slowest = r.max(ms)
        r.barrier()
        q.put((rank, slowest, bench.throughput(4.0e13, world, slowest)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [15.0, 15.0]
    assert got[0][2] == pytest.approx(2 * 4.0e13 / 15e-3 / 1e12)


def test_single_rank_is_a_no_op():
    r = bench.Ranks(1, torch.device("cpu"))
    r.barrier()
    assert r.max(3.5) == 3.5
    assert bench.throughput(1e12, 1, 1.0) == pytest.approx(1000.0)
