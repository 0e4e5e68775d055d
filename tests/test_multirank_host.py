"""Host logic of the benchmark's multi-GPU path, on CPU with the gloo backend.

One process per GPU runs an independent replica of the workload (the path
has no exchange between GPUs); the job's time is the slowest rank's, and the
job's throughput is every rank's bytes over that time.  These tests run the
same helpers over two gloo ranks: the maximum must reach every rank, a rank
that is slower in one timing and faster in another must not be averaged in,
and the launcher's environment must be read the way torchrun sets it.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        # rank 0 is slower in the first timing, rank 1 in the second
        mine = [10.0 + 5.0 * (rank == 0), 20.0 + 7.0 * (rank == 1), 1.5 + rank]
        got = bench.max_over_ranks(mine)
        out.put((rank, (ws, r, local), got, bench.job_gbps(ws, 1e9, got[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, env, got, gbps in res:
        assert env == (2, rank, rank)
        assert got == [15.0, 27.0, 2.5]                  # element-wise maximum, same on every rank
        assert gbps == pytest.approx(2 * 1e9 / 15e-3 / 1e9)  # both replicas' bytes in the slowest time


def test_single_process_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.job_gbps(1, 26.2e6, 0.025) == pytest.approx(1048.0)
