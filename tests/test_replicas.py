"""Replica bookkeeping of bench.py on N > 1 ranks, run as world-size-2 gloo
processes on the CPU: every rank takes the same collective steps, the timed
duration is the maximum over ranks and the throughput counts all ranks' work."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    bench.barrier(w)
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms, w)
    value = bench.replica_throughput(w, 100, 1, ms_max)
    bench.barrier(w)
    dist.destroy_process_group()
    out[rank] = (ms_max, value)


def test_two_replicas_take_max_time_and_sum_work():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]                      # every rank reports the same numbers
    ms_max, value = res[0]
    assert ms_max == pytest.approx(15.0)
    assert value == pytest.approx(2 * 100 / 0.015)


def test_single_process_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_throughput(1, 10, 8, 20.0) == pytest.approx(4000.0)
