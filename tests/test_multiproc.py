"""The multi-rank path of bench.py on CPU: two gloo ranks (127.0.0.1) check that the timed
duration is reduced to the slowest rank's, that barriers pass, and that the whole-job rate
counts every rank's replica (weak scaling, no collective in the data path)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    ws, r, local = bench._dist()
    assert (ws, r, local) == (world, rank, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(True, None)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max = bench._max_over_ranks(ms, True, None)
        rate = bench.whole_job_rate(3.0e12, 4, world, ms_max)
        bench._barrier(True, None)
        out.put((rank, ms_max, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(2))
    for rank, ms_max, rate in res:
        assert ms_max == pytest.approx(15.0)
        # 2 ranks x 4 steps x 3e12 ops in 15 ms
        assert rate == pytest.approx(2 * 4 * 3.0e12 / 15e-3)


def test_single_rank_rate_is_units_over_time():
    import bench
    assert bench._max_over_ranks(7.5, False, None) == 7.5
    assert bench.whole_job_rate(1e9, 10, 1, 5.0) == pytest.approx(1e9 * 10 / 5e-3)
