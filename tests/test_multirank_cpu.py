"""The N > 1 bench path on the CPU: two gloo ranks.

Each rank runs its own batch (weak scaling, no data-path collective); the
job time is the max of the ranks' device times and the whole-job value is
every rank's work over that time. These functions are the ones bench.py uses.
"""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        job = bench.job_time_ms(local_ms[rank], world)
        value = bench.job_tops(6.0 * 4096 * 6912 * 2560, world, 10, job)
        out[rank] = (job, value)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_value():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    local = [40.0, 55.5]
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, local, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 55.5
    expected = 6.0 * 4096 * 6912 * 2560 * 2 * 10 / (55.5e-3) / 1e12
    assert out[0][1] == pytest.approx(expected)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.job_time_ms(12.5, 1) == 12.5
    assert bench.job_tops(1e12, 1, 1, 1000.0) == pytest.approx(1.0)
