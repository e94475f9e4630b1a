"""The bench's multi-rank plumbing on CPU: two gloo ranks, the max-over-ranks
timing and the weak-scaling whole-job rate; the reference arm's non-zero
ranks do no work."""
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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 1.0 + rank  # rank 1 is the slow one
        ms = bench.reduce_max(local_ms, world, "cpu")
        results[rank] = (ms, bench.whole_job_gbps(1_000_000_000, ms, world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    assert got[0] == got[1]
    ms, gbps = got[0]
    assert ms == 2.0
    assert gbps == pytest.approx(2 * 1e9 / 2e-3 / 1e9)  # both ranks' bytes over the slow rank's time


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.whole_job_gbps(302_030_848 * 16, 1.0, 1) == pytest.approx(302_030_848 * 16 / 1e-3 / 1e9)


def test_reference_arm_other_ranks_do_nothing(capsys):
    class A:
        workload, steps, warmup, gpus = "yarn262k", 2, 1, 2
    assert bench.run_reference(A(), rank=1) is None
    assert capsys.readouterr().out == ""
