"""The bench's multi-rank plumbing on CPU: two gloo ranks, the max-over-ranks
timing and the weak-scaling whole-job rate; the reference arm's non-zero
ranks do no work, and its rank 0 prints the one JSON line the driver reads."""
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


def test_reference_arm_prints_its_contract_line(capsys, monkeypatch):
    """Rank 0 of the reference arm: one JSON line with the keys the driver
    reads (the oracle's sample kept small here)."""
    import json
    monkeypatch.setattr(bench, "calibrate_sample", lambda w, seconds, n_threads=0: 4 * w.block_size)

    class A:
        workload, steps, warmup, gpus = "tiny_4k", 2, 1, 1
    bench.run_reference(A(), rank=0)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and "64 of 4096" in d["cpu_baseline"]["sample"]
    assert d["config"]["workload"] == "tiny_4k"
