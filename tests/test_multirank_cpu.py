"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1).

bench.py runs one independent replica per GPU (no data-path collective);
what crosses ranks is host-side: the barriers around the timed region, the
max over ranks of every device time, and the whole-job throughput (each
rank's bytes, over the slowest rank's time).  Here two spawned processes
take those steps with gloo on CPU tensors; a third check runs the
reference arm as rank 1 of 2, which must exit 0 without doing any work.
"""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.rank_barrier(world)
        # rank r "measured" 1.5 + r ms: every rank must end with the slowest
        ms = bench.max_over_ranks(1.5 + rank, world, "cpu")
        bench.rank_barrier(world)
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        got = dict(out)
    assert got == {0: 2.5, 1: 2.5}


def test_whole_job_value_is_weak_scaling():
    # each rank streams its own bytes per step; N ranks in the max time
    one = bench.whole_job_gbps(388.8e6, 0.4, 1)
    assert abs(one - 972.0) < 1e-9
    assert abs(bench.whole_job_gbps(388.8e6, 0.4, 8) - 8 * one) < 1e-6
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--gpus", "2",
                                     "--steps", "1", "--warmup", "3"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_keeps_the_contract(monkeypatch, capsys):
    """Rank 0 of the reference arm: one JSON line with the main arm's metric,
    unit, workload and direction, exactly the requested timed and warm-up
    steps, and the oracle described as the CPU baseline."""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("LOCAL_RANK", "0")
    monkeypatch.setattr(bench, "REF_BUDGET_S", 0.01)   # the smallest sample: 16 rows
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "2",
                                     "--warmup", "3"])
    assert bench.main() == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.WORKLOAD
    assert line["steps"] == 2 and line["warmup"] == 3
    assert line["value"] > 0 and line["ms_per_step"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "16 of 14336 output rows" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
