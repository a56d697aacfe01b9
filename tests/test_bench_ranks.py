"""bench.py's multi-process plumbing on CPU: two gloo ranks agree on the
slowest rank's time and on the whole-job rate; the reference arm runs on rank 0
only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = 1.5 + rank  # rank 1 is the slower replica
        slow = bench.max_over_ranks(ms, world, "cpu")
        rate = bench.whole_job_rate(512, world, slow)
        out[rank] = (slow, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1]
    slow, rate = out[0]
    assert slow == 2.5
    assert rate == pytest.approx(512 * 2 / 2.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.whole_job_rate(8, 1, 1.0) == pytest.approx(8000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import types
    import bench
    import workloads
    args = types.SimpleNamespace(steps=1, warmup=0, gpus=2)
    bench.run_reference(args, workloads.get("tiny"), rank=1, world=2)
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("path", ["smoothquant", "forward", "per-tensor", "ste-train", "weight-only"])
def test_reference_arm_line_on_rank_zero(capsys, path):
    """The reference arm (the CPU oracle) prints one JSON line per run with
    the keys the driver reads, for every bench path."""
    import json
    import types
    import bench
    import workloads
    args = types.SimpleNamespace(steps=1, warmup=0, gpus=1, path=path)
    bench.run_reference(args, workloads.get("tiny"), rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["metric"] == bench.metric_for(path)
    for k in ("value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config",
              "cpu_baseline", "e2e"):
        assert k in line
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0


def test_step_stats():
    import bench
    mean, median = bench.step_stats([1.0, 2.0, 10.0])
    assert mean == pytest.approx(13.0 / 3) and median == 2.0
