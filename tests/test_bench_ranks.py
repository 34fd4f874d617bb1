"""CPU tests of bench.py's multi-rank plumbing: the slowest rank's time and the whole-job
throughput over world_size 2 gloo ranks, and the reference arm's non-zero ranks."""
import os
import socket
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(1.5 + rank, "cpu")  # rank 1 is the slow one
        v = bench.job_throughput(world, 1e9, 10, t)
        with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
            f.write(f"{t} {v}")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_with_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for r in range(2):
        t, v = map(float, (tmp_path / f"r{r}").read_text().split())
        assert t == 2.5                       # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 1e9 * 10 / 2.5 / 1e9)  # both ranks' bytes over that time


def test_max_over_ranks_without_a_process_group():
    import bench
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
    assert bench.job_throughput(1, 2e9, 5, 2.0) == pytest.approx(5.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    args = types.SimpleNamespace(steps=3, warmup=3, reference_budget=1.0)
    assert bench.run_reference(args, rank=1, world=2) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(capsys):
    # the reference arm times the CPU oracle and prints the same metric as the GPU arm, with
    # impl "reference", no host<->device bytes and a cpu_baseline describing the run
    import json
    import bench
    args = types.SimpleNamespace(steps=1, warmup=3, reference_budget=2.0)
    bench.run_reference(args, rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
