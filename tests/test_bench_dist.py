"""bench.py's multi-process path on CPU: two gloo ranks on 127.0.0.1.

The DP shards as independent replicas (one solve per GPU, no data-path
collective), so what the ranks share is only the timing plumbing: a barrier on
both sides of the timed region, the slowest rank's time (max over ranks), and
the whole job's units divided by it.  The reference arm runs on rank 0 alone.
"""
import io
import json
import os
import socket
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    r, w, _ = bench.dist_setup(None, backend="gloo")
    try:
        bench.barrier(w)
        ms = bench.max_over_ranks(10.0 + 5.0 * r, w)     # the ranks' own times differ
        bench.barrier(w)
        value = bench.job_value(100.0, ms, w)
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"rank": r, "world": w, "ms": ms, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_use_the_slowest_time_and_every_ranks_units(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["world"] == world
        assert g["ms"] == 15.0                           # max over ranks, seen by every rank
        assert g["value"] == pytest.approx(world * 100.0 / 0.015)


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_value(10.0, 2.0, 1) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        workload, steps, warmup, cpu_seconds = "tiny", 1, 0, 0.0
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(Args, rank=1, world=2)      # returns before any work or output
    assert buf.getvalue() == ""


def test_reference_arm_line_on_rank_zero():
    class Args:
        workload, steps, warmup, cpu_seconds = "tiny", 1, 0, 0.0
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(Args, rank=0, world=1)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["unit"] == bench.UNIT and line["metric"] == bench.METRIC
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
