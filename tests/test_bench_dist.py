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
import time
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


def _fake_smi(tmp_path, rows):
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\n" + "".join(f"echo '{r}'\n" for r in rows) + "sleep 30\n")
    fake.chmod(0o755)


def _sample(pci=None, idx=0, n_rows=3):
    with bench.ClockSampler(idx, pci) as clk:
        for _ in range(100):                  # until the fake has printed its rows
            if len(open(clk.path).read().splitlines()) >= n_rows:
                break
            time.sleep(0.05)
    path = clk.path
    s = clk.summary()
    assert not os.path.exists(path)
    return s


def test_clock_sampler_parses_samples_and_leaves_no_file(tmp_path, monkeypatch):
    """The sampler reads nvidia-smi's CSV (median SM clock, the throttle reasons
    seen) and removes its samples file; without nvidia-smi it says so."""
    bus = "00000000:1B:00.0"
    _fake_smi(tmp_path, [
        f"{bus}, 0, 1500, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
        f"{bus}, 0, 1400, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
        f"{bus}, 0, 1600, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active"])
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    for pci in (None, (0, 0x1B, 0), (0, 0x99, 0)):   # one GPU listed: always that one
        s = _sample(pci)
        assert s["sm_mhz"] == 1500.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
        assert s["reasons"] == ["sw_power_cap"] and s["gpu"] == bus

    monkeypatch.setenv("PATH", str(tmp_path / "empty"))
    with bench.ClockSampler(0) as clk:
        pass
    path = clk.path
    assert clk.summary()["reasons"] == ["nvidia-smi unavailable"]
    assert not os.path.exists(path)


def test_clock_sampler_picks_the_cuda_device_among_several(tmp_path, monkeypatch):
    """With every GPU of a node listed, the rows of the CUDA device's PCI address
    are the ones summarised (a process that sees a remapped device set still
    reads its own GPU); with no address, nvidia-smi's index decides."""
    rows = []
    for i, (bus, mhz, thr) in enumerate([("00000000:0A:00.0", 1900, "Not Active"),
                                         ("00000000:1B:00.0", 1450, "Active"),
                                         ("00000000:2C:00.0", 1700, "Not Active")]):
        rows.append(f"{bus}, {i}, {mhz}, 1965, 900.0, 0x0, Not Active, {thr}, Not Active, Not Active")
    _fake_smi(tmp_path, rows)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    s = _sample(pci=(0, 0x1B, 0), idx=0)
    assert s["gpu"] == "00000000:1B:00.0" and s["sm_mhz"] == 1450.0
    assert s["reasons"] == ["hw_thermal_slowdown"]
    s = _sample(pci=None, idx=2)
    assert s["gpu"] == "00000000:2C:00.0" and s["sm_mhz"] == 1700.0 and s["reasons"] == []
    assert bench._parse_bus_id("00000001:C3:1F.0") == (1, 0xC3, 0x1F)
    assert bench._parse_bus_id("n/a") is None
