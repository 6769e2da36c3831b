"""The N > 1 (replica) paths of bench.py, on CPU.

The decode/prefill path does not shard: `bench.py --gpus N` runs N
independent replicas, one process per GPU, with no collective in the data
path. What multi-process code there is: the job's time is the largest of the
ranks' timed regions (one MAX all-reduce); a timed region whose clock record
on rank 0 shows a slowdown is run once more by every rank together; and the
reference arm runs on rank 0 only, the other ranks leaving at once. These are
checked here with two gloo ranks (no GPU) and a stand-in for the clock
sampler.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench

        got = bench.max_over_ranks(values[rank], world, torch.device("cpu"))
        with open(os.path.join(outdir, f"rank{rank}"), "w") as f:
            f.write(repr(got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    values = [12.5, 31.25]
    mp.start_processes(_rank_main, args=(2, _free_port(), values, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    got = [float((tmp_path / f"rank{r}").read_text()) for r in range(2)]
    assert got == [max(values)] * 2


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.0, 1, None) == 7.0


@pytest.mark.parametrize("rank", [1, 3])
def test_reference_arm_other_ranks_exit_without_work(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="4", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "4",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


class _FakeSampler:
    """Stands in for the nvidia-smi sampler: hands out prepared clock records."""

    records = []

    def __init__(self, gpu_index):
        pass

    def stop(self):
        return dict(_FakeSampler.records.pop(0))


GOOD = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}
THERMAL = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_thermal_slowdown"], "samples": 3}
LOCKED = {"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}
POWER = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_rejections():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.clock_rejections(GOOD) == [] and bench.clock_rejections(None) == []
    assert bench.clock_rejections(THERMAL) == ["sw_thermal_slowdown"]
    assert len(bench.clock_rejections(LOCKED)) == 1  # held low with no reason: a leftover lock
    assert bench.clock_rejections(POWER) == []  # the power cap is kept and noted
    assert bench.clock_rejections(dict(GOOD, reasons=["hw_slowdown", "sw_power_cap"])) == ["hw_slowdown"]


@pytest.mark.parametrize("first,runs", [(GOOD, 1), (POWER, 1), (THERMAL, 2), (LOCKED, 2)])
def test_timed_region_remeasures_once(first, runs):
    sys.path.insert(0, ROOT)
    import bench

    _FakeSampler.records = [first, THERMAL]  # a second rejection is reported, not retried
    calls = []
    res, clk = bench.timed_region(lambda: calls.append(1) or len(calls), 0, 1, None, sampler=_FakeSampler)
    assert len(calls) == runs and res == runs
    if runs == 1:
        assert clk["first_run_rejected"] is None and clk["rejections"] == []
    else:
        assert clk["first_run_rejected"] and clk["rejections"] == ["sw_thermal_slowdown"]


def _region_rank(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench

        _FakeSampler.records = [THERMAL, GOOD]  # only rank 0 samples
        calls = []
        _, clk = bench.timed_region(lambda: calls.append(1), rank, world, torch.device("cpu"), sampler=_FakeSampler)
        with open(os.path.join(outdir, f"rank{rank}"), "w") as f:
            f.write(f"{len(calls)} {clk is not None}")
    finally:
        dist.destroy_process_group()


def test_timed_region_every_rank_remeasures_together(tmp_path):
    import torch.multiprocessing as mp

    mp.start_processes(_region_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    got = [(tmp_path / f"rank{r}").read_text() for r in range(2)]
    assert got == ["2 True", "2 False"]
