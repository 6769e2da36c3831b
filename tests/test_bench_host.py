"""Host-side pieces of bench.py, on CPU: the load-balance report of a prefill
step, the `config` object and the roofline denominators."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_quantized_moe_gemv_b200 import workload as wlm  # noqa: E402


def test_load_balance_by_hand():
    c = np.array([0, 0, 5, 128, 129, 300, 8192, 1023, 1024])
    r = bench.load_balance(c)
    assert r["rows"] == 10801 and r["experts_empty"] == 2 and r["experts_below_one_tile"] == 1
    assert r["rows_max"] == 8192 and r["rows_median_nonempty"] == 300.0
    # tiles of 128 rows: 0 0 1 1 2 3 64 8 8
    assert r["row_tiles"] == 87 and abs(r["tile_fill"] - 10801 / (87 * 128)) < 1e-15
    assert r["groups_over_one_tile"] == 5  # 129, 300, 8192, 1023, 1024
    assert r["rows_histogram"] == {"0": 2, "1-127": 1, "128-1023": 4, "1024-8191": 1, ">=8192": 1}
    assert sum(r["rows_histogram"].values()) == c.size


def test_load_balance_empty_and_zero():
    r = bench.load_balance(np.zeros(16, dtype=np.int32))
    assert r["rows"] == 0 and r["experts_empty"] == 16 and r["row_tiles"] == 0 and r["tile_fill"] == 0.0
    assert r["rows_median_nonempty"] == 0.0
    json.dumps(r)  # plain JSON types only


def test_config_names_the_workload():
    cfg = bench.workload_config(wlm.WORKLOADS["prefill32k"], world=2)
    assert cfg["global_batch"] == 2 * 32768 and cfg["parallelism"] == "replicas x2"
    assert "experts 0-255 int4 sym g32" in cfg["workload"] and "experts 256-511 int2 asym g16" in cfg["workload"]
    assert "5% uniform rows" in cfg["workload"] and "int8 per-channel" in cfg["workload"]
    d1 = bench.workload_config(wlm.WORKLOADS["decode1"])
    assert d1["workload"].startswith("decode1: T=1 ") and "fresh token per step" in d1["workload"]


def test_peaks_and_traffic_sources():
    peaks, kind = bench.load_peaks()
    assert kind in ("measured", "fallback")
    assert float(peaks["hbm_gbs"]) > 1000 and float(peaks["bf16_tflops"]) > 100
    for wl, (traffic, src) in bench.NCU_TRAFFIC.items():
        assert wl in wlm.WORKLOADS
        assert os.path.exists(os.path.join(ROOT, src)), src
        assert traffic is None or traffic > 0


def test_traffic_figures_match_their_profile_summaries():
    # the DRAM traffic the bench reports is the figure its ncu summary states
    # (read + write per launch or call, written with thousands separators)
    import re
    for wl, (traffic, src) in bench.NCU_TRAFFIC.items():
        if traffic is None:
            continue
        text = open(os.path.join(ROOT, src)).read()
        stated = {int(m.replace(",", "")) for m in re.findall(r"(\d{1,3}(?:,\d{3}){2,}) B\b", text)}
        assert traffic in stated, (wl, traffic, sorted(stated))


def test_clock_sampler_parses_nvidia_smi_rows(tmp_path, monkeypatch):
    # a stand-in nvidia-smi printing two samples in the queried column order
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\n"
                    "echo '0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active'\n"
                    "echo '0, 1950, 1965, 710.5, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "sleep 5\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}:{os.environ['PATH']}")
    rec = bench.ClockSampler(0).stop()
    assert rec == {"sm_mhz": 1957.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}
    assert bench.clock_rejections(rec) == []


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    assert bench.ClockSampler(0).stop() is None


def test_reference_arm_prints_the_contract_line():
    import subprocess
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("decode1:")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
