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
