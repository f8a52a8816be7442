"""The benchmark's reference arm (the CPU oracle) on the small workload: one
JSON line with the metric of the GPU arm and the fields a reference line
carries (no GPU needed)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.timeout(600)
def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "tiny"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    import bench
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["warmup"] >= 3 and d["steps"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_kernel_table_separates_calls_and_launches():
    import bench
    t = bench.kernel_table({"attn": (10.0, 5), "cov": (6.0, 15), "pool": (0.0, 0)}, 5)
    assert set(t) == {"attn", "cov"}
    assert t["attn"]["ms_per_call"] == 2.0 and t["attn"]["ms_per_launch"] == 2.0
    assert abs(t["cov"]["ms_per_call"] - 1.2) < 1e-12 and abs(t["cov"]["ms_per_launch"] - 0.4) < 1e-12
    assert t["cov"]["launches"] == 15 and abs(t["attn"]["share"] + t["cov"]["share"] - 1.0) < 1e-12


def test_every_workload_has_a_config_line():
    import bench
    import workloads as W
    for name in W.ORDER:
        w = W.WORKLOADS[name]
        c = bench.config_of(w, 1)
        assert c["workload"] == name and c["seq_len"] == w.N and c["topk"] == w.topk
        assert w.N % w.Bq == 0 and w.N % w.Bk == 0 and 0 <= w.topk <= w.Nk
        assert (w.cov_lambda > 0) == ("cov_select" in c["mode"])
