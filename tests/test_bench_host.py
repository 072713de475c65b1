"""bench.py's host side on the CPU: the reference arm's JSON line (the float64 oracle timed on a
bounded token sample), the algorithmic byte count per token, the roofline record, and the rule
that a recorded ncu traffic figure applies only to the kernel sources it was taken on."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "2", "--steps", "2",
                          "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 0
    assert d["value"] > 0 and d["higher_is_better"] is True and d["unit"] == "tokens/s"
    assert d["config"]["workload"] == "n4096_T2048_bf16_gauss"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_algorithmic_bytes_per_token(bench):
    from rotation_activation_quantization_b200 import synthetic as syn

    w = syn.workload(4)  # n = 28672 bf16
    assert bench.bytes_per_token(w, "asym4") == 2 * 28672 + 28672 // 2 + 8
    assert bench.bytes_per_token(w, "sym8") == 2 * 28672 + 28672 + 4
    w1 = syn.workload(1)  # n = 1024 fp32
    assert bench.bytes_per_token(w1, "asym4") == 4 * 1024 + 512 + 8


def test_recorded_traffic_follows_the_sources(bench):
    from rotation_activation_quantization_b200 import synthetic as syn

    digest = bench.kernel_sources_digest()
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for index in (2, 3, 4):
        w = syn.workload(index)
        e = rec[w.name]
        got = bench.recorded_traffic(w, digest)
        if e["kernel_sources"] == digest:
            assert got == float(e["dram_bytes_per_token"]) * w.T
        else:
            assert got is None
        assert bench.recorded_traffic(w, "0" * 16) is None


def test_roofline_entry_arithmetic(bench):
    from rotation_activation_quantization_b200 import synthetic as syn

    w = syn.workload(3)
    peaks = {"hbm_gbs": 6554.6, "source": "measured"}
    m = {"w": w, "achieved": 3900.0, "bpt": bench.bytes_per_token(w, "asym4"), "sym": False,
         "avg_launch_ms": 0.075}
    r = bench.roofline_entry(m, "asym4", peaks, "0" * 16)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6554.6
    assert r["frac"] == pytest.approx(3900.0 / 6554.6) and r["frac_of_nominal_8tbs"] == pytest.approx(3900.0 / 8000.0)
    assert r["traffic"] is None and r["tokens_per_launch"] == w.T
