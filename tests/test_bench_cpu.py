"""bench.py's host-side contract, checked without a GPU."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_product_arm_fails_loudly_without_a_gpu():
    r = _run("--steps", "1", "--warmup", "1")
    assert r.returncode != 0
    assert "no CUDA device" in r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("decode_gemv d_in=4096 d_out=4096 d=8")


def _bench_module():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    return bench


def test_ncu_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    """roofline.traffic comes from one ncu capture and stands only while every
    captured source file hashes as it did then."""
    import hashlib
    bench = _bench_module()
    sha = hashlib.sha1(open(os.path.join(ROOT, "bench.py"), "rb").read()).hexdigest()
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"sources": {"bench.py": sha}, "per_call": {1: 123}})
    assert bench.traffic_for(1) == 123 and bench.traffic_for(4) is None
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"sources": {"bench.py": "0" * 40}, "per_call": {1: 123}})
    assert bench.traffic_for(1) is None
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"sources": {"no/such/file.cu": sha}, "per_call": {1: 123}})
    assert bench.traffic_for(1) is None
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"sources": {}, "per_call": {1: 123}})
    assert bench.traffic_for(1) is None


def test_peaks_fall_back_to_the_recipe_values_without_a_measurement(monkeypatch):
    bench = _bench_module()
    monkeypatch.setattr(bench, "ROOT", os.path.join(ROOT, "no_such_directory"))
    p, src = bench.peaks()
    assert src == "fallback"
    assert p == {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def test_roofline_fraction_and_sums():
    bench = _bench_module()
    r = bench._roof("hbm", 3267.4, 6534.8, "GB/s", traffic=1.0)
    assert r["frac"] == 3267.4 / 6534.8 and r["bound"] == "hbm" and r["traffic"] == 1.0
    assert bench._sum_or_none([1, 2, 3]) == 6.0 and bench._sum_or_none([1, None]) is None
