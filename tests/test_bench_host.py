"""Host-side pieces of bench.py, on CPU: the algorithmic work table the
roofline divides by, the recorded-traffic lookup, and the reference arm's
JSON line (the CPU oracle on a small sample)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from dora_inputs import workload  # noqa: E402


def test_kernel_work_matches_the_method():
    wl = workload("c3")
    T, di, do, r = wl.T, wl.d_in, wl.d_out, wl.r
    fl, by = bench.kernel_work("fwd_compose_gemm", wl)
    assert fl == 2 * T * do * (di + r)           # 575.5 GFLOP at c3
    assert abs(fl / 1e9 - 575.5) < 0.1
    fl, by = bench.kernel_work("compose_bwd", wl)
    assert by == 2 * 3 * T * do + 4 * do           # dy, pre in; dz out; C
    fl, by = bench.kernel_work("merge_gemm", wl)
    assert by == 2 * (2 * do * di + do * r + r * di) + 4 * do
    assert bench.kernel_work("no_such_kernel", wl) == (0, 0)


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    h = bench.source_hash("fwd_compose_gemm")
    assert h is not None and len(h) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_traffic.md").write_text(
        "| kernel | source hash | bytes per launch | capture |\n|---|---|---|---|\n"
        f"| fwd_compose_gemm | {h} | 123456 | test |\n| merge_gemm | 0000000000000000 | 99 | stale |\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_hash", lambda k: h if k == "fwd_compose_gemm" else "ffffffffffffffff")
    assert bench.recorded_traffic("fwd_compose_gemm") == 123456.0
    assert bench.recorded_traffic("merge_gemm") is None  # hash no longer matches
    assert bench.recorded_traffic("dx_gemm") is None     # never recorded


def test_layer_roofline_reproduces_the_step_bounds():
    """At 1649 TFLOP/s and 6539.5 GB/s the c3 step's bounds are norm 34 us, forward 365 us,
    compose backward 30.8 us and backward GEMMs 396 us (4.96 M tokens/s); c2's norm is
    HBM-bound at 5.2 us."""
    peaks = {"bf16_tflops": 1649.0, "hbm_gbs": 6539.5}
    t, tot = bench.layer_roofline(workload("c3"), peaks)
    us = {k: v * 1e6 for k, v in t.items()}
    assert abs(us["norm"] - 34.3) < 0.3 and abs(us["forward"] - 364.6) < 0.5
    assert abs(us["compose_bwd"] - 30.8) < 0.1 and abs(us["bwd_gemms"] - 395.9) < 0.5
    assert abs(4096 / tot / 1e6 - 4.96) < 0.01
    t2, _ = bench.layer_roofline(workload("c2"), peaks)
    assert abs(t2["norm"] * 1e6 - 5.17) < 0.05
    assert bench.layer_roofline(workload("c1"), peaks) == (None, None)
    assert bench.norm_flops(workload("c3")) == 2 * 8192 * 8192 * 384 + 2 * 384 ** 2 * 8192 + 2 * 8192 * 384 ** 2 \
        + 2 * 8192 * 8192 + 2 * 8192 * 384


def _reference_line(*extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *extra],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_reference_arm_line():
    line = _reference_line("--workload", "c1", "--steps", "2", "--warmup", "1")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert "whole steps" in line["cpu_baseline"]["sample"]


def test_reference_arm_samples_rows_when_whole_steps_do_not_fit():
    line = _reference_line("--workload", "c2", "--steps", "1", "--warmup", "1", "--ref-budget-s", "0.001")
    assert "64 of 4096 output rows" in line["cpu_baseline"]["sample"]
    assert line["value"] > 0 and line["config"]["tokens_per_gpu"] == 2048
