"""bench.py's measurement plumbing, on the CPU: the ncu traffic figure is
reported only for the kernel sources it was captured on, the rotated operand
copies of the per-row measurements exceed L2, and the reference arm prints the
contract's JSON line."""
import json
import os
import subprocess
import sys

import bench


def test_traffic_only_for_the_captured_sources(monkeypatch):
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        entry = json.load(f)["mxfp8_gemm_ffn_up"]
    monkeypatch.setattr(bench, "_src_hash", lambda: entry["src_hash"])
    assert bench._ncu_traffic("mxfp8_gemm_ffn_up") == entry["bytes_per_launch"]
    monkeypatch.setattr(bench, "_src_hash", lambda: "0" * 16)      # the kernels changed since the capture
    assert bench._ncu_traffic("mxfp8_gemm_ffn_up") is None
    assert bench._ncu_traffic("no_such_kernel") is None


def test_rotated_copies_exceed_l2():
    for nbytes in (1 << 20, 58_720_256, 180 << 20, 400 << 20):
        n = bench._copies(nbytes)
        assert n >= 2 and n * nbytes >= 320 << 20                 # > the 126 MB L2 in total


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                       cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "impl", "cpu_baseline", "e2e", "config"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_percentiles_nearest_rank():
    p = bench.percentiles([float(i) for i in range(1, 102)])      # 1 .. 101
    assert (p["p10"], p["p50"], p["p90"]) == (11.0, 51.0, 91.0)
    assert p["mean"] == 51.0
    assert bench.percentiles([]) is None
    q = bench.percentiles([3.0])
    assert q["p10"] == q["p50"] == q["p90"] == 3.0


def test_rows_summary_ranges():
    rows = {"quantize_rowwise_8192x8192": {"ms": 1.0, "GB/s": 5.0, "frac_hbm": 0.9},
            "fp8_gemm_8192x2048x8192": {"ms": 1.0, "TFLOPS": 2.0, "frac_fp8_peak": 0.8},
            "decode": {"a": {"gemm_frac_hbm": 0.5, "frac_hbm": 0.4, "fused_frac_hbm": 0.45},
                       "b": {"gemm_frac_hbm": 0.7, "frac_hbm": 0.6, "fused_frac_hbm": 0.65}},
            "timing": "x"}
    s = bench._rows_summary(rows)
    assert s["quantize_rowwise_8192x8192"] == {"frac_hbm": 0.9}
    assert s["fp8_gemm_8192x2048x8192"] == {"frac_fp8_peak": 0.8}
    assert s["decode_gemm_alone"] == {"frac_hbm_min": 0.5, "frac_hbm_max": 0.7, "cases": 2}
    assert s["decode_quantize_gemm"]["frac_hbm_min"] == 0.45
