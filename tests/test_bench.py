"""bench.py's own accounting, on the CPU: algorithmic bytes and FLOPs, the
roofline bound, the parity metrics of the bench line, the hash gate on the
committed ncu traffic, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_and_flops():
    sl = torch.tensor([1000, 0, 64, -5], dtype=torch.int32)  # negative lengths count as empty
    b = bench.algorithmic_bytes(sl, 2, 16)
    assert b["kv"] == 1064 * 576 * 2
    assert b["q"] == 4 * 2 * 16 * 576 * 2
    assert b["o"] == 4 * 2 * 16 * 512 * 2
    assert b["lse"] == 4 * 2 * 16 * 4
    assert b["total"] == b["kv"] + b["q"] + b["o"] + b["lse"]
    assert bench.algorithmic_flops(sl, 2, 16) == 2 * 16 * 2 * 1064 * (576 + 512)
    # the headline: 16 x 65536 tokens, 1,208,517,632 algorithmic bytes per call
    head = bench.algorithmic_bytes(torch.full((16,), 65536, dtype=torch.int32), 1, 16)
    assert head["total"] == 1208517632


def test_kernel_roofline_picks_the_binding_resource():
    byt = {"total": 1.0e9}
    # 1 GB at 5000 GB/s = 200 us; 1e12 FLOP at 1000 TFLOP/s = 1000 us -> tensor-bound
    r = bench.kernel_roofline(byt, 1e12, 2.0, 5000.0, 1000.0, "measured", None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(1e12 / 2e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1000.0)
    r = bench.kernel_roofline(byt, 1e9, 0.25, 5000.0, 1000.0, "measured", 123)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 123
    assert r["achieved"] == pytest.approx(1e9 / 0.25e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 5000.0)


def test_bench_parity_metrics():
    rng = np.random.default_rng(5)
    ref = rng.standard_normal((6, 512))
    ref_l = rng.standard_normal(6)
    ref_l[2] = -np.inf
    out_rows = np.zeros((10, 512), dtype=np.float32)
    lse_rows = np.zeros(10, dtype=np.float32)
    rows = [1, 4, 5, 7, 8, 9]
    out_rows[rows] = ref + 1e-3
    lse_rows[rows] = ref_l * (1 + 1e-6)
    p = bench.bench_parity([(rows[:3], ref[:3], ref_l[:3]), (rows[3:], ref[3:], ref_l[3:])], out_rows, lse_rows)
    assert p["rows"] == 6 and p["lse_neginf_match"]
    assert p["rmse"] == pytest.approx(1e-3, rel=1e-3)
    assert p["max_abs_err_over_max_ref"] == pytest.approx(1e-3 / np.abs(ref).max(), rel=1e-3)
    assert p["lse_rel_err"] <= 2e-6
    assert bench.bench_parity([], out_rows, lse_rows) is None


def test_ncu_traffic_is_gated_by_the_source_hash(monkeypatch):
    d = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: d["kernel_source_hash"])
    assert bench.ncu_traffic("x", 10 ** 9) == int(d["dram_bytes_per_kv_byte"] * 10 ** 9)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.ncu_traffic("x", 10 ** 9) is None


def test_reference_arm_prints_its_json_line(oracle_mod):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "b1_l1024_h16", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
