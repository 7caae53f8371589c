"""bench.py's host side on CPU: the reference arm's JSON line carries the keys of
the bench contract, and the oracle samples of the backward and momentum modes
run on a bounded slice of the workload."""
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_delta_rule_141_b200 import workloads as W  # noqa: E402


def test_reference_arm_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "0", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["config"]["workload"] == W.WORKLOADS[0].name
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_variant_oracle_samples():
    w = W.WORKLOADS[0]
    x = W.make_inputs(w, bench.rank_seed(0, 0))
    rng = np.random.default_rng(3)
    up = (rng.standard_normal((w.B, w.Hv, w.T, w.dv)).astype(np.float32), None)
    rate, threads, desc = bench.oracle_variant_sample(w, x, 64, up, None, None, budget_s=0.2)
    assert rate > 0 and threads >= 1 and "recurrent_grad" in desc
    kappa = np.ones((w.B, (w.T + 63) // 64), np.int32)
    rate, threads, desc = bench.oracle_variant_sample(w, x, 64, None, 0.25, kappa, budget_s=0.2)
    assert rate > 0 and "momentum" in desc


def test_forward_oracle_sample_is_bounded():
    # long sequences: a token prefix first (the oracle's cost per token does not depend on
    # the position), so the timed work stays near the budget; the rate counts B*T tokens
    w, x = W.workload_inputs(4, T=4096)
    rate, threads, desc, dt = bench.oracle_sample(w, x, 128, "exact", budget_s=0.05)
    assert rate > 0 and threads >= 1
    assert "the first 2048 of their 4096 tokens" in desc, desc
    n = int(desc.split()[0])
    assert abs(rate * dt - n * 2048 / w.Hv) <= 1e-6 * rate * dt


def test_roofline_arithmetic():
    peaks = {"hbm_gbs": 6448.0, "bf16_tflops": 1726.0}
    # the gdn_scalar_bf16 step: 279 MB and 3.69e10 FLOP in 0.217 ms is HBM-bound
    r = bench.roofline(3.69e10, 279e6, 0.217, peaks)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 279e6 / 0.217e-3 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6448.0) < 1e-12
    assert abs(r["tc_frac"] - 3.69e10 / 0.217e-3 / 1726e12) < 1e-12
    # at 324 FLOP per byte (above the ridge of ~268) the tensor bound applies
    r = bench.roofline(1.34e11, 414e6, 0.1, peaks)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - 1.34e11 / 1e-4 / 1726e12) < 1e-12
    assert abs(r["hbm_frac"] - 414e6 / 1e-4 / 6448e9) < 1e-12


def test_recorded_traffic_follows_the_sources(tmp_path, monkeypatch):
    """A committed DRAM figure is reported only while the kernels' source files are the
    ones it was measured on: any edit to them turns it into null."""
    src = tmp_path / "k.cuh"
    src.write_text("// kernel source\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"files": ["k.cuh"], "fingerprint": bench.files_fingerprint(["k.cuh"]),
             "bytes_per_launch": 4365551616}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"wl/C128/exact/tc2": entry}))
    assert bench.recorded_traffic("wl", 128, "exact", "tc2") == 4365551616
    assert bench.recorded_traffic("wl", 64, "exact", "tc2") is None   # no entry for that chunk
    src.write_text("// kernel source, edited\n")
    assert bench.recorded_traffic("wl", 128, "exact", "tc2") is None

