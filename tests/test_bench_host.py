"""Host-side logic of bench.py (no GPU): the L2 label of each workload, the clock
sampler's window filter, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import bench
from sparse_window_attention_b200 import synth


def test_l2_label_follows_the_input_bytes():
    small = bench.workload_config(synth.WORKLOADS["flux1k"], 1)["l2"]
    large = bench.workload_config(synth.WORKLOADS["flux2k"], 1)["l2"]
    assert "< 126 MB L2" in small and "l2_flushed" in small
    assert "> 126 MB L2; no flush" in large


def test_shard_mode_is_named_in_the_config():
    wl = synth.WORKLOADS["flux2k"]
    assert "split over 4 GPU(s)" in bench.workload_config(wl, 4, strong=True)["parallelism"]
    assert bench.workload_config(wl, 4)["parallelism"].startswith("replicas")


def test_clock_samples_outside_the_timed_region_are_dropped():
    s = bench.ClockSampler(0)
    s.source = "nvml from a separate process, every 0.5 ms"
    s.max_mhz = 1965.0
    s.lines = ["100.000100 1500 8", "100.001000 1965 4", "100.002000 1900 0", "100.009000 1800 64"]
    s.t0, s.t1 = 100.0005, 100.0025
    out = s.summary()
    assert out["samples"] == 2 and out["sm_mhz"] == (1965 + 1900) / 2
    assert out["reasons"] == ["sw_power_cap"]  # hw_slowdown and hw_thermal_slowdown fell outside
    # interval samples ("ta tb mhz bits"): a query that overlaps the region counts
    s.lines = ["99.990 100.0007 1700 0", "100.0026 100.004 1800 0", "100.0010 100.0012 1965 0"]
    out = s.summary()
    assert out["samples"] == 2 and out["sm_mhz"] == (1700 + 1965) / 2


def test_reference_arm_prints_one_contract_line(repo_root):
    r = subprocess.run([sys.executable, os.path.join(repo_root, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3", "--workload", "tiny"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["nproc"] >= 1
