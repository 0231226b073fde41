"""bench.py's reference arm on CPU (the tiny fp32 workload): one JSON line with the
keys the contract asks for, and the same workload ``config`` as the GPU arm prints
(including the parallelism key), so the two lines compare like for like."""
import argparse
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line_and_config():
    args = argparse.Namespace(workload="tiny_f32", steps=2, warmup=1, backward=False,
                              cpu_sample_tokens=16, cpu_sample_tokens_bwd=4)
    out = bench.run_reference(args)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["metric"] == bench.METRIC
    assert out["value"] > 0 and out["e2e"]["value"] == out["value"]
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0
    from workloads import WORKLOADS
    ours = bench.workload_config(WORKLOADS["tiny_f32"], {"parallelism": bench.parallelism(1)})
    assert out["config"] == ours
    json.dumps(out)


def test_default_run_headline_is_prefill():
    """No --workload: both arms time the prefill workload, the headline of the default
    line; the command-line options the driver and users rely on are present."""
    assert bench.SUITE_HEADLINE == "prefill"
    assert set(bench.SUITE_FORWARD) == {"decode", "skew", "long"}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"],
                       capture_output=True, text=True, timeout=120)
    assert p.returncode == 0
    for opt in ("--gpus", "--steps", "--warmup", "--impl", "--workload", "--backward"):
        assert opt in p.stdout, opt
