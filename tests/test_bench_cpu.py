"""bench.py's reference arm on CPU (the tiny fp32 workload): one JSON line with the
keys the contract asks for, and the same workload ``config`` as the GPU arm prints
(including the parallelism key), so the two lines compare like for like."""
import argparse
import json
import os
import subprocess
import sys

import pytest
import torch

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


def test_batch_size_and_diagnostic_options():
    """--tokens runs a workload's recipe at another batch size (same seed); the
    zero-weight power diagnostic is refused for the default line and the reference arm,
    and leaves the routing inputs unchanged."""
    from workloads import WORKLOADS, make_inputs
    ns = argparse.Namespace(workload="prefill", tokens=96)
    wl = bench.with_tokens(WORKLOADS["prefill"], ns)
    assert wl.T == 96 and wl.seed == WORKLOADS["prefill"].seed and wl.kind == "plain"
    with pytest.raises(SystemExit):
        bench.with_tokens(WORKLOADS["prefill"], argparse.Namespace(workload=None, tokens=96))
    for argv in (["--zero-weights"], ["--impl", "reference", "--workload", "tiny_f32",
                                      "--zero-weights"]):
        with pytest.raises(SystemExit):
            bench.main(argv)
    inp = make_inputs(WORKLOADS["tiny_f32"], "cpu")
    x, wg = inp["x"].clone(), inp["Wg"].clone()
    bench.zero_expert_weights(inp, argparse.Namespace(zero_weights=True))
    assert all(float(inp[k].abs().max()) == 0.0 for k in ("W1", "W3", "W2"))
    assert torch.equal(inp["x"], x) and torch.equal(inp["Wg"], wg)
    assert bench.SWEEP_TOKENS == (192, 256, 384) and set(bench.SWEEP_ROUTINGS) == {"prefill", "skew"}
