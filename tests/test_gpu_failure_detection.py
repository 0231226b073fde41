"""Device-side failure detection, tested without faulting, trapping or hanging a GPU.

Every wait inside libmoe's kernels (pipeline mbarriers, the fused small-batch FFN's
dependency counters) is bounded: a wait that runs out raises a flag in the workspace
status word and the kernel exits in order.  moe_selftest_wait_timeout runs those same
wait primitives against a barrier and a counter that nothing completes, with a short
limit; the test checks that both give up, that the flag is reported, and that the
context and workspace stay usable for the real layer afterwards.
"""
import time

import numpy as np
import pytest
import torch

import sparse_mixture_experts_26_b200 as moe
from oracle import moe_oracle as O
from workloads import make_inputs, small

pytestmark = pytest.mark.gpu


def test_bounded_waits_give_up_and_report():
    wl = small("fd", T=16, d=128, h=256, seed=12)
    inp = make_inputs(wl, "cuda")
    ws = moe.alloc_workspace(wl.T, wl.d, wl.h, wl.E, 2, torch.bfloat16)
    t0 = time.perf_counter()
    outcome = moe.moe_selftest_wait_timeout(ws, 0.05)
    elapsed = time.perf_counter() - t0
    assert outcome == (2, 2)          # both waits gave up
    assert elapsed < 5.0              # bounded by the 50 ms limit (plus launch costs)
    assert moe.moe_device_status(ws) & 0x1   # MOE_DEV_FLAG_TIMEOUT was raised
    assert moe.moe_device_status(ws) == 0    # reading clears it
    # the context and the workspace still work for the real layer
    y = moe.layer_forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], ws=ws)
    assert moe.moe_device_status(ws) == 0
    c = {k: v.double().cpu().numpy() for k, v in inp.items()}
    ref = O.moe_layer(c["x"], c["Wg"], c["W1"], c["W3"], c["W2"])["y"]
    got = y.double().cpu().numpy()
    assert np.linalg.norm(got - ref) <= 5e-3 * np.linalg.norm(ref)


def test_selftest_rejects_bad_limits():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    for bad in (0.0, -1.0, 11.0):
        with pytest.raises(moe.MoeError):
            moe.moe_selftest_wait_timeout(ws, bad)
