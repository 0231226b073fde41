"""The library keeps no unsynchronised host state: in a fresh process, the first layer
calls (forward and backward) come from several host threads at once, each with its own
stream and workspaces, over shapes that reach every FFN kernel family; the results must
equal those of the same calls made one after another.  ctypes releases the GIL around
each foreign call, so the threads really run the library's host code concurrently."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys, threading, torch
sys.path.insert(0, sys.argv[1])
import sparse_mixture_experts_26_b200 as moe
from workloads import make_inputs, small

cases = [small("thr", T=T, d=256, h=384, seed=70 + T, kind="skew") for T in (16, 100, 300, 1100)]
inputs = [make_inputs(wl, "cuda") for wl in cases]
dys = [torch.randn(wl.T, wl.d, generator=torch.Generator().manual_seed(wl.T)).to(torch.bfloat16).cuda()
       for wl in cases]
torch.cuda.synchronize()

def run(i, stream, out):
    inp, wl = inputs[i], cases[i]
    with torch.cuda.stream(stream):
        ws = moe.alloc_workspace(wl.T, wl.d, wl.h, wl.E, 2, inp["x"].dtype, "cuda")
        y = torch.empty_like(inp["x"])
        moe.moe_layer_forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], y, ws)
        g = moe.layer_backward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], dys[i], ws)
        stream.synchronize()
        out[i] = (y, g, moe.moe_device_status(ws))

streams = [torch.cuda.Stream() for _ in cases]
start = threading.Barrier(len(cases))
par = {}
def worker(i):
    start.wait()
    run(i, streams[i], par)
threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(cases))]
for t in threads: t.start()
for t in threads: t.join()
ser = {}
for i in range(len(cases)):
    run(i, streams[i], ser)
for i in range(len(cases)):
    (y1, g1, s1), (y2, g2, s2) = par[i], ser[i]
    assert s1 == 0 and s2 == 0, (i, s1, s2)
    assert torch.equal(y1, y2), i
    for a, b in zip(g1, g2):
        assert torch.equal(a, b), i
print("ok")
"""


def test_first_calls_from_concurrent_threads():
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
