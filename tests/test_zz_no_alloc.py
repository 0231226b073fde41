"""moe_expert_ffn_static: the expert FFN for callers that cannot allocate device memory.

Such callers -- an op inside an engine that owns every device allocation and hands
its ops no allocator, or a serving loop that must not allocate after start-up --
cannot give the library a workspace.  The static entry point keeps its scratch in
a fixed array inside the library instead.  These tests call it through the C ABI
(ctypes on libmoe.so) and check that two calls in a row give what the workspace
entry point gives, and what the fp64 oracle gives, within the tests' bf16 / fp32
tolerances, and that a shape whose scratch would not fit is refused with
MOE_ERR_WORKSPACE before anything runs.

The file name makes pytest collect it last; it must pass on its own in a fresh
process as well as after the other GPU tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_mixture_experts_26_b200 as moe
from oracle import moe_oracle as O
from workloads import make_inputs, small

pytestmark = pytest.mark.gpu

MOE_OK, MOE_ERR_WORKSPACE = 0, 3
STATIC_BYTES = 8 << 20


def c_lib():
    lib = ctypes.CDLL(moe.LIB_PATH)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.moe_expert_ffn_static.restype = i32
    lib.moe_expert_ffn_static.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
    return lib


def grouped_inputs(wl):
    """Inputs plus the grouped rows and offsets, made by the existing entry points."""
    inp = make_inputs(wl, "cuda")
    x = inp["x"]
    T, d = x.shape
    E = wl.E
    idx = torch.empty(T, 2, dtype=torch.int32, device="cuda")
    w = torch.empty(T, 2, dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pt = torch.empty(2 * T, dtype=torch.int32, device="cuda")
    inv = torch.empty(T, 2, dtype=torch.int32, device="cuda")
    xp = torch.empty(2 * T, d, dtype=x.dtype, device="cuda")
    ws = moe.alloc_workspace(T, d, wl.h, E, 2, x.dtype)
    moe.moe_route(x, inp["Wg"], idx, w)
    moe.moe_permute(idx, x, off, pt, inv, xp, ws, E)
    return inp, xp, off, ws


def call_static(lib, xp, off, inp, wl, y):
    dt = 1 if xp.dtype == torch.bfloat16 else 0
    return lib.moe_expert_ffn_static(
        xp.data_ptr(), off.data_ptr(), inp["W1"].data_ptr(), inp["W3"].data_ptr(),
        inp["W2"].data_ptr(), xp.shape[0], wl.d, wl.h, wl.E, dt, y.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def rel_fro(a, b):
    a = a.double().cpu().numpy() if torch.is_tensor(a) else a
    b = b.double().cpu().numpy() if torch.is_tensor(b) else b
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


class PerExpert:
    """Hands the oracle one expert's weights at a time (exact values as float32)."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return self.t[e].float().cpu().numpy()


def oracle_Y(xp, off, inp):
    return O.expert_ffn_grouped(xp.float().cpu().numpy(), off.cpu().numpy(),
                                PerExpert(inp["W1"]), PerExpert(inp["W3"]),
                                PerExpert(inp["W2"]))


@pytest.mark.parametrize("wl,tol", [
    (small("static_bf16", T=16, d=4096, h=14336, seed=21), 5e-3),   # a Mixtral decode batch
    (small("static_bf16_small", T=100, d=256, h=384, seed=22), 5e-3),
    (small("static_f32", T=64, d=128, h=256, dtype="f32", seed=23), 1e-5),
])
def test_static_scratch_matches_workspace_entry_point(wl, tol):
    lib = c_lib()
    inp, xp, off, ws = grouped_inputs(wl)
    ref = torch.empty(xp.shape[0], wl.d, dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn(xp, off, inp["W1"], inp["W3"], inp["W2"], ref, ws)
    Y64 = oracle_Y(xp, off, inp)
    for _ in range(2):  # two calls in a row share (and reuse) the one scratch array
        y = torch.full_like(ref, float("nan"))
        assert call_static(lib, xp, off, inp, wl, y) == MOE_OK
        torch.cuda.synchronize()
        assert torch.isfinite(y).all()
        assert rel_fro(y, ref) <= tol      # the workspace entry point
        assert rel_fro(y, Y64) <= tol      # the fp64 oracle


def test_static_scratch_single_expert():
    """One expert (E = 1) with an odd group padded to an even row count, as the
    workspace entry point takes it; the padding row's output is unspecified."""
    lib = c_lib()
    wl = small("static_e1", T=20, d=128, h=192, E=2, seed=24)
    inp = make_inputs(wl, "cuda")
    rows = 37
    xp = torch.zeros(rows + 1, wl.d, dtype=torch.bfloat16, device="cuda")
    xp[:rows] = inp["x"].repeat(2, 1)[:rows]
    one = {k: inp[k][:1].contiguous() for k in ("W1", "W3", "W2")}
    off = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    e1 = small("static_e1", T=(rows + 1) // 2, d=128, h=192, E=1)
    Y64 = oracle_Y(xp[:rows], off, one)
    for _ in range(2):
        y = torch.full((rows + 1, wl.d), float("nan"), device="cuda")
        assert call_static(lib, xp, off, one, e1, y) == MOE_OK
        torch.cuda.synchronize()
        assert rel_fro(y[:rows], Y64) <= 5e-3


def test_static_scratch_rejects_shapes_beyond_its_limit():
    lib = c_lib()
    wl = small("static_big", T=147, d=4096, h=14336)  # 294 rows * 14336 * 2 B > 8 MiB - 256
    assert 2 * wl.T * wl.h * 2 > STATIC_BYTES - 256
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    rc = lib.moe_expert_ffn_static(p, p, p, p, p, 2 * wl.T, wl.d, wl.h, wl.E, 1, p,
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == MOE_ERR_WORKSPACE
