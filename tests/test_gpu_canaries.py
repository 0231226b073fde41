"""Out-of-bounds write detection by guard bands (canaries), through the C ABI.

Every output buffer and both workspaces are views into a larger allocation whose
leading and trailing 4 KiB hold a byte pattern; after the calls the pattern must be
intact.  The views start 4 KiB into their allocation, so they keep the library's
alignment requirement.  Shapes cover the small-batch (weight-streaming), single-SM
grouped and CTA-pair paths, a capacity, fp32, and the backward pass.
"""
import pytest
import torch

import sparse_mixture_experts_26_b200 as moe
from workloads import make_inputs, small

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A tensor view with guard bands of PATTERN bytes on both sides."""

    def __init__(self, shape, dtype, zero=False):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8,
                              device="cuda")
        self.nbytes = nbytes
        inner = self.raw[GUARD:GUARD + nbytes]
        if zero:
            inner.zero_()
        self.t = inner.view(dtype).view(shape)

    def intact(self):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.nbytes:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


def guarded_ws(T, d, h, E, dtype):
    return Guarded((moe.moe_workspace_bytes(T, d, h, E, 2, dtype),), torch.uint8, zero=True)


@pytest.mark.parametrize("T,d,h,kind,dtype,cap", [
    (16, 256, 384, "skew", "bf16", -1),     # weight-streaming FFN
    (100, 256, 384, "skew", "bf16", -1),    # weight-streaming FFN, 128-token tiles
    (300, 136, 200, "plain", "bf16", -1),   # single-SM grouped GEMM, ragged tiles
    (1100, 256, 384, "plain", "bf16", -1),  # CTA-pair grouped GEMM
    (1500, 136, 200, "skew", "bf16", 300),  # capacity on the pair path
    (37, 24, 40, "plain", "f32", -1),       # fp32 CUDA-core FFN
])
def test_layer_writes_stay_in_bounds(T, d, h, kind, dtype, cap):
    wl = small("can", T=T, d=d, h=h, seed=T, kind=kind, dtype=dtype)
    inp = make_inputs(wl, "cuda")
    x = inp["x"]
    ws = guarded_ws(T, d, h, wl.E, x.dtype)
    y = Guarded((T, d), x.dtype)
    moe.moe_layer_forward_capacity(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], y.t, ws.t, cap)
    assert moe.moe_device_status(ws.t) == 0
    assert ws.intact() and y.intact()


@pytest.mark.parametrize("T", [16, 300, 1100])
def test_stepwise_writes_stay_in_bounds(T):
    wl = small("can2", T=T, d=256, h=384, seed=T + 1)
    inp = make_inputs(wl, "cuda")
    x, E, d = inp["x"], wl.E, wl.d
    ws = guarded_ws(T, d, wl.h, E, x.dtype)
    idx = Guarded((T, 2), torch.int32)
    w = Guarded((T, 2), torch.float32)
    off = Guarded((E + 1,), torch.int32)
    pt = Guarded((2 * T,), torch.int32)
    inv = Guarded((T, 2), torch.int32)
    xp = Guarded((2 * T, d), x.dtype)
    Y = Guarded((2 * T, d), torch.float32)
    y = Guarded((T, d), x.dtype)
    moe.moe_route(x, inp["Wg"], idx.t, w.t)
    moe.moe_permute(idx.t, x, off.t, pt.t, inv.t, xp.t, ws.t, E)
    moe.moe_expert_ffn(xp.t, off.t, inp["W1"], inp["W3"], inp["W2"], Y.t, ws.t)
    moe.moe_combine(Y.t, inv.t, w.t, y.t)
    assert moe.moe_device_status(ws.t) == 0
    for name, g in (("ws", ws), ("idx", idx), ("w", w), ("offsets", off), ("perm_token", pt),
                    ("inv_perm", inv), ("x_perm", xp), ("Y", Y), ("y", y)):
        assert g.intact(), name


@pytest.mark.parametrize("T,cap", [(40, -1), (100, -1), (1100, -1), (1500, 300)])
def test_backward_writes_stay_in_bounds(T, cap):
    wl = small("can3", T=T, d=136, h=192, seed=T + 2, kind="skew")
    inp = make_inputs(wl, "cuda")
    x, E, d, h = inp["x"], wl.E, wl.d, wl.h
    ws = guarded_ws(T, d, h, E, x.dtype)
    bws = Guarded((moe.moe_backward_workspace_bytes(T, d, h, E),), torch.uint8, zero=True)
    y = torch.empty_like(x)
    moe.moe_layer_forward_capacity(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], y, ws.t, cap)
    g = torch.Generator(device="cpu")
    g.manual_seed(T)
    dy = torch.randn(T, d, generator=g).to(torch.bfloat16).cuda()
    dx = Guarded((T, d), x.dtype)
    dWg = Guarded(tuple(inp["Wg"].shape), torch.float32)
    dW1 = Guarded(tuple(inp["W1"].shape), torch.float32)
    dW3 = Guarded(tuple(inp["W3"].shape), torch.float32)
    dW2 = Guarded(tuple(inp["W2"].shape), torch.float32)
    moe.moe_layer_backward(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], dy, dx.t, dWg.t,
                           dW1.t, dW3.t, dW2.t, ws.t, bws.t, cap)
    assert moe.moe_device_status(bws.t) == 0
    for name, gb in (("ws", ws), ("bwd_ws", bws), ("dx", dx), ("dWg", dWg), ("dW1", dW1),
                     ("dW3", dW3), ("dW2", dW2)):
        assert gb.intact(), name
