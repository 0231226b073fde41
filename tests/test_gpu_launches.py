"""The number of libmoe kernels one layer call launches, counted by the CUDA profiler
(CUPTI through torch.profiler), against ``launches_per_layer`` — the figure the
benchmark reports as its launch count."""
import pytest
import torch

import sparse_mixture_experts_26_b200 as moe
from workloads import make_inputs, small

pytestmark = pytest.mark.gpu


def _kernel_names(fn):
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA], acc_events=True) as prof:
        fn()
        torch.cuda.synchronize()
    return [e.name for e in prof.events()
            if e.device_type == torch.autograd.DeviceType.CUDA]


@pytest.mark.parametrize("T,d,E", [(16, 256, 8), (100, 256, 8), (300, 256, 8), (700, 256, 8),
                                   (1100, 256, 8), (1100, 136, 8), (700, 256, 16)])
def test_layer_launch_count(T, d, E):
    """Above 512 tokens the router counts the grouping (no count pass) where the fp64
    tensor-core router applies (E <= 8, d a multiple of 32)."""
    wl = small("lc", T=T, d=d, h=384, E=E, seed=T)
    inp = make_inputs(wl, "cuda")
    x = inp["x"]
    ws = moe.alloc_workspace(T, d, 384, wl.E, 2, x.dtype, x.device)
    y = torch.empty_like(x)

    def call():
        moe.moe_layer_forward(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], y, ws)

    call()  # first call outside the profile (lazy module loading)
    torch.cuda.synchronize()
    sanity = _kernel_names(lambda: torch.ones(8, device="cuda").add_(1))
    if not sanity:
        pytest.skip("the CUDA profiler records no kernels on this system")
    names = _kernel_names(call)
    ours = [n for n in names if "moe::" in n]
    assert len(ours) == moe.launches_per_layer(T, d, E), ours
    assert len(ours) == len(names), names  # nothing but libmoe kernels


@pytest.mark.parametrize("T,cap", [(16, -1), (300, -1), (700, -1), (1100, -1), (1100, 200)])
def test_backward_launch_count(T, cap):
    """The kernels one backward call queues, against ``launches_per_backward``: the
    padded copies run only on the CTA-pair weight-gradient path without a capacity."""
    wl = small("lcb", T=T, d=256, h=384, seed=T + 3)
    inp = make_inputs(wl, "cuda")
    x = inp["x"]
    ws = moe.alloc_workspace(T, 256, 384, wl.E, 2, x.dtype, x.device)
    bws = moe.alloc_backward_workspace(T, 256, 384, wl.E, 2, x.dtype, x.device)
    y = torch.empty_like(x)
    dy = torch.ones_like(x)
    f32 = dict(dtype=torch.float32, device=x.device)
    dx = torch.empty_like(x)
    grads = [torch.empty(inp[k].shape, **f32) for k in ("Wg", "W1", "W3", "W2")]
    moe.moe_layer_forward_capacity(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], y, ws, cap)

    def call():
        moe.moe_layer_backward(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], dy, dx, *grads,
                               ws, bws, cap)

    call()  # first call outside the profile (lazy module loading)
    torch.cuda.synchronize()
    sanity = _kernel_names(lambda: torch.ones(8, device="cuda").add_(1))
    if not sanity:
        pytest.skip("the CUDA profiler records no kernels on this system")
    names = _kernel_names(call)
    ours = [n for n in names if "moe::" in n]
    assert len(ours) == moe.launches_per_backward(T, cap), ours
    assert len(ours) == len(names), names
    assert moe.moe_device_status(bws) == 0
