"""Expert parallelism on one GPU (world size 1: every expert is local) and the pieces
it relies on: the layer through ExpertParallelMoE matches the fp64 oracle (routing
bit-exact, y within the bf16 tolerance) and equals moe_layer_forward bit for bit, and
the expert FFN takes a single expert and a padding row outside every group.  The
exchange itself is covered on CPU by tests/test_ep_cpu.py (gloo, two ranks)."""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_26_b200 as moe
from oracle import moe_oracle as O
from sparse_mixture_experts_26_b200.ep import ExpertParallelMoE
from workloads import make_inputs, small

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,kind", [(16, "skew"), (300, "plain"), (1100, "plain")])
def test_single_rank_expert_parallel_equals_the_layer(T, kind):
    wl = small("ep1", T=T, d=256, h=384, seed=40 + T, kind=kind)
    inp = make_inputs(wl, "cuda")
    layer = ExpertParallelMoE(inp["Wg"], inp["W1"], inp["W3"], inp["W2"])
    routing = {}
    y_ep = layer.forward(inp["x"], routing)
    c = {k: v.double().cpu().numpy() for k, v in inp.items()}
    ref = O.moe_layer(c["x"], c["Wg"], c["W1"], c["W3"], c["W2"])
    np.testing.assert_array_equal(routing["idx"].cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(routing["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(routing["perm_token"].cpu().numpy(), ref["perm_token"])
    got = y_ep.double().cpu().numpy()
    assert np.linalg.norm(got - ref["y"]) / np.linalg.norm(ref["y"]) <= 5e-3
    ws = moe.alloc_workspace(T, 256, 384, wl.E, 2, inp["x"].dtype)
    y = moe.layer_forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], ws=ws)
    assert torch.equal(y_ep, y)


@pytest.mark.parametrize("rows", [7, 40, 301, 1501])  # small-batch, single-SM, pair paths
def test_expert_ffn_single_expert_with_padding_row(rows):
    """One expert, an odd number of grouped rows padded to an even count (the padding
    row belongs to no group; its output row is unspecified)."""
    wl = small("ep2", T=(rows + 1) // 2, d=128, h=192, E=2, seed=rows)
    inp = make_inputs(wl, "cuda")
    padded = rows + (rows & 1)
    x = torch.zeros(padded, 128, dtype=torch.bfloat16, device="cuda")
    x[:rows] = inp["x"].repeat(2, 1)[:rows]
    W1, W3, W2 = (inp[k][:1].contiguous() for k in ("W1", "W3", "W2"))
    off = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    Y = torch.full((padded, 128), float("nan"), device="cuda")
    ws = torch.zeros(moe.moe_expert_ffn_workspace_bytes(padded, 128, 192, 1),
                     dtype=torch.uint8, device="cuda")
    moe.moe_expert_ffn(x, off, W1, W3, W2, Y, ws)
    assert moe.moe_device_status(ws) == 0
    ref = O.expert_swiglu(x[:rows].double().cpu().numpy(), W1[0].double().cpu().numpy(),
                          W3[0].double().cpu().numpy(), W2[0].double().cpu().numpy())
    got = Y[:rows].double().cpu().numpy()
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3
