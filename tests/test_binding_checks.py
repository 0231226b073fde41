"""The Python binding checks shapes, dtypes and devices before it hands bare pointers
to the C ABI (which cannot see them).  CPU tensors: every check here fails before
anything reaches the library or a GPU."""
import pytest
import torch

import sparse_mixture_experts_26_b200 as moe

T, d, h, E = 4, 16, 24, 8
bf = torch.bfloat16


def layer(**over):
    t = dict(x=torch.zeros(T, d, dtype=bf), Wg=torch.zeros(d, E, dtype=bf),
             W1=torch.zeros(E, h, d, dtype=bf), W3=torch.zeros(E, h, d, dtype=bf),
             W2=torch.zeros(E, d, h, dtype=bf), y=torch.zeros(T, d, dtype=bf),
             ws=torch.zeros(64, dtype=torch.uint8))
    t.update(over)
    return t


def forward(t):
    moe.moe_layer_forward(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], t["y"], t["ws"])


@pytest.mark.parametrize("name,bad,err", [
    ("y", torch.zeros(T + 1, d, dtype=bf), ValueError),
    ("y", torch.zeros(T, d, dtype=torch.float32), TypeError),
    ("Wg", torch.zeros(E, d, dtype=bf), ValueError),        # transposed router
    ("W2", torch.zeros(E, h, d, dtype=bf), ValueError),     # W2 laid out like W1
    ("W3", torch.zeros(E, h, d, dtype=torch.float32), TypeError),
    ("ws", torch.zeros(16, dtype=torch.int32), TypeError),
])
def test_forward_rejects_bad_operands(name, bad, err):
    with pytest.raises(err, match=name):
        forward(layer(**{name: bad}))


def test_forward_rejects_host_tensors_after_the_shape_checks():
    with pytest.raises(ValueError, match="CUDA"):
        forward(layer())


def test_stepwise_entry_points_check_their_buffers():
    x = torch.zeros(T, d, dtype=bf)
    with pytest.raises(TypeError, match="topk_idx"):
        moe.moe_route(x, torch.zeros(d, E, dtype=bf), torch.zeros(T, 2, dtype=torch.int64),
                      torch.zeros(T, 2))
    with pytest.raises(ValueError, match="x_perm"):
        moe.moe_permute(torch.zeros(T, 2, dtype=torch.int32), x,
                        torch.zeros(E + 1, dtype=torch.int32),
                        torch.zeros(2 * T, dtype=torch.int32),
                        torch.zeros(T, 2, dtype=torch.int32), torch.zeros(T, d, dtype=bf),
                        torch.zeros(64, dtype=torch.uint8), E)
    with pytest.raises(TypeError, match="y_perm"):
        moe.moe_expert_ffn(torch.zeros(2 * T, d, dtype=bf), torch.zeros(E + 1, dtype=torch.int32),
                           torch.zeros(E, h, d, dtype=bf), torch.zeros(E, h, d, dtype=bf),
                           torch.zeros(E, d, h, dtype=bf), torch.zeros(2 * T, d, dtype=bf),
                           torch.zeros(64, dtype=torch.uint8))
    with pytest.raises(ValueError, match="offsets"):
        moe.moe_expert_ffn(torch.zeros(2 * T, d, dtype=bf), torch.zeros(E, dtype=torch.int32),
                           torch.zeros(E, h, d, dtype=bf), torch.zeros(E, h, d, dtype=bf),
                           torch.zeros(E, d, h, dtype=bf), torch.zeros(2 * T, d),
                           torch.zeros(64, dtype=torch.uint8))
    with pytest.raises(ValueError, match="inv_perm"):
        moe.moe_combine(torch.zeros(2 * T, d), torch.zeros(T, dtype=torch.int32),
                        torch.zeros(T, 2), x)


def test_backward_checks_gradient_buffers():
    t = layer()
    f32 = torch.float32
    grads = dict(dx=torch.zeros(T, d, dtype=bf), dWg=torch.zeros(d, E, dtype=f32),
                 dW1=torch.zeros(E, h, d, dtype=f32), dW3=torch.zeros(E, h, d, dtype=f32),
                 dW2=torch.zeros(E, d, h, dtype=f32))
    dy = torch.zeros(T, d, dtype=bf)
    for name, bad in (("dW1", torch.zeros(E, h, d, dtype=bf)),
                      ("dW2", torch.zeros(E, h, d, dtype=f32)),
                      ("dy", torch.zeros(T, d + 8, dtype=bf))):
        g = dict(grads)
        y_in = dy
        if name == "dy":
            y_in = bad
        else:
            g[name] = bad
        with pytest.raises((ValueError, TypeError), match=name):
            moe.moe_layer_backward(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], y_in, g["dx"],
                                   g["dWg"], g["dW1"], g["dW3"], g["dW2"], t["ws"], t["ws"])
