"""Parity of the CUDA layer with the CPU oracle, through the C ABI.

Gates: routing indices, group offsets, the permutation and the gathered rows are
bit-exact; gate weights are within 2 float32 ulp (fp64 exp vs numpy exp, rounded
once); the layer output is within a relative Frobenius error of 5e-3 for bf16 and
1e-5 for fp32.  Per-token relative errors above 2e-2 are reported as failures too,
so one bad row cannot hide in a large batch.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_26_b200 as moe
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs, small

pytestmark = pytest.mark.gpu

BF16_TOL = 5e-3
F32_TOL = 1e-5
TOKEN_TOL = 2e-2


def f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def raw16(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy()


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def worst_token(a, b):
    num = np.linalg.norm(a - b, axis=1)
    den = np.maximum(np.linalg.norm(b, axis=1), 1e-30)
    return float((num / den).max())


class PerExpert:
    """Hands the oracle one expert's weights at a time (exact values as float32)."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return self.t[e].float().cpu().numpy()


def run_steps(inp, E):
    """Route -> permute -> expert FFN -> combine through the step-wise entry points."""
    x = inp["x"]
    T, d = x.shape
    h = inp["W1"].shape[1]
    dev = x.device
    ws = moe.alloc_workspace(T, d, h, E, 2, x.dtype, dev)
    idx = torch.empty(T, 2, dtype=torch.int32, device=dev)
    w = torch.empty(T, 2, dtype=torch.float32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    pt = torch.empty(2 * T, dtype=torch.int32, device=dev)
    inv = torch.empty(T, 2, dtype=torch.int32, device=dev)
    xp = torch.empty(2 * T, d, dtype=x.dtype, device=dev)
    Y = torch.empty(2 * T, d, dtype=torch.float32, device=dev)
    y = torch.empty_like(x)
    moe.moe_route(x, inp["Wg"], idx, w)
    moe.moe_permute(idx, x, off, pt, inv, xp, ws, E)
    moe.moe_expert_ffn(xp, off, inp["W1"], inp["W3"], inp["W2"], Y, ws)
    moe.moe_combine(Y, inv, w, y)
    flags = moe.moe_device_status(ws)
    assert flags == 0, f"device status flags {flags:#x}"
    return dict(idx=idx, w=w, offsets=off, perm_token=pt, inv_perm=inv, x_perm=xp, Y=Y, y=y,
                ws=ws)


def layer_y(inp):
    x = inp["x"]
    T, d = x.shape
    E, h, _ = inp["W1"].shape
    ws = moe.alloc_workspace(T, d, h, E, 2, x.dtype, x.device)
    y = moe.layer_forward(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], ws=ws)
    assert moe.moe_device_status(ws) == 0
    return y


def check_routing_and_permutation(g, x_cpu, Wg_cpu, E):
    logits = O.router_logits(x_cpu, Wg_cpu)
    idx = O.top2_select(logits)
    np.testing.assert_array_equal(g["idx"].cpu().numpy(), idx)
    w_ref = O.gate_weights_f32(logits, idx)
    w_gpu = g["w"].cpu().numpy()
    ulp = np.spacing(w_ref)
    assert (np.abs(w_gpu - w_ref) <= 2 * ulp).all()
    assert ((w_gpu[:, 0] + w_gpu[:, 1]) == np.float32(1)).all()
    off, pt, inv = O.permutation(idx, E)
    np.testing.assert_array_equal(g["offsets"].cpu().numpy(), off)
    np.testing.assert_array_equal(g["perm_token"].cpu().numpy(), pt)
    np.testing.assert_array_equal(g["inv_perm"].cpu().numpy(), inv)
    return logits, idx, off, pt, inv


SMALL = [  # (T, d, h, kind): ragged row blocks, K tails, N tails, empty groups
    # T <= 128 runs the weight-streaming kernels (token tiles of 16, 32, 64 or 128)
    (1, 64, 128, "plain"), (2, 64, 128, "plain"), (3, 128, 256, "plain"),
    (5, 136, 200, "plain"), (16, 256, 384, "skew"), (17, 128, 256, "plain"),
    (33, 128, 256, "plain"), (64, 256, 512, "plain"), (65, 128, 256, "plain"),
    (100, 136, 200, "skew"), (128, 256, 512, "plain"),
    # 128 < T < 512 runs the single-SM grouped GEMM (128-row blocks); h a multiple of
    # 112 selects its 112-output GEMM1 tiles
    (129, 256, 512, "plain"), (300, 136, 200, "plain"), (511, 128, 256, "skew"),
    (200, 128, 224, "plain"), (300, 256, 448, "skew"), (450, 136, 336, "long"),
    # ... at larger d and h: many K blocks per tile, ragged K (1000 = 15 x 64 + 40)
    (300, 1000, 1792, "plain"), (400, 1024, 2048, "skew"), (160, 512, 3584, "long"),
    # >= 1024 grouped rows run the CTA-pair grouped GEMM (256-row blocks; an expert's
    # last block of <= 128 rows runs in the pair's 128-row mode)
    (512, 128, 256, "plain"), (513, 128, 256, "long"), (700, 256, 384, "skew"),
    (1000, 512, 1024, "plain"), (1100, 256, 384, "plain"), (1500, 136, 200, "skew"),
    (2500, 128, 256, "long"),
]


@pytest.mark.parametrize("T,d,h,kind", SMALL)
def test_layer_bf16_small_shapes(T, d, h, kind):
    wl = small("p", T=T, d=d, h=h, seed=100 + T, kind=kind)
    inp = make_inputs(wl, "cuda")
    g = run_steps(inp, wl.E)
    x_cpu = f64(inp["x"])
    logits, idx, off, pt, inv = check_routing_and_permutation(g, x_cpu, f64(inp["Wg"]), wl.E)
    # gathered rows: byte-identical to x[perm_token]
    np.testing.assert_array_equal(raw16(g["x_perm"]), O.gather_rows(raw16(inp["x"]), pt))
    ref = O.moe_layer(x_cpu, f64(inp["Wg"]), f64(inp["W1"]), f64(inp["W3"]), f64(inp["W2"]))
    Y = g["Y"].double().cpu().numpy()
    assert rel_fro(Y, ref["Y"]) <= BF16_TOL
    y = f64(g["y"])
    err = rel_fro(y, ref["y"])
    assert err <= BF16_TOL, err
    assert worst_token(y, ref["y"]) <= TOKEN_TOL
    # the fused entry point runs the same kernels (above 512 tokens the router also
    # counts the grouping, so the count pass is skipped): identical bits
    assert torch.equal(layer_y(inp), g["y"])


def gemm2_width(row_blocks, d, grid=148):
    """The single-SM GEMM2 tile width the kernel picks: the width w of 256, 224, 192, 160
    or 128 columns that minimises rounds(row_blocks * ceil(d / w) tiles) * (128 + w)."""
    best, best_cost = 256, None
    for w in (256, 224, 192, 160, 128):
        cost = -(-row_blocks * -(-d // w) // grid) * (128 + w)
        if best_cost is None or cost < best_cost:
            best, best_cost = w, cost
    return best


@pytest.mark.parametrize("sizes,width", [
    ([100] * 8, 256),                                   # 8 row blocks: one round
    ([200, 200, 60, 60, 60, 60, 60, 60], 160),          # 10 row blocks
    ([200, 200, 200, 200, 50, 50, 50, 50], 192),        # 12
    ([129] * 6 + [100, 100], 224),                      # 14, single-row second blocks
    ([300, 0, 0, 250, 130, 100, 100, 100], 160),        # empty groups, 10 row blocks
])
def test_grouped_ffn_every_gemm2_tile_width(sizes, width):
    """The grouped expert FFN (257..1023 rows) on crafted group sizes whose row-block
    counts make the kernel's GEMM2 take each of its tile widths (ragged last column
    tile: d = 4096 is no multiple of 160, 192 or 224), against the fp64 oracle."""
    d, h, E = 4096, 256, 8
    blocks = sum(-(-n // 128) for n in sizes)
    assert gemm2_width(blocks, d) == width
    wl = small("g2w", T=16, d=d, h=h, seed=70 + blocks)
    inp = make_inputs(wl, "cuda")
    P = sum(sizes)
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 + blocks)
    xp = torch.randn(P, d, generator=g).to(torch.bfloat16).cuda()
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32,
                       device="cuda")
    ws = moe.alloc_workspace(P // 2, d, h, E, 2, torch.bfloat16, "cuda")
    Y = torch.full((P, d), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn(xp, off, inp["W1"], inp["W3"], inp["W2"], Y, ws)
    assert moe.moe_device_status(ws) == 0
    ref = O.expert_ffn_grouped(xp.float().cpu().numpy(), off.cpu().numpy(),
                               PerExpert(inp["W1"]), PerExpert(inp["W3"]), PerExpert(inp["W2"]))
    got = Y.double().cpu().numpy()
    assert np.isfinite(got).all()
    err = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    print(f"GEMM2_WIDTH {width} blocks={blocks} rel_fro={err:.3e}")
    assert err <= 5e-3


def test_router_counts_are_cleared_between_calls():
    """Above 512 tokens the router accumulates the grouping's per-chunk counts in the
    workspace and the scan clears them: repeated layer calls on one workspace,
    interleaved with a smaller batch (one-launch grouping) and with the step-wise
    moe_permute (its own count pass), reproduce the first result bit for bit."""
    wl = small("cnt", T=1300, d=256, h=384, seed=11, kind="skew")
    inp = make_inputs(wl, "cuda")
    sub = {k: (v[:700].contiguous() if k == "x" else v) for k, v in inp.items()}
    small_b = {k: (v[:300].contiguous() if k == "x" else v) for k, v in inp.items()}
    ref, ref_sub, ref_small = layer_y(inp), layer_y(sub), layer_y(small_b)
    ws = moe.alloc_workspace(1300, 256, 384, wl.E, 2, torch.bfloat16, "cuda")
    for _ in range(3):
        for b, r in ((inp, ref), (sub, ref_sub), (small_b, ref_small)):
            y = torch.full_like(b["x"], float("nan"))
            moe.moe_layer_forward(b["x"], b["Wg"], b["W1"], b["W3"], b["W2"], y, ws)
            assert torch.equal(y, r)
        g = run_steps(sub, wl.E)  # step-wise entry points on a fresh workspace
        assert torch.equal(g["y"], ref_sub)
    assert moe.moe_device_status(ws) == 0


@pytest.mark.parametrize("T,kind", [(1, "plain"), (16, "skew"), (40, "plain"), (64, "skew"),
                                    (100, "plain"), (128, "skew")])
def test_small_batch_layer_repeated_calls(T, kind):
    """The small-batch expert FFN is one cooperative launch whose dependency counters
    must be zero again after every call: repeated calls on one workspace, interleaved
    with a smaller batch, each into an output pre-filled with NaN, reproduce the
    step-wise result bit for bit."""
    wl = small("rep", T=T, d=256, h=384, seed=900 + T, kind=kind)
    inp = make_inputs(wl, "cuda")
    x, Wg, W1, W3, W2 = (inp[k] for k in ("x", "Wg", "W1", "W3", "W2"))
    Ts = max(1, T // 3)
    sub = {k: (v[:Ts].contiguous() if k == "x" else v) for k, v in inp.items()}
    ref = run_steps(inp, wl.E)["y"]
    ref_sub = run_steps(sub, wl.E)["y"]
    ws = moe.alloc_workspace(T, 256, 384, wl.E, 2, x.dtype, x.device)
    for _ in range(3):
        y = torch.full_like(x, float("nan"))
        moe.moe_layer_forward(x, Wg, W1, W3, W2, y, ws)
        assert torch.equal(y, ref)
        y_sub = torch.full_like(sub["x"], float("nan"))
        moe.moe_layer_forward(sub["x"], Wg, W1, W3, W2, y_sub, ws)
        assert torch.equal(y_sub, ref_sub)
    assert moe.moe_device_status(ws) == 0


@pytest.mark.parametrize("T,d,h", [(64, 128, 256), (1, 8, 8), (37, 24, 40), (300, 64, 96)])
def test_layer_f32(T, d, h):
    wl = WORKLOADS["tiny_f32"] if (T, d, h) == (64, 128, 256) else small(
        "f", T=T, d=d, h=h, dtype="f32", seed=T)
    inp = make_inputs(wl, "cuda")
    g = run_steps(inp, wl.E)
    x_cpu = f64(inp["x"])
    check_routing_and_permutation(g, x_cpu, f64(inp["Wg"]), wl.E)
    ref = O.moe_layer(x_cpu, f64(inp["Wg"]), f64(inp["W1"]), f64(inp["W3"]), f64(inp["W2"]))
    err = rel_fro(f64(g["y"]), ref["y"])
    assert err <= F32_TOL, err
    assert torch.equal(layer_y(inp), g["y"])


def test_route_ties_pick_lower_index():
    wl = small("tie", T=33, d=64, h=64)
    inp = make_inputs(wl, "cuda")
    inp["Wg"][:] = inp["Wg"][:, :1].clone()
    g = run_steps(inp, 8)
    assert (g["idx"].cpu() == torch.tensor([0, 1], dtype=torch.int32)).all()
    assert (g["w"].cpu() == 0.5).all()


def test_empty_batch_is_a_noop():
    x = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    Wg = torch.zeros(64, 8, dtype=torch.bfloat16, device="cuda")
    W1 = torch.zeros(8, 64, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(x)
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward(x, Wg, W1, W1, W1, y, ws)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T", [16, 257])  # weight-streaming and grouped-GEMM kernels
def test_exact_invariants_on_gpu(T):
    """Bit-exact properties that need no oracle: W2 x 2 doubles y; permuting tokens
    permutes y; relabelling experts consistently leaves y unchanged."""
    wl = small("inv", T=T, d=256, h=384, seed=77)
    inp = make_inputs(wl, "cuda")
    y = layer_y(inp)
    s = dict(inp, W2=inp["W2"] * 2)
    assert torch.equal(layer_y(s), y * 2)
    p = torch.randperm(T, generator=torch.Generator().manual_seed(0)).cuda()
    s = dict(inp, x=inp["x"][p].contiguous())
    assert torch.equal(layer_y(s), y[p])
    q = torch.tensor([3, 7, 0, 5, 1, 6, 2, 4], device="cuda")
    s = dict(inp, Wg=inp["Wg"][:, q].contiguous(), W1=inp["W1"][q].contiguous(),
             W3=inp["W3"][q].contiguous(), W2=inp["W2"][q].contiguous())
    assert torch.equal(layer_y(s), y)


@pytest.mark.parametrize("name,T", [("decode", None), ("prefill", None), ("skew", None),
                                    ("long", None),
                                    # batches between the two: single-SM grouped GEMMs
                                    # (511 tokens: 13 row blocks, 192-column GEMM2 tiles)
                                    ("prefill", 192), ("prefill", 511), ("skew", 256),
                                    ("skew", 384)])
def test_full_size_workloads(name, T):
    """The Mixtral-8x7B-shaped workloads at full size: routing and permutation over all
    tokens, gathered rows byte-exact, and y against the fp64 oracle over every token
    (relative Frobenius error of the whole output, and every token's own error).  A
    sample of tokens is checked first, so a gross error fails in seconds."""
    wl = WORKLOADS[name] if T is None else WORKLOADS[name].with_tokens(T)
    inp = make_inputs(wl, "cuda")
    g = run_steps(inp, wl.E)
    x_cpu = inp["x"].float().cpu().numpy()
    Wg_cpu = inp["Wg"].float().cpu().numpy()
    logits, idx, off, pt, inv = check_routing_and_permutation(g, x_cpu, Wg_cpu, wl.E)
    np.testing.assert_array_equal(raw16(g["x_perm"]), O.gather_rows(raw16(inp["x"]), pt))
    counts = np.diff(off)
    if name == "skew":
        assert counts[6] + counts[7] <= 0.01 * 2 * wl.T and counts[0] == counts.max()
    assert torch.equal(layer_y(inp), g["y"])
    W1, W3, W2 = PerExpert(inp["W1"]), PerExpert(inp["W3"]), PerExpert(inp["W2"])
    y_all = f64(g["y"])
    del g
    # fast pre-check on sampled tokens
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, min(wl.T, 64),
                                                                  replace=False)]))
    ref = O.moe_layer(x_cpu[sample], Wg_cpu, W1, W3, W2)
    assert rel_fro(y_all[sample], ref["y"]) <= BF16_TOL
    assert worst_token(y_all[sample], ref["y"]) <= TOKEN_TOL
    # the whole output
    ref = O.moe_layer(x_cpu, Wg_cpu, W1, W3, W2)["y"]
    err, tok = rel_fro(y_all, ref), worst_token(y_all, ref)
    print(f"PARITY {name} T={wl.T}: rel_fro(y) over all {wl.T} tokens = {err:.3e}, "
          f"worst token = {tok:.3e}")
    assert err <= BF16_TOL, err
    assert tok <= TOKEN_TOL, tok


@pytest.mark.parametrize("T", [40, 700])  # one-launch and four-launch permutation paths
def test_out_of_range_expert_ids_are_flagged(T):
    """Expert ids outside [0, E) are skipped by the permutation kernels' bounds checks
    and reported through the workspace status word (flag 0x2)."""
    d, E = 64, 8
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    idx = torch.randint(0, E, (T, 2), dtype=torch.int32, device="cuda")
    idx[:, 1] = (idx[:, 0] + 1) % E
    idx[3, 1] = E + 5
    idx[T - 1, 0] = -2
    ws = moe.alloc_workspace(T, d, 64, E, 2, torch.bfloat16)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pt = torch.full((2 * T,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((T, 2), -7, dtype=torch.int32, device="cuda")
    xp = torch.zeros(2 * T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(idx, x, off, pt, inv, xp, ws, E)
    assert moe.moe_device_status(ws) & 0x2
    assert int(off[-1]) == 2 * T - 2  # the two bad pairs are left out
    assert int(inv[3, 1]) == -7 and int(inv[T - 1, 0]) == -7


@pytest.mark.parametrize("E", [2, 4, 16, 32])
@pytest.mark.parametrize("T", [40, 300, 700])  # weight-streaming, grouped and pair kernels;
                                                # above 512 tokens the router counts the
                                                # grouping for E <= 8
def test_other_expert_counts(E, T):
    """The layer for E other than 8 (the ABI allows 2..32): routing and permutation
    bit-exact, output within the bf16 tolerance."""
    wl = small("e", T=T, d=128, h=256, E=E, seed=E * 1000 + T)
    inp = make_inputs(wl, "cuda")
    g = run_steps(inp, E)
    x_cpu = f64(inp["x"])
    check_routing_and_permutation(g, x_cpu, f64(inp["Wg"]), E)
    ref = O.moe_layer(x_cpu, f64(inp["Wg"]), f64(inp["W1"]), f64(inp["W3"]), f64(inp["W2"]))
    assert rel_fro(f64(g["y"]), ref["y"]) <= BF16_TOL
    assert torch.equal(layer_y(inp), g["y"])


def capped_y(inp, capacity):
    x = inp["x"]
    T, d = x.shape
    E, h, _ = inp["W1"].shape
    ws = moe.alloc_workspace(T, d, h, E, 2, x.dtype, x.device)
    y = torch.empty_like(x)
    moe.moe_layer_forward_capacity(x, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], y, ws,
                                   capacity)
    assert moe.moe_device_status(ws) == 0
    return y


@pytest.mark.parametrize("T,d,h,kind,cap,dtype", [
    (16, 256, 384, "skew", 3, "bf16"),       # fused weight-streaming kernel
    (40, 128, 256, "skew", 5, "bf16"),
    (100, 128, 256, "skew", 12, "bf16"),     # fused kernel, 128-token tiles
    (300, 136, 200, "skew", 40, "bf16"),     # single-SM grouped GEMM
    (1500, 136, 200, "skew", 300, "bf16"),   # CTA-pair grouped GEMM (half tiles too)
    (1100, 256, 384, "plain", 260, "bf16"),
    (64, 128, 256, "skew", 10, "f32"),       # fp32 CUDA-core FFN
])
def test_capacity_layer(T, d, h, kind, cap, dtype):
    """Opt-in capacity: each expert keeps its first `cap` pairs in token order."""
    wl = small("cap", T=T, d=d, h=h, seed=300 + T, kind=kind, dtype=dtype)
    inp = make_inputs(wl, "cuda")
    y = f64(capped_y(inp, cap))
    c = {k: f64(v) for k, v in inp.items()}
    ref = O.moe_layer(c["x"], c["Wg"], c["W1"], c["W3"], c["W2"], capacity=cap)
    assert not ref["keep"].all()  # the cap really drops pairs here
    tol = F32_TOL if dtype == "f32" else BF16_TOL
    assert rel_fro(y, ref["y"]) <= tol
    assert worst_token(y, ref["y"]) <= (tol if dtype == "f32" else TOKEN_TOL)


@pytest.mark.parametrize("T", [16, 300, 1500])
def test_capacity_special_cases_on_gpu(T):
    wl = small("cap0", T=T, d=128, h=256, seed=7, kind="skew")
    inp = make_inputs(wl, "cuda")
    y_full = layer_y(inp)
    assert torch.equal(capped_y(inp, 2 * T), y_full)  # no group exceeds 2T rows
    assert torch.equal(capped_y(inp, -1), y_full)     # negative: no limit
    assert (capped_y(inp, 0) == 0).all()


def test_capacity_full_size_skewed():
    """Skewed Mixtral-shaped workload at capacity factor 1.25 (1280 rows per expert):
    expert 0 (~3500 rows) is cut; sampled tokens against the fp64 oracle."""
    wl = WORKLOADS["skew"]
    cap = O.capacity_from_factor(1.25, wl.T, 2, wl.E)
    inp = make_inputs(wl, "cuda")
    y = capped_y(inp, cap)
    x_cpu = inp["x"].float().cpu().numpy()
    Wg_cpu = inp["Wg"].float().cpu().numpy()
    idx = O.top2_select(O.router_logits(x_cpu, Wg_cpu))
    keep = O.capacity_keep(idx, wl.E, cap)
    assert (~keep).sum() > 1000
    rng = np.random.default_rng(1)
    sample = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, 64, replace=False)]))
    # the oracle's capacity decision needs every token's routing; apply it per sample
    w = O.gate_weights(O.router_logits(x_cpu[sample], Wg_cpu), idx[sample]) * keep[sample]
    ref = np.zeros((len(sample), wl.d))
    for j in range(2):
        for e in range(wl.E):
            rows = np.nonzero(idx[sample, j] == e)[0]
            if len(rows):
                ref[rows] += w[rows, j:j + 1] * O.expert_swiglu(
                    x_cpu[sample][rows], inp["W1"][e].float().cpu().numpy(),
                    inp["W3"][e].float().cpu().numpy(), inp["W2"][e].float().cpu().numpy())
    got = y[torch.as_tensor(sample, device="cuda")].double().cpu().numpy()
    assert rel_fro(got, ref) <= BF16_TOL
    assert worst_token(got, ref) <= TOKEN_TOL
