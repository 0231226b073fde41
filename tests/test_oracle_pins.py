"""Pins for the CPU oracle: closed forms, brute force, invariants and the pages' numbers.

Each test checks the oracle against something other than itself:
* the top-2 choice against an exhaustive search over all expert pairs;
* the gate against its closed form (a two-way softmax is a logistic function) and
  against the other way the pages write it (softmax, top-2, renormalise);
* the whole layer against a hand-derived closed-form case whose sigmoid values are
  exact (sigma(ln 3) = 3/4, sigma(ln 7) = 7/8), against a brute-force layer that
  evaluates every expert and masks with the dense gate, and against an
  independent plain-C loop implementation;
* the permutation against its definition written as loops;
* the shapes against the parameter counts the pages print.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs, small

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(t):
    return t.double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


def _inputs(w):
    return {k: _np(v) for k, v in make_inputs(w, "cpu").items()}


# ---------------------------------------------------------------- routing

def _pair_bruteforce(l):
    """Best expert pair by exhaustive search: largest l_a + l_b, ties -> smallest indices;
    slot 0 is the larger logit (ties -> lower index)."""
    best = None
    for a, b in itertools.combinations(range(len(l)), 2):
        key = (l[a] + l[b], -a, -b)
        if best is None or key > best[0]:
            best = (key, a, b)
    _, a, b = best
    return (a, b) if (l[a] > l[b] or (l[a] == l[b] and a < b)) else (b, a)


def test_top2_matches_pair_bruteforce_with_ties():
    rng = np.random.default_rng(7)
    # small integers make exact ties frequent
    logits = rng.integers(-3, 4, size=(400, 8)).astype(np.float64)
    logits[:50] = rng.standard_normal((50, 8))
    idx = O.top2_select(logits)
    for t in range(logits.shape[0]):
        assert tuple(idx[t]) == _pair_bruteforce(list(logits[t])), t


def test_top2_all_equal_picks_first_two():
    idx = O.top2_select(np.zeros((3, 8)))
    assert idx.tolist() == [[0, 1]] * 3


def test_gate_closed_form_exact_values():
    # l1 - l2 = ln 3 -> (3/4, 1/4); ln 7 -> (7/8, 1/8); equal -> (1/2, 1/2)
    logits = np.array([[math.log(3.0), 0, -1, -2, -3, -4, -5, -6],
                       [-1, -2, 0, 0, -3, -4, -5, math.log(7.0)],
                       [0.25] * 8])
    idx = O.top2_select(logits)
    assert idx.tolist() == [[0, 1], [7, 2], [0, 1]]
    w = O.gate_weights(logits, idx)
    np.testing.assert_allclose(w, [[0.75, 0.25], [0.875, 0.125], [0.5, 0.5]], rtol=1e-15)


def test_gate_dense_forms_agree_and_are_logistic():
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((300, 8)) * 3
    G3 = O.gate_dense_topk_softmax(logits)          # -inf mask, then softmax
    G2 = O.gate_dense_softmax_topk_renorm(logits)   # softmax, top-2, renormalise
    np.testing.assert_allclose(G3, G2, rtol=0, atol=1e-15)
    idx = O.top2_select(logits)
    w = O.gate_weights(logits, idx)
    rows = np.arange(300)[:, None]
    np.testing.assert_allclose(G3[rows, idx], w, rtol=0, atol=1e-15)
    # exactly two non-zero weights, summing to one, the larger on slot 0
    assert ((G3 > 0).sum(axis=1) == 2).all()
    np.testing.assert_allclose(G3.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert (w[:, 0] >= 0.5).all()
    # logistic closed form of the larger weight
    l = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(w[:, 0], 1 / (1 + np.exp(-(l[:, 0] - l[:, 1]))), rtol=1e-15)


def test_gate_f32_pair_sums_to_one_exactly():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((1000, 8)) * 4
    idx = O.top2_select(logits)
    wf = O.gate_weights_f32(logits, idx)
    assert wf.dtype == np.float32
    assert ((wf[:, 0] + wf[:, 1]) == np.float32(1.0)).all()
    assert (wf[:, 0] >= 0.5).all()
    np.testing.assert_allclose(wf[:, 0], O.gate_weights(logits, idx)[:, 0], rtol=6e-8)


def test_identical_router_columns_tie_to_experts_0_and_1():
    w = small("tie", T=9, d=16, h=8)
    inp = _inputs(w)
    inp["Wg"][:] = inp["Wg"][:, :1]
    out = O.moe_layer(**inp)
    assert out["idx"].tolist() == [[0, 1]] * 9
    np.testing.assert_array_equal(out["w"], 0.5)


# ---------------------------------------------------------------- permutation

def _perm_by_loops(idx, E):
    T, k = idx.shape
    rows = []
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    rows.append((t, j))
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + sum(1 for t in range(T) for j in range(k) if idx[t, j] == e))
    inv = np.zeros((T, k), np.int64)
    for r, (t, j) in enumerate(rows):
        inv[t, j] = r
    return np.array(offsets), np.array([t for t, _ in rows]), inv


@pytest.mark.parametrize("T,E", [(1, 8), (2, 8), (37, 8), (200, 8), (64, 3)])
def test_permutation_matches_loop_definition(T, E):
    rng = np.random.default_rng(T * 10 + E)
    logits = rng.standard_normal((T, E))
    logits[:, E - 1] -= 5.0  # makes the last expert rare or empty
    idx = O.top2_select(logits)
    off, pt, inv = O.permutation(idx, E)
    off2, pt2, inv2 = _perm_by_loops(idx, E)
    np.testing.assert_array_equal(off, off2)
    np.testing.assert_array_equal(pt, pt2)
    np.testing.assert_array_equal(inv, inv2)


def test_permutation_invariants():
    rng = np.random.default_rng(3)
    T, E = 513, 8
    idx = O.top2_select(rng.standard_normal((T, E)))
    off, pt, inv = O.permutation(idx, E)
    P = 2 * T
    assert off[0] == 0 and off[-1] == P and (np.diff(off) >= 0).all()
    assert sorted(inv.ravel().tolist()) == list(range(P))  # bijection
    for e in range(E):
        toks = pt[off[e]:off[e + 1]]
        assert (np.diff(toks) > 0).all()  # ascending, no token twice in a group
        for t in toks:
            assert e in idx[t]
    for t in range(T):
        for j in range(2):
            r = inv[t, j]
            assert pt[r] == t and off[idx[t, j]] <= r < off[idx[t, j] + 1]


# ---------------------------------------------------------------- whole layer

def closed_form_case():
    """T=2, d=2, h=3, E=8 with exactly known sigmoids; returns (inputs, idx, w, y)."""
    ln3, ln7 = math.log(3.0), math.log(7.0)
    rng = np.random.default_rng(11)
    d, h, E = 2, 3, 8
    x = np.array([[1.0, 0.0], [0.0, 1.0]])
    Wg = np.array([[ln3, 0, -1, -2, -3, -4, -5, -6],
                   [-1, -2, 0, 0, -3, -4, -5, ln7]])
    W1 = rng.integers(-4, 5, size=(E, h, d)) * 0.37
    W3 = rng.integers(-4, 5, size=(E, h, d)) * 0.29
    W2 = rng.integers(-4, 5, size=(E, d, h)) * 0.41
    # token 0 (x = e_0): experts 0 (w 3/4) and 1 (w 1/4)
    W1[0][:, 0] = [ln3, 0, -ln3]
    W3[0][:, 0] = [2, 5, 4]
    W2[0] = [[1, 7, 1], [2, 0, -1]]
    W1[1][:, 0] = [0, ln3, ln3]
    W3[1][:, 0] = [1, 1, -2]
    W2[1] = [[1, 1, 1], [0, 2, 1]]
    # token 1 (x = e_1): experts 7 (w 7/8) and 2 (w 1/8; 2 beats 3 on a tie)
    W1[7][:, 1] = [ln7, 0, 0]
    W3[7][:, 1] = [8, 3, 3]
    W2[7] = [[1, 0, 0], [0, 1, 1]]
    W1[2][:, 1] = [0, 0, -ln7]
    W3[2][:, 1] = [1, 1, 8]
    W2[2] = [[0, 0, 1], [1, 1, 0]]
    # by hand: E0(x0) = (ln3/2, 4 ln3), E1(x0) = (-3 ln3/4, 0),
    #          E7(x1) = (7 ln7, 0),     E2(x1) = (-ln7, 0)
    y = np.array([[3 * ln3 / 16, 3 * ln3], [6 * ln7, 0.0]])
    inputs = dict(x=x, Wg=Wg, W1=W1, W3=W3, W2=W2)
    return inputs, [[0, 1], [7, 2]], [[0.75, 0.25], [0.875, 0.125]], y


def _closed_form_holds(layer=O.moe_layer):
    inp, idx, w, y = closed_form_case()
    out = layer(**inp)
    return (out["idx"].tolist() == idx and np.allclose(out["w"], w, rtol=1e-14, atol=0)
            and np.allclose(out["y"], y, rtol=1e-13, atol=1e-15))


def test_layer_closed_form():
    inp, idx, w, y = closed_form_case()
    out = O.moe_layer(**inp)
    assert out["idx"].tolist() == idx
    np.testing.assert_allclose(out["w"], w, rtol=1e-14)
    np.testing.assert_allclose(out["y"], y, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(O.moe_layer_dense(**inp), y, rtol=1e-13, atol=1e-15)
    _, _, yl = oracle.loops_layer(**inp)
    np.testing.assert_allclose(yl, y, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("mistake", ["silu_on_w3", "no_silu", "drop_second", "dense_softmax",
                                     "tie_to_higher", "w_swapped", "sigmoid_sign"])
def test_planted_mistakes_are_caught(monkeypatch, mistake):
    """Each plausible slip, planted in the oracle, breaks the closed-form pin."""
    if mistake == "silu_on_w3":
        def sw(xr, W1e, W3e, W2e):
            xr = np.asarray(xr, np.float64)
            return ((xr @ W1e.T) * O.silu(xr @ W3e.T)) @ W2e.T
        monkeypatch.setattr(O, "expert_swiglu", sw)
    elif mistake == "no_silu":
        monkeypatch.setattr(O, "silu", lambda z: np.asarray(z, np.float64))
    elif mistake == "drop_second":
        orig = O.combine
        monkeypatch.setattr(O, "combine", lambda Y, inv, w: orig(Y, inv[:, :1], w[:, :1]))
    elif mistake == "dense_softmax":
        def gw(l, idx):
            p = np.exp(l - l.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            return np.take_along_axis(p, idx.astype(np.int64), axis=1)
        monkeypatch.setattr(O, "gate_weights", gw)
    elif mistake == "tie_to_higher":
        def ts(l, k=2):
            l = np.asarray(l, np.float64)[:, ::-1]
            order = np.argsort(-l, axis=1, kind="stable")[:, :k]
            return (l.shape[1] - 1 - order).astype(np.int32)
        monkeypatch.setattr(O, "top2_select", ts)
    elif mistake == "w_swapped":
        orig = O.gate_weights
        monkeypatch.setattr(O, "gate_weights", lambda l, idx: orig(l, idx)[:, ::-1])
    elif mistake == "sigmoid_sign":
        monkeypatch.setattr(O, "silu", lambda z: np.asarray(z) / (1.0 + np.exp(np.asarray(z))))
    assert not _closed_form_holds()


def test_routed_equals_bruteforce_on_tiny_workload():
    inp = _inputs(WORKLOADS["tiny_f32"])
    out = O.moe_layer(**inp)
    yd = O.moe_layer_dense(**inp)
    err = np.linalg.norm(out["y"] - yd) / np.linalg.norm(yd)
    assert err < 1e-13


@pytest.mark.parametrize("T,d,h,kind", [(1, 8, 8, "plain"), (3, 16, 24, "plain"),
                                        (37, 24, 40, "skew"), (129, 32, 16, "long")])
def test_routed_equals_bruteforce_small_shapes(T, d, h, kind):
    inp = _inputs(small("s", T=T, d=d, h=h, seed=T, kind=kind))
    out = O.moe_layer(**inp)
    yd = O.moe_layer_dense(**inp)
    assert np.linalg.norm(out["y"] - yd) <= 1e-13 * np.linalg.norm(yd)
    if kind == "skew":
        counts = np.diff(out["offsets"])
        assert counts[0] == counts.max()


def test_loops_oracle_equals_routed_on_tiny_workload():
    inp = _inputs(WORKLOADS["tiny_f32"])
    out = O.moe_layer(**inp)
    idx, w, y = oracle.loops_layer(**inp)
    np.testing.assert_array_equal(idx, out["idx"])
    np.testing.assert_allclose(w, out["w"], rtol=1e-15)
    assert np.linalg.norm(y - out["y"]) <= 1e-13 * np.linalg.norm(out["y"])


def test_identical_experts_reduce_to_one_dense_swiglu():
    """With all experts equal the gate weights sum to one, so the layer is one FFN."""
    inp = _inputs(small("same", T=23, d=16, h=24, seed=5))
    for name in ("W1", "W3", "W2"):
        inp[name][:] = inp[name][3]
    out = O.moe_layer(**inp)
    x = inp["x"]
    a = x @ inp["W1"][0].T
    b = x @ inp["W3"][0].T
    dense = (a * (1.0 / (1.0 + np.exp(-a))) * b) @ inp["W2"][0].T
    np.testing.assert_allclose(out["y"], dense, rtol=1e-12, atol=1e-14)


def test_scaling_and_equivariance():
    inp = _inputs(small("eq", T=31, d=16, h=24, seed=9))
    base = O.moe_layer(**inp)["y"]
    # W2 x 2 (or W3 x 2) doubles y
    for name in ("W2", "W3"):
        s = dict(inp)
        s[name] = inp[name] * 2.0
        np.testing.assert_allclose(O.moe_layer(**s)["y"], 2 * base, rtol=1e-13, atol=1e-15)
    # permuting tokens permutes the output
    p = np.random.default_rng(0).permutation(31)
    s = dict(inp)
    s["x"] = inp["x"][p]
    np.testing.assert_allclose(O.moe_layer(**s)["y"], base[p], rtol=1e-13, atol=1e-15)
    # relabelling experts consistently leaves y unchanged
    q = np.random.default_rng(1).permutation(8)
    s = dict(inp)
    s["Wg"] = inp["Wg"][:, q]
    for name in ("W1", "W3", "W2"):
        s[name] = inp[name][q]
    np.testing.assert_allclose(O.moe_layer(**s)["y"], base, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- shapes

def _golden_counts():
    vals = {}
    with open(os.path.join(GOLDEN, "mixtral_param_counts.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v, dec = line.split()
                vals[k] = (float(v), int(dec))
    return vals


def test_param_counts_match_the_pages():
    c = O.mixtral_param_counts()
    g = _golden_counts()
    for key, n in (("total", c["total"]), ("active", c["active"])):
        for src in ("glossary", "summary"):
            v, dec = g[f"{key}_{src}"]
            assert round(n / 1e9, dec) == v, (key, src, n)
    assert c["total"] == 46_702_792_704 and c["active"] == 12_879_925_248


# ---------------------------------------------------------------- capacity (opt-in)

def _capped_by_loops(inp, capacity):
    """Per token, by loops: keep pair (t, j) iff fewer than `capacity` earlier pairs
    (in token, then slot order) went to the same expert; sum the kept experts."""
    l = O.router_logits(inp["x"], inp["Wg"])
    idx = O.top2_select(l)
    w = O.gate_weights(l, idx)
    E = inp["Wg"].shape[1]
    seen = [0] * E
    y = np.zeros(inp["x"].shape)
    for t in range(idx.shape[0]):
        for j in range(2):
            e = int(idx[t, j])
            if seen[e] < capacity:
                y[t] += w[t, j] * O.expert_swiglu(inp["x"][t:t + 1], inp["W1"][e], inp["W3"][e],
                                                  inp["W2"][e])[0]
            seen[e] += 1
    return y


@pytest.mark.parametrize("capacity", [0, 1, 3, 7, 1000])
def test_capacity_matches_per_token_loops(capacity):
    inp = _inputs(small("cap", T=29, d=16, h=24, seed=4, kind="skew"))
    out = O.moe_layer(**inp, capacity=capacity)
    np.testing.assert_allclose(out["y"], _capped_by_loops(inp, capacity), rtol=1e-12, atol=1e-14)


def test_capacity_special_cases():
    inp = _inputs(small("cap2", T=40, d=16, h=24, seed=6, kind="skew"))
    full = O.moe_layer(**inp)
    counts = np.diff(full["offsets"])
    # a capacity at or above every group's size changes nothing
    big = O.moe_layer(**inp, capacity=int(counts.max()))
    np.testing.assert_array_equal(big["y"], full["y"])
    assert big["keep"].all()
    # capacity 0 drops everything
    np.testing.assert_array_equal(O.moe_layer(**inp, capacity=0)["y"], 0.0)
    # the number of kept pairs per expert is min(count, capacity)
    for c in (1, 4, 9):
        keep = O.capacity_keep(full["idx"], 8, c)
        kept = np.bincount(full["idx"][keep].ravel(), minlength=8)
        np.testing.assert_array_equal(kept, np.minimum(counts, c))
    assert O.capacity_from_factor(1.0, 4096, 2, 8) == 1024
    assert O.capacity_from_factor(1.25, 4096, 2, 8) == 1280
    assert O.capacity_from_factor(1.25, 10, 2, 8) == 4


# ---------------------------------------------------------------- backward (training)

def _fd_case(seed=1, T=4, d=5, h=3, E=4):
    rng = np.random.default_rng(seed)
    return dict(x=rng.normal(size=(T, d)), Wg=rng.normal(size=(d, E)),
                W1=rng.normal(size=(E, h, d)) / 2, W3=rng.normal(size=(E, h, d)) / 2,
                W2=rng.normal(size=(E, d, h)) / 2), rng.normal(size=(T, d))


def _finite_differences(inp, dy, capacity=None, eps=1e-6):
    """Central differences of L = sum(dy * y) with respect to every input entry."""
    names = ("x", "Wg", "W1", "W3", "W2")

    def loss(args):
        return float((O.moe_layer(*args, capacity=capacity)["y"] * dy).sum())

    out = {}
    for i, n in enumerate(names):
        A = inp[n]
        fd = np.zeros_like(A)
        for ix in np.ndindex(A.shape):
            plus = [inp[m].copy() for m in names]
            minus = [inp[m].copy() for m in names]
            plus[i][ix] += eps
            minus[i][ix] -= eps
            fd[ix] = (loss(plus) - loss(minus)) / (2 * eps)
        out["d" + n] = fd
    return out


def _fd_agrees(g, fd, tol=1e-7):
    return all(np.abs(fd[k] - g[k]).max() <= tol * max(np.abs(fd[k]).max(), 1e-12)
               for k in fd)


@pytest.mark.parametrize("capacity", [None, 1])
def test_backward_matches_finite_differences(capacity):
    """The top-2 choice is held fixed: random inputs keep every logit gap far above
    the step, so central differences of the forward oracle pin every gradient."""
    inp, dy = _fd_case()
    g = O.moe_layer_backward(**inp, dy=dy, capacity=capacity)
    fd = _finite_differences(inp, dy, capacity)
    for k in fd:
        np.testing.assert_allclose(g[k], fd[k], rtol=0, atol=1e-7 * np.abs(fd[k]).max())
    if capacity is not None:
        # dropped pairs pass nothing on
        assert not g["fwd"]["keep"].all()
        np.testing.assert_array_equal(g["dw"][~g["fwd"]["keep"]], 0.0)


@pytest.mark.parametrize("mistake", ["silu_grad_is_sigmoid", "gate_sign", "no_router_term"])
def test_backward_planted_mistakes_are_caught(monkeypatch, mistake):
    inp, dy = _fd_case(seed=2)
    fd = _finite_differences(inp, dy)
    if mistake == "silu_grad_is_sigmoid":
        monkeypatch.setattr(O, "_silu_grad", lambda z: 1.0 / (1.0 + np.exp(-np.asarray(z))))
        g = O.moe_layer_backward(**inp, dy=dy)
    else:
        g = dict(O.moe_layer_backward(**inp, dy=dy))
        if mistake == "gate_sign":
            g["dWg"] = -g["dWg"]
        else:
            g["dx"] = g["dx"] - g["dlogits"] @ inp["Wg"].T
    assert not _fd_agrees(g, fd)


@pytest.mark.parametrize("T,d,h,kind", [(1, 8, 16, "plain"), (37, 24, 40, "skew"),
                                        (64, 16, 24, "long")])
def test_backward_routed_equals_dense(T, d, h, kind):
    """O1 (per group, sigmoid of the logit gap) against O2 (every expert, softmax
    Jacobian of the masked dense gate)."""
    inp = _inputs(small("bw", T=T, d=d, h=h, seed=50 + T, kind=kind))
    dy = np.random.default_rng(T).normal(size=(T, d))
    g = O.moe_layer_backward(**inp, dy=dy)
    gd = O.moe_layer_backward_dense(**inp, dy=dy)
    for k in ("dx", "dWg", "dW1", "dW3", "dW2", "dlogits"):
        scale = max(np.abs(gd[k]).max(), 1e-300)
        assert np.abs(g[k] - gd[k]).max() <= 1e-12 * scale, k


def test_backward_invariants():
    inp = _inputs(small("bwi", T=50, d=16, h=24, seed=9, kind="skew"))
    rng = np.random.default_rng(3)
    dy1, dy2 = rng.normal(size=(50, 16)), rng.normal(size=(50, 16))
    g1 = O.moe_layer_backward(**inp, dy=dy1)
    g2 = O.moe_layer_backward(**inp, dy=dy2)
    g12 = O.moe_layer_backward(**inp, dy=dy1 + 2 * dy2)
    for k in ("dx", "dWg", "dW1", "dW3", "dW2", "dw"):
        np.testing.assert_allclose(g12[k], g1[k] + 2 * g2[k], rtol=1e-10,
                                   atol=1e-12 * np.abs(g12[k]).max())
    # a shift of all logits changes nothing: each token's logit gradients sum to 0,
    # and only the two chosen experts' logits receive any
    s = g1["dlogits"].sum(axis=1)
    assert np.abs(s).max() <= 1e-14 * np.abs(g1["dlogits"]).max()
    assert (np.count_nonzero(g1["dlogits"], axis=1) <= 2).all()
    # experts nobody chose get no weight gradient
    counts = np.bincount(g1["fwd"]["idx"].ravel(), minlength=8)
    for e in np.flatnonzero(counts == 0):
        assert not g1["dW1"][e].any() and not g1["dW2"][e].any()


@pytest.mark.parametrize("T,d,h,E,kind", [(1, 8, 16, 8, "plain"), (37, 24, 40, 8, "skew"),
                                          (64, 16, 24, 8, "long"), (29, 16, 8, 4, "plain")])
def test_backward_routed_equals_loops(T, d, h, E, kind):
    """O1 (grouped by expert, NumPy) against O3 (per token, plain C loops written from
    the chain rule), which shares no code or data layout with it."""
    inp = _inputs(small("bwl", T=T, d=d, h=h, E=E, seed=70 + T, kind=kind))
    dy = np.random.default_rng(T + 1).normal(size=(T, d))
    g = O.moe_layer_backward(**inp, dy=dy)
    loops = dict(zip(("dx", "dWg", "dW1", "dW3", "dW2"), oracle.loops_layer_backward(**inp, dy=dy)))
    for k, v in loops.items():
        scale = max(np.abs(v).max(), 1e-300)
        assert np.abs(g[k] - v).max() <= 1e-12 * scale, k


def test_loops_backward_matches_finite_differences():
    """The C loops on their own, against central differences of the C forward."""
    inp, dy = _fd_case(seed=4)
    names = ("x", "Wg", "W1", "W3", "W2")
    got = dict(zip(("d" + n for n in names), oracle.loops_layer_backward(**inp, dy=dy)))
    eps = 1e-6

    def loss(args):
        return float((oracle.loops_layer(*args)[2] * dy).sum())

    for i, n in enumerate(names):
        A = inp[n]
        fd = np.zeros_like(A)
        for ix in np.ndindex(A.shape):
            plus = [inp[m].copy() for m in names]
            minus = [inp[m].copy() for m in names]
            plus[i][ix] += eps
            minus[i][ix] -= eps
            fd[ix] = (loss(plus) - loss(minus)) / (2 * eps)
        np.testing.assert_allclose(got["d" + n], fd, rtol=0, atol=1e-7 * np.abs(fd).max())
