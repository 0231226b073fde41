"""CPU fp64 oracle for the Mixtral top-2-of-8 sparse-MoE SwiGLU feed-forward layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links this
module; only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code, table or
helper with the CUDA library; the two meet only through the seeded input generator.

What it computes (sources, cited as page title + section/equation):

* Router logits ``l = x . W_g`` over ``E`` experts, shape ``[T, E]``
  -- crackai "Mixtral of Experts", section "Top-2 Routing in Detail" (gate_logits);
  notion notes "Mixtral of Experts", section "Sparse gating", eq. G(x).
* Gate ``G(x) = Softmax(TopK(x . W_g))`` where every logit outside the top k is set
  to -inf before the softmax, so only k experts get non-zero weight
  -- notion notes, "Sparse gating", eq. G(x) and the sentence under it.
* The same weights written the other way round: softmax over all E, keep the top
  two, divide by their sum -- ml-canon "52 Mixtral", section "PyTorch Mixtral's MoE
  FFN (top-2 of 8)".  Both forms are computed here and must agree.
* K = 2 and the expert function is SwiGLU -- notion notes, "Implementation";
  atlas "Mixtral", "Design overview" (SwiGLU, inner dimension 14336).  The SwiGLU
  form ``E_e(x) = W2[e] (silu(W1[e] x) * (W3[e] x))`` with ``silu(z) = z sigma(z)``
  is the plain reading of "SwiGLU architecture" (gate branch W1, linear branch W3,
  no biases: the pages show none).
* Output ``y = sum_i G(x)_i E_i(x)`` -- notion notes, "Architectural details" and
  "Implementation", eq. y; crackai, "Top-2 Routing in Detail"
  (y = w_1 Expert_{i1}(x) + w_2 Expert_{i2}(x)).
* Grouping tokens by expert and scattering results back -- ml-canon "52 Mixtral",
  "Questions worth asking" (gather and scatter); notion notes, "Expert Parallelism"
  (output returned to the original token location).

Readings where the pages are silent (each is also listed in the design notes):

* Ties in the top-2 choice go to the lower expert index; experts are ordered by
  (logit descending, index ascending) and slot 0 holds the larger logit.
* Selection is made on the fp64 logits (exact products of the bf16/fp32 inputs,
  summed in fp64), never on rounded softmax values.
* ``w1 = 1 / (1 + exp(l2 - l1))`` in fp64, rounded once to float32;
  ``w2 = 1 - w1`` evaluated in float32 so that the pair sums to exactly 1.
* No capacity limit and no token dropping: every token reaches exactly 2 experts.
* The permutation is a stable counting sort by expert of the flattened
  (token, slot) index ``f = t*k + j``: within one expert's group rows are in
  ascending token order.
* Inputs are taken as exact values (bf16/fp32 promoted to fp64); nothing is rounded
  in between.

Every public function here is pinned by tests in ``tests/test_oracle_pins.py``
against closed forms, brute force on tiny inputs and the pages' printed numbers.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "router_logits",
    "top2_select",
    "gate_weights",
    "gate_weights_f32",
    "gate_dense_topk_softmax",
    "gate_dense_softmax_topk_renorm",
    "permutation",
    "gather_rows",
    "silu",
    "expert_swiglu",
    "expert_ffn_grouped",
    "combine",
    "moe_layer",
    "moe_layer_dense",
    "mixtral_param_counts",
    "capacity_keep",
    "capacity_from_factor",
    "moe_layer_backward",
    "moe_layer_backward_dense",
]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def router_logits(x, Wg) -> np.ndarray:
    """``l[t, e] = sum_i x[t, i] * W_g[i, e]`` in fp64.

    crackai "Mixtral of Experts", "Top-2 Routing in Detail": gate_logits = x . W_gate,
    shape [tokens, 8]; notion notes, "Sparse gating", eq. G(x) (x . W_g).
    """
    return _f64(x) @ _f64(Wg)


def top2_select(logits, k: int = 2) -> np.ndarray:
    """Indices of the k largest logits per token, ordered (logit desc, index asc).

    notion notes, "Sparse gating" (TopK keeps the top-k values); K = 2 per
    "Implementation".  Ties are broken toward the lower expert index (reading: the
    pages are silent).  A stable ascending sort of ``-logits`` yields exactly that
    order.  Returns int32 ``[T, k]``.
    """
    l = _f64(logits)
    order = np.argsort(-l, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gate_weights(logits, idx) -> np.ndarray:
    """fp64 weights of the two kept experts: softmax restricted to the top two.

    For k = 2 the restricted softmax is ``w1 = 1/(1 + exp(l2 - l1))`` and
    ``w2 = 1/(1 + exp(l1 - l2))`` (the softmax of two numbers); notion notes,
    "Sparse gating", eq. G(x).
    """
    l = _f64(logits)
    l1 = np.take_along_axis(l, idx[:, :1].astype(np.int64), axis=1)[:, 0]
    l2 = np.take_along_axis(l, idx[:, 1:2].astype(np.int64), axis=1)[:, 0]
    w1 = 1.0 / (1.0 + np.exp(l2 - l1))
    w2 = 1.0 / (1.0 + np.exp(l1 - l2))
    return np.stack([w1, w2], axis=1)


def gate_weights_f32(logits, idx) -> np.ndarray:
    """The float32 weights as the layer stores them (reading of the silent rounding).

    ``w1`` is the fp64 value rounded once to float32, and ``w2 = 1 - w1`` is
    evaluated in float32 so that ``w1 + w2 == 1`` exactly in float32.
    """
    w = gate_weights(logits, idx)
    w1 = w[:, 0].astype(np.float32)
    w2 = (np.float32(1.0) - w1).astype(np.float32)
    return np.stack([w1, w2], axis=1)


def gate_dense_topk_softmax(logits, k: int = 2) -> np.ndarray:
    """Dense ``G(x) = Softmax(TopK(l))``: logits outside the top k set to -inf.

    notion notes, "Sparse gating", eq. G(x): "all other values ... are set to -inf,
    leading to 0 weights".  Returns fp64 ``[T, E]``.
    """
    l = _f64(logits)
    idx = top2_select(l, k)
    masked = np.full_like(l, -np.inf)
    rows = np.arange(l.shape[0])[:, None]
    masked[rows, idx] = l[rows, idx]
    m = masked.max(axis=1, keepdims=True)
    e = np.exp(masked - m)  # exp(-inf) == 0
    return e / e.sum(axis=1, keepdims=True)


def gate_dense_softmax_topk_renorm(logits, k: int = 2) -> np.ndarray:
    """Dense gate from softmax over all E, then top k, then renormalise.

    ml-canon "52 Mixtral", "PyTorch Mixtral's MoE FFN (top-2 of 8)": softmax over the
    experts, keep the top two, divide by their sum.  The kept set is chosen on the
    logits (softmax is monotone) with the same tie rule.  Returns fp64 ``[T, E]``.
    """
    l = _f64(logits)
    m = l.max(axis=1, keepdims=True)
    p = np.exp(l - m)
    p = p / p.sum(axis=1, keepdims=True)
    idx = top2_select(l, k)
    rows = np.arange(l.shape[0])[:, None]
    kept = p[rows, idx]
    kept = kept / kept.sum(axis=1, keepdims=True)
    G = np.zeros_like(l)
    G[rows, idx] = kept
    return G


def permutation(idx, E: int):
    """Group the flattened (token, slot) pairs by expert (stable counting sort).

    ml-canon "52 Mixtral", "Questions worth asking" (gather tokens by expert and
    scatter them back); notion notes, "Expert Parallelism" (results returned to the
    original token location).  Row order inside a group is ascending in the
    flattened index ``f = t*k + j`` (reading: the pages are silent).

    Returns ``offsets[E+1]`` (group e owns rows offsets[e]:offsets[e+1]),
    ``perm_token[P]`` (source token of each row) and ``inv_perm[T, k]`` (row that
    holds pair (t, j)), all int32.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable")
    perm_token = perm // k
    inv = np.empty(T * k, dtype=np.int64)
    inv[perm] = np.arange(T * k)
    return (offsets.astype(np.int32), perm_token.astype(np.int32),
            inv.reshape(T, k).astype(np.int32))


def gather_rows(x, perm_token) -> np.ndarray:
    """``x_perm[r] = x[perm_token[r]]`` (pure data movement; dtype preserved)."""
    return np.asarray(x)[np.asarray(perm_token, dtype=np.int64)]


def silu(z) -> np.ndarray:
    """``silu(z) = z * sigma(z) = z / (1 + exp(-z))`` in fp64."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_swiglu(xr, W1e, W3e, W2e) -> np.ndarray:
    """One expert's SwiGLU FFN on rows ``xr[n, d]``: ``(silu(xr W1e^T) * (xr W3e^T)) W2e^T``.

    Shapes: ``W1e, W3e`` are ``[h, d]``, ``W2e`` is ``[d, h]`` (the stacked layouts
    W1/W3 ``[E, h, d]`` and W2 ``[E, d, h]``).  notion notes, "Implementation"
    (SwiGLU expert function); atlas "Mixtral", "Design overview" (inner dim 14336).
    """
    xr = _f64(xr)
    a = xr @ _f64(W1e).T
    b = xr @ _f64(W3e).T
    return (silu(a) * b) @ _f64(W2e).T


def expert_ffn_grouped(x_perm, offsets, W1, W3, W2) -> np.ndarray:
    """Run every expert group through its own SwiGLU FFN; returns fp64 ``Y[P, d]``.

    An empty group contributes nothing (no rows).  ``W1``/``W3``/``W2`` only need
    to support ``[e]`` indexing, so large stacks can be handed over one expert at a
    time.
    """
    x_perm = _f64(x_perm)
    P, d = x_perm.shape
    Y = np.zeros((P, d), dtype=np.float64)
    E = len(offsets) - 1
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            Y[lo:hi] = expert_swiglu(x_perm[lo:hi], W1[e], W3[e], W2[e])
    return Y


def combine(Y, inv_perm, w) -> np.ndarray:
    """``y[t] = sum_j w[t, j] * Y[inv_perm[t, j]]`` in fp64.

    crackai "Mixtral of Experts", "Top-2 Routing in Detail":
    y = w_1 Expert_{i1}(x) + w_2 Expert_{i2}(x); notion notes, eq. y.
    """
    Y = _f64(Y)
    w = _f64(w)
    inv = np.asarray(inv_perm, dtype=np.int64)
    y = np.zeros((inv.shape[0], Y.shape[1]), dtype=np.float64)
    for j in range(inv.shape[1]):
        y += w[:, j:j + 1] * Y[inv[:, j]]
    return y


def capacity_from_factor(factor: float, T: int, k: int, E: int) -> int:
    """Per-expert capacity for a capacity factor: ceil(factor * T * k / E) rows.

    ml-canon "52 Mixtral", "Questions worth asking": a capacity factor caps the
    tokens each expert takes (the pages give no formula; this is the usual one:
    the factor times an even share of the T*k (token, slot) pairs).
    """
    import math
    return int(math.ceil(factor * T * k / E))


def capacity_keep(idx, E: int, capacity) -> np.ndarray:
    """Boolean ``[T, k]``: is pair (t, j) within its expert's capacity?

    Reading (the pages only say "a cap on tokens per expert"): each expert keeps the
    first ``capacity`` of its pairs in the stable grouping order (ascending token,
    then slot) and drops the rest.  ``capacity=None`` keeps everything.
    """
    idx = np.asarray(idx)
    keep = np.ones(idx.shape, dtype=bool)
    if capacity is None:
        return keep
    T, k = idx.shape
    seen = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            keep[t, j] = seen[e] < capacity
            seen[e] += 1
    return keep


def moe_layer(x, Wg, W1, W3, W2, k: int = 2, capacity=None) -> dict:
    """The routed layer (oracle O1): route, group by expert, SwiGLU per group, combine.

    With ``capacity`` (opt-in), a pair beyond its expert's capacity is dropped: its
    expert output is not computed and it contributes nothing to y; the other
    weights are left as they are (see ``capacity_keep``).

    Returns a dict with every intermediate: ``logits`` (fp64), ``idx`` (int32
    ``[T, k]``), ``w`` (fp64), ``w_f32`` (float32 as stored by the layer),
    ``offsets``, ``perm_token``, ``inv_perm`` (int32), ``Y`` (fp64 ``[P, d]``) and
    ``y`` (fp64 ``[T, d]``).  ``y`` uses the fp64 gate (the definition).
    """
    logits = router_logits(x, Wg)
    E = logits.shape[1]
    idx = top2_select(logits, k)
    w = gate_weights(logits, idx)
    offsets, perm_token, inv_perm = permutation(idx, E)
    x_perm = gather_rows(_f64(x), perm_token)
    keep = capacity_keep(idx, E, capacity)
    if capacity is not None:
        # only the first `capacity` rows of each group are run through the expert
        Y = np.zeros((x_perm.shape[0], x_perm.shape[1]), dtype=np.float64)
        for e in range(E):
            lo = int(offsets[e])
            hi = min(int(offsets[e + 1]), lo + int(capacity))
            if hi > lo:
                Y[lo:hi] = expert_swiglu(x_perm[lo:hi], W1[e], W3[e], W2[e])
    else:
        Y = expert_ffn_grouped(x_perm, offsets, W1, W3, W2)
    y = combine(Y, inv_perm, w * keep)
    return dict(logits=logits, idx=idx, w=w, w_f32=gate_weights_f32(logits, idx),
                offsets=offsets, perm_token=perm_token, inv_perm=inv_perm, Y=Y, y=y,
                keep=keep)


def moe_layer_dense(x, Wg, W1, W3, W2, k: int = 2) -> np.ndarray:
    """Brute-force layer (oracle O2): every expert on every token, weighted by dense G.

    ``y = sum_{e=0}^{E-1} G(x)_e E_e(x)`` with ``G`` the -inf-masked softmax, exactly
    as notion notes, "Implementation", eq. y is written (experts with G = 0 are still
    evaluated and multiplied by zero).  No grouping or permutation.
    """
    x = _f64(x)
    G = gate_dense_topk_softmax(router_logits(x, Wg), k)
    y = np.zeros(x.shape, dtype=np.float64)
    for e in range(G.shape[1]):
        y += G[:, e:e + 1] * expert_swiglu(x, W1[e], W3[e], W2[e])
    return y


def _silu_grad(z) -> np.ndarray:
    """d silu / dz = sigma(z) (1 + z (1 - sigma(z))) in fp64."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def moe_layer_backward(x, Wg, W1, W3, W2, dy, k: int = 2, capacity=None) -> dict:
    """Gradients of the routed layer (oracle O1) for an upstream gradient ``dy[T, d]``.

    crackai "Mixtral of Experts", "Key Takeaways": routing is learned jointly with the
    model, so the gradient reaches the router through the gate weights.  Reading (the
    pages state no backward pass): the exact derivative of ``y`` with the top-2 choice
    held fixed (it is piecewise constant in the inputs), computed group by group:

    * grouped row ``r`` of token ``t``, slot ``j``: ``dY[r] = w[t, j] dy[t]`` and
      ``dw[t, j] = <dy[t], Y[r]>``;
    * per expert, with ``a = x W1^T``, ``b = x W3^T``, ``H = silu(a) b``:
      ``dW2 = dY^T H``, ``dH = dY W2``, ``da = dH b silu'(a)``, ``db = dH silu(a)``,
      ``dW1 = da^T x``, ``dW3 = db^T x``, ``dx_perm = da W1 + db W3``;
    * ``dx[t] = sum_j dx_perm[inv[t, j]]``;
    * gate: ``w1 = sigma(l_i1 - l_i2)``, ``w2 = 1 - w1``, so the logit gap receives
      ``(dw1 - dw2) w1 w2``, logit ``i1`` that amount and logit ``i2`` its negative;
      ``dWg = x^T dlogits`` and ``dx += dlogits Wg^T``.

    A pair dropped by ``capacity`` contributes nothing to ``y`` and so receives and
    passes on no gradient.  Returns ``dx, dWg, dW1, dW3, dW2`` (fp64, shaped like the
    inputs), ``dw [T, k]``, ``dlogits [T, E]``, ``dY [P, d]`` (grouped order),
    ``dH [P, h]`` and the forward dict under ``fwd``.
    """
    if k != 2:
        raise ValueError("the gate derivative is written for k = 2")
    fwd = moe_layer(x, Wg, W1, W3, W2, k, capacity)
    x = _f64(x)
    Wg = _f64(Wg)
    dy = _f64(dy)
    T, d = x.shape
    E = fwd["logits"].shape[1]
    idx, w, keep = fwd["idx"], fwd["w"], fwd["keep"]
    offsets, perm_token, inv = fwd["offsets"], fwd["perm_token"], fwd["inv_perm"]
    inv = np.asarray(inv, dtype=np.int64)
    P = T * k
    h = np.asarray(W1[0]).shape[0] if E else 0
    slot = np.empty(P, dtype=np.int64)
    for j in range(k):
        slot[inv[:, j]] = j
    tok = np.asarray(perm_token, dtype=np.int64)
    wk = w * keep
    dY = wk[tok, slot][:, None] * dy[tok]
    dw = np.zeros((T, k), dtype=np.float64)
    for j in range(k):
        dw[:, j] = np.einsum("td,td->t", dy, fwd["Y"][inv[:, j]]) * keep[:, j]
    x_perm = gather_rows(x, tok)
    dx_perm = np.zeros((P, d), dtype=np.float64)
    dH = np.zeros((P, h), dtype=np.float64)
    dW1 = np.zeros((E, h, d), dtype=np.float64)
    dW3 = np.zeros((E, h, d), dtype=np.float64)
    dW2 = np.zeros((E, d, h), dtype=np.float64)
    for e in range(E):
        lo = int(offsets[e])
        hi = int(offsets[e + 1])
        if capacity is not None:
            hi = min(hi, lo + int(capacity))
        if hi <= lo:
            continue
        W1e, W3e, W2e = _f64(W1[e]), _f64(W3[e]), _f64(W2[e])
        xr = x_perm[lo:hi]
        a = xr @ W1e.T
        b = xr @ W3e.T
        He = silu(a) * b
        g = dY[lo:hi]
        dW2[e] = g.T @ He
        dHe = g @ W2e
        dH[lo:hi] = dHe
        da = dHe * b * _silu_grad(a)
        db = dHe * silu(a)
        dW1[e] = da.T @ xr
        dW3[e] = db.T @ xr
        dx_perm[lo:hi] = da @ W1e + db @ W3e
    dx = np.zeros((T, d), dtype=np.float64)
    for j in range(k):
        dx += dx_perm[inv[:, j]]
    gap = (dw[:, 0] - dw[:, 1]) * w[:, 0] * w[:, 1]
    dlogits = np.zeros((T, E), dtype=np.float64)
    rows = np.arange(T)
    dlogits[rows, idx[:, 0]] += gap
    dlogits[rows, idx[:, 1]] -= gap
    dWg = x.T @ dlogits
    dx += dlogits @ Wg.T
    return dict(dx=dx, dWg=dWg, dW1=dW1, dW3=dW3, dW2=dW2, dw=dw, dlogits=dlogits, dY=dY,
                dH=dH, fwd=fwd)


def moe_layer_backward_dense(x, Wg, W1, W3, W2, dy, k: int = 2) -> dict:
    """Brute-force gradients (oracle O2): every expert on every token, dense gate.

    ``y = sum_e G_e E_e(x)`` with ``G`` the -inf-masked softmax of notion notes,
    "Sparse gating", eq. G(x) (mask held fixed).  ``dG_e = <dy, E_e(x)>``; the softmax
    Jacobian gives ``dlogits = G * (dG - <G, dG>)`` (zero outside the mask, because G
    is); each expert's weights get ``G_e`` times its plain SwiGLU gradient.  No
    grouping, no permutation, and a different route through the gate derivative than
    ``moe_layer_backward``.
    """
    x = _f64(x)
    Wg = _f64(Wg)
    dy = _f64(dy)
    T, d = x.shape
    G = gate_dense_topk_softmax(router_logits(x, Wg), k)
    E = G.shape[1]
    h = np.asarray(W1[0]).shape[0]
    dx = np.zeros((T, d), dtype=np.float64)
    dW1 = np.zeros((E, h, d), dtype=np.float64)
    dW3 = np.zeros((E, h, d), dtype=np.float64)
    dW2 = np.zeros((E, d, h), dtype=np.float64)
    dG = np.zeros((T, E), dtype=np.float64)
    for e in range(E):
        W1e, W3e, W2e = _f64(W1[e]), _f64(W3[e]), _f64(W2[e])
        a = x @ W1e.T
        b = x @ W3e.T
        He = silu(a) * b
        Ye = He @ W2e.T
        dG[:, e] = np.einsum("td,td->t", dy, Ye)
        g = G[:, e:e + 1] * dy
        dW2[e] = g.T @ He
        dHe = g @ W2e
        da = dHe * b * _silu_grad(a)
        db = dHe * silu(a)
        dW1[e] = da.T @ x
        dW3[e] = db.T @ x
        dx += da @ W1e + db @ W3e
    dlogits = G * (dG - np.sum(G * dG, axis=1, keepdims=True))
    dWg = x.T @ dlogits
    dx += dlogits @ Wg.T
    return dict(dx=dx, dWg=dWg, dW1=dW1, dW3=dW3, dW2=dW2, dlogits=dlogits)


def mixtral_param_counts(d: int = 32 * 128, h: int = 14336, E: int = 8, k: int = 2,
                         layers: int = 32, vocab: int = 32000, n_heads: int = 32,
                         n_kv_heads: int = 8, head_dim: int = 128) -> dict:
    """Closed-form parameter counts of the whole model from the pages' dimensions.

    atlas "Mixtral", "Design overview": 32 layers, 8 experts per layer, SwiGLU
    inner dim 14336, 32 query / 8 KV heads of dim 128; vocab 32000 ("Notable
    omissions").  The model dim is the heads x head_dim product (the pages never
    print it directly).  Attention is grouped-query (q and o are d x d; k and v
    are d x (kv_heads * head_dim)); embeddings are untied (input + output); each
    layer has two RMSNorm weight vectors and there is a final norm.  Returns total
    and active (k of E experts) counts.
    """
    expert = 3 * d * h
    router = d * E
    attn = 2 * d * (n_heads * head_dim) + 2 * d * (n_kv_heads * head_dim)
    norms = 2 * d
    per_layer_shared = attn + router + norms
    embed = 2 * vocab * d
    total = layers * (E * expert + per_layer_shared) + embed + d
    active = layers * (k * expert + per_layer_shared) + embed + d
    return dict(total=total, active=active, expert_per_layer=E * expert)
