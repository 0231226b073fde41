"""Mixtral top-2-of-8 sparse-MoE SwiGLU layer on NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libmoe.so`` (C ABI declared in ``include/moe.h``).
Every step of the layer runs in the library's CUDA kernels; this module only
checks tensor properties, passes device pointers and the current CUDA stream, and
turns status codes into exceptions.  There is no CPU fallback: importing the
package fails if the library has not been built.

Entry points (same names as the C ABI):
    moe_route, moe_permute, moe_expert_ffn, moe_combine, moe_layer_forward,
    moe_workspace_bytes, moe_device_status, moe_status_string
plus the conveniences ``alloc_workspace`` and ``layer_forward``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "LIB_PATH", "MoeError", "moe_workspace_bytes", "moe_route", "moe_permute",
    "moe_expert_ffn", "moe_combine", "moe_layer_forward", "moe_device_status",
    "moe_status_string", "moe_layer_forward_events", "alloc_workspace", "layer_forward",
    "EXPORTED_SYMBOLS", "launches_per_layer", "launches_per_backward", "moe_expert_ffn_static",
    "moe_layer_forward_capacity", "moe_selftest_wait_timeout", "moe_backward_workspace_bytes",
    "moe_layer_backward", "alloc_backward_workspace", "layer_backward",
    "moe_layer_backward_events", "moe_layer_forward_train",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
_STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                 3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}
EXPORTED_SYMBOLS = ("moe_workspace_bytes", "moe_route", "moe_permute", "moe_expert_ffn",
                    "moe_combine", "moe_layer_forward", "moe_layer_forward_events",
                    "moe_device_status", "moe_status_string", "moe_expert_ffn_static",
                    "moe_layer_forward_capacity", "moe_selftest_wait_timeout",
                    "moe_backward_workspace_bytes", "moe_layer_backward",
                    "moe_layer_backward_events", "moe_layer_forward_train")
def launches_per_layer(T: int, d: int = 4096, E: int = 8, bf16: bool = True) -> int:
    """Kernels one moe_layer_forward queues: router 1, permutation 1 (T <= 512) or 4
    (count, scan, rank, gather; 3 where the bf16 fp64-tensor-core router counts the
    grouping itself: E <= 8, d a multiple of 32 and at most 6144), expert FFN 1
    (T <= 128: gate/up and down fused) or 2, combine 1; none for T == 0."""
    if T <= 0:
        return 0
    router_counts = bf16 and E <= 8 and d % 32 == 0 and d <= 6144
    perm = 1 if T <= 512 else (3 if router_counts else 4)
    return 1 + perm + (1 if T <= 128 else 2) + 1


def launches_per_backward(T: int, capacity: int = -1) -> int:
    """Kernels one moe_layer_backward queues: prep, dH, du/dv, dX, dx, the two
    weight-gradient GEMMs, the dWg partials and their sum (9), plus, without a
    capacity, the element-wise du/dv kernel beside the recomputing one (one of the two
    returns at once, by what the forward kept) and the padded copies of dY and x_perm
    above 1024 grouped rows; none for T == 0."""
    if T <= 0:
        return 0
    free = capacity < 0
    return 9 + (1 if free else 0) + (1 if 2 * T > 1024 and free else 0)


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} -> {_STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with "
            "`python sparse_mixture_experts_26_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz, u32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    sigs = {
        "moe_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
        "moe_route": (i32, [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]),
        "moe_permute": (i32, [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
        "moe_expert_ffn": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, sz, vp]),
        "moe_combine": (i32, [vp, vp, vp, i32, i32, i32, i32, vp, vp]),
        "moe_layer_forward": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp,
                                    sz, vp]),
        "moe_layer_forward_events": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                           vp, vp, sz, vp, i32, vp]),
        "moe_device_status": (i32, [vp, sz, u32p, vp]),
        "moe_status_string": (ctypes.c_char_p, [i32]),
        "moe_expert_ffn_static": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]),
        "moe_layer_forward_capacity": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                             i32, vp, vp, sz, vp]),
        "moe_selftest_wait_timeout": (i32, [vp, sz, ctypes.c_double, vp, vp]),
        "moe_backward_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
        "moe_layer_backward": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                     vp, vp, vp, vp, vp, vp, sz, vp, sz, vp]),
        "moe_layer_forward_train": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp,
                                          vp, sz, vp, sz, vp]),
        "moe_layer_backward_events": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                            i32, vp, vp, vp, vp, vp, vp, sz, vp, sz, vp, i32,
                                            vp]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def moe_status_string(code: int) -> str:
    return _lib.moe_status_string(int(code)).decode()


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise MoeError(fn, code, moe_status_string(code))


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _dev(*ts: torch.Tensor) -> torch.device:
    """Check that the tensors are contiguous CUDA tensors on one device; return it.
    The library launches on the current device, so every call runs under it."""
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
    dev = ts[0].device
    for t in ts[1:]:
        if t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")
    return dev


def _expect(name: str, t: torch.Tensor, shape, dtype=None) -> None:
    """The C ABI receives bare pointers: shapes and dtypes are checked here."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")


def _expect_numel(name: str, t: torch.Tensor, n: int, dtype) -> None:
    if t.numel() != n:
        raise ValueError(f"{name}: {t.numel()} elements, expected {n}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")


def _layer_dims(x, Wg, W1, W3, W2):
    """T, d, h, E of a layer call, after checking every operand against them."""
    if x.dim() != 2 or W1.dim() != 3:
        raise ValueError("x must be [T, d] and W1 [E, h, d]")
    T, d = x.shape
    E, h, _ = W1.shape
    _dt(x)
    _expect("Wg", Wg, (d, E), x.dtype)
    _expect("W1", W1, (E, h, d), x.dtype)
    _expect("W3", W3, (E, h, d), x.dtype)
    _expect("W2", W2, (E, d, h), x.dtype)
    return T, d, h, E


def _ws(name: str, ws: torch.Tensor) -> None:
    if ws.dtype != torch.uint8 or ws.dim() != 1:
        raise TypeError(f"{name}: expected a 1-D uint8 tensor")


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def moe_workspace_bytes(T: int, d: int, h: int, E: int = 8, k: int = 2,
                        dtype: torch.dtype = torch.bfloat16) -> int:
    dt = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32
    return int(_lib.moe_workspace_bytes(T, d, h, E, k, dt))


def moe_expert_ffn_workspace_bytes(rows: int, d: int, h: int, E: int,
                                   dtype: torch.dtype = torch.bfloat16) -> int:
    """Workspace bytes moe_expert_ffn needs for `rows` (even) grouped rows of E experts."""
    return moe_workspace_bytes(max(rows // 2, 1), d, h, max(E, 2), 2, dtype)


def alloc_workspace(T: int, d: int, h: int, E: int = 8, k: int = 2,
                    dtype: torch.dtype = torch.bfloat16, device="cuda") -> torch.Tensor:
    """A zeroed workspace of ``moe_workspace_bytes`` bytes (the status word starts at 0)."""
    n = moe_workspace_bytes(T, d, h, E, k, dtype)
    if n == 0:
        raise MoeError("moe_workspace_bytes", 2, "unsupported shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_route(x, Wg, topk_idx, topk_w, k: int = 2, stream=None) -> None:
    T, d = x.shape
    E = Wg.shape[1]
    _expect("Wg", Wg, (d, E), x.dtype)
    _expect("topk_idx", topk_idx, (T, k), torch.int32)
    _expect("topk_w", topk_w, (T, k), torch.float32)
    dev = _dev(x, Wg, topk_idx, topk_w)
    with torch.cuda.device(dev):
        _check("moe_route", _lib.moe_route(_ptr(x), _ptr(Wg), T, d, E, k, _dt(x),
                                           _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def moe_permute(topk_idx, x, offsets, perm_token, inv_perm, x_perm, ws, E: int, k: int = 2,
                stream=None) -> None:
    T, d = x.shape
    _expect("topk_idx", topk_idx, (T, k), torch.int32)
    _expect_numel("offsets", offsets, E + 1, torch.int32)
    _expect_numel("perm_token", perm_token, T * k, torch.int32)
    _expect_numel("inv_perm", inv_perm, T * k, torch.int32)
    _expect("x_perm", x_perm, (T * k, d), x.dtype)
    _ws("ws", ws)
    dev = _dev(topk_idx, x, offsets, perm_token, inv_perm, x_perm, ws)
    with torch.cuda.device(dev):
        _check("moe_permute", _lib.moe_permute(
            _ptr(topk_idx), _ptr(x), T, d, E, k, _dt(x), _ptr(offsets), _ptr(perm_token),
            _ptr(inv_perm), _ptr(x_perm), _ptr(ws), ws.numel() * ws.element_size(),
            _stream(stream)))


def _ffn_dims(x_perm, offsets, W1, W3, W2, y_perm):
    rows, d = x_perm.shape
    E, h, _ = W1.shape
    _dt(x_perm)
    _expect_numel("offsets", offsets, E + 1, torch.int32)
    _expect("W1", W1, (E, h, d), x_perm.dtype)
    _expect("W3", W3, (E, h, d), x_perm.dtype)
    _expect("W2", W2, (E, d, h), x_perm.dtype)
    _expect("y_perm", y_perm, (rows, d), torch.float32)
    return rows, d, h, E


def moe_expert_ffn(x_perm, offsets, W1, W3, W2, y_perm, ws, stream=None) -> None:
    rows, d, h, E = _ffn_dims(x_perm, offsets, W1, W3, W2, y_perm)
    _ws("ws", ws)
    dev = _dev(x_perm, offsets, W1, W3, W2, y_perm, ws)
    with torch.cuda.device(dev):
        _check("moe_expert_ffn", _lib.moe_expert_ffn(
            _ptr(x_perm), _ptr(offsets), _ptr(W1), _ptr(W3), _ptr(W2), rows, d, h, E,
            _dt(x_perm), _ptr(y_perm), _ptr(ws), ws.numel() * ws.element_size(),
            _stream(stream)))


def moe_combine(y_perm, inv_perm, topk_w, y, k: int = 2, stream=None) -> None:
    T, d = y.shape
    _expect("y_perm", y_perm, (T * k, d), torch.float32)
    _expect_numel("inv_perm", inv_perm, T * k, torch.int32)
    _expect_numel("topk_w", topk_w, T * k, torch.float32)
    dev = _dev(y_perm, inv_perm, topk_w, y)
    with torch.cuda.device(dev):
        _check("moe_combine", _lib.moe_combine(_ptr(y_perm), _ptr(inv_perm), _ptr(topk_w), T, d,
                                               k, _dt(y), _ptr(y), _stream(stream)))


def moe_layer_forward(x, Wg, W1, W3, W2, y, ws, k: int = 2, stream=None) -> None:
    T, d, h, E = _layer_dims(x, Wg, W1, W3, W2)
    _expect("y", y, (T, d), x.dtype)
    _ws("ws", ws)
    dev = _dev(x, Wg, W1, W3, W2, y, ws)
    with torch.cuda.device(dev):
        _check("moe_layer_forward", _lib.moe_layer_forward(
            _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), T, d, h, E, k, _dt(x), _ptr(y),
            _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_layer_forward_train(x, Wg, W1, W3, W2, y, ws, bwd_ws, k: int = 2, stream=None) -> None:
    """``moe_layer_forward`` that also keeps the pre-activations a, b (fp32) in
    ``bwd_ws``, for the ``moe_layer_backward`` call that follows."""
    T, d, h, E = _layer_dims(x, Wg, W1, W3, W2)
    _expect("y", y, (T, d), x.dtype)
    _ws("ws", ws)
    _ws("bwd_ws", bwd_ws)
    dev = _dev(x, Wg, W1, W3, W2, y, ws, bwd_ws)
    with torch.cuda.device(dev):
        _check("moe_layer_forward_train", _lib.moe_layer_forward_train(
            _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), T, d, h, E, k, _dt(x), _ptr(y),
            _ptr(ws), ws.numel() * ws.element_size(), _ptr(bwd_ws),
            bwd_ws.numel() * bwd_ws.element_size(), _stream(stream)))


def moe_layer_forward_capacity(x, Wg, W1, W3, W2, y, ws, capacity: int, k: int = 2,
                               stream=None) -> None:
    """The layer with each expert keeping at most ``capacity`` (token, slot) pairs, in
    token order; dropped pairs contribute nothing.  ``capacity < 0``: no limit."""
    T, d, h, E = _layer_dims(x, Wg, W1, W3, W2)
    _expect("y", y, (T, d), x.dtype)
    _ws("ws", ws)
    dev = _dev(x, Wg, W1, W3, W2, y, ws)
    with torch.cuda.device(dev):
        _check("moe_layer_forward_capacity", _lib.moe_layer_forward_capacity(
            _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), T, d, h, E, k, _dt(x),
            int(capacity), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_layer_forward_events(x, Wg, W1, W3, W2, y, ws, events, k: int = 2,
                             stream=None) -> None:
    """``moe_layer_forward`` recording ``events`` (up to 5 created handles, or None to skip
    one) between its stages."""
    T, d, h, E = _layer_dims(x, Wg, W1, W3, W2)
    _expect("y", y, (T, d), x.dtype)
    _ws("ws", ws)
    dev = _dev(x, Wg, W1, W3, W2, y, ws)
    handles = (ctypes.c_void_p * max(1, len(events)))(*[int(e) if e else None for e in events])
    with torch.cuda.device(dev):
        _check("moe_layer_forward_events", _lib.moe_layer_forward_events(
            _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), T, d, h, E, k, _dt(x), _ptr(y),
            _ptr(ws), ws.numel() * ws.element_size(), ctypes.addressof(handles), len(events),
            _stream(stream)))


def moe_device_status(ws, stream=None) -> int:
    """Synchronise, return and clear the workspace's device status flags."""
    dev = _dev(ws)
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        code = _lib.moe_device_status(_ptr(ws), ws.numel() * ws.element_size(),
                                      ctypes.addressof(flags), _stream(stream))
    if code not in (0, 5):
        _check("moe_device_status", code)
    return int(flags.value)


def moe_expert_ffn_static(x_perm, offsets, W1, W3, W2, y_perm, stream=None) -> None:
    """``moe_expert_ffn`` without a workspace, for callers that cannot allocate device
    memory: the scratch is a fixed 8 MiB array inside the library (see include/moe.h
    for the size limit, the first-call set-up and why overlapping calls race)."""
    rows, d, h, E = _ffn_dims(x_perm, offsets, W1, W3, W2, y_perm)
    dev = _dev(x_perm, offsets, W1, W3, W2, y_perm)
    with torch.cuda.device(dev):
        _check("moe_expert_ffn_static", _lib.moe_expert_ffn_static(
            _ptr(x_perm), _ptr(offsets), _ptr(W1), _ptr(W3), _ptr(W2), rows, d, h, E,
            _dt(x_perm), _ptr(y_perm), _stream(stream)))


def moe_selftest_wait_timeout(ws, limit_seconds: float = 0.05, stream=None):
    """Run the bounded-wait self-test; returns (barrier outcome, counter outcome), each 2
    when the wait gave up as it must.  The timeout flag is left in the status word."""
    dev = _dev(ws)
    out = (ctypes.c_uint32 * 2)()
    with torch.cuda.device(dev):
        _check("moe_selftest_wait_timeout", _lib.moe_selftest_wait_timeout(
            _ptr(ws), ws.numel() * ws.element_size(), float(limit_seconds),
            ctypes.addressof(out), _stream(stream)))
    return int(out[0]), int(out[1])


def layer_forward(x, Wg, W1, W3, W2, ws=None, out=None, stream=None) -> torch.Tensor:
    """Run the whole layer, allocating the workspace and output with torch if not given."""
    T, d = x.shape
    E, h, _ = W1.shape
    if ws is None:
        ws = alloc_workspace(T, d, h, E, 2, x.dtype, x.device)
    if out is None:
        out = torch.empty_like(x)
    moe_layer_forward(x, Wg, W1, W3, W2, out, ws, stream=stream)
    return out


def moe_backward_workspace_bytes(T: int, d: int, h: int, E: int = 8, k: int = 2,
                                 dtype: torch.dtype = torch.bfloat16) -> int:
    dt = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32
    return int(_lib.moe_backward_workspace_bytes(T, d, h, E, k, dt))


def alloc_backward_workspace(T: int, d: int, h: int, E: int = 8, k: int = 2,
                             dtype: torch.dtype = torch.bfloat16, device="cuda") -> torch.Tensor:
    n = moe_backward_workspace_bytes(T, d, h, E, k, dtype)
    if n == 0:
        raise MoeError("moe_backward_workspace_bytes", 2, "unsupported shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _backward_dims(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws):
    T, d, h, E = _layer_dims(x, Wg, W1, W3, W2)
    _expect("dy", dy, (T, d), x.dtype)
    _expect("dx", dx, (T, d), x.dtype)
    _expect("dWg", dWg, (d, E), torch.float32)
    _expect("dW1", dW1, (E, h, d), torch.float32)
    _expect("dW3", dW3, (E, h, d), torch.float32)
    _expect("dW2", dW2, (E, d, h), torch.float32)
    _ws("fwd_ws", fwd_ws)
    _ws("bwd_ws", bwd_ws)
    return T, d, h, E


def moe_layer_backward(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws,
                       capacity: int = -1, k: int = 2, stream=None) -> None:
    """Gradients of the layer for upstream gradient ``dy``; ``fwd_ws`` is the workspace
    of the forward call on the same inputs (``capacity`` as given to it, -1 for none)."""
    T, d, h, E = _backward_dims(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws)
    dev = _dev(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws)
    with torch.cuda.device(dev):
        _check("moe_layer_backward", _lib.moe_layer_backward(
            _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dy), T, d, h, E, k, _dt(x),
            int(capacity), _ptr(dx), _ptr(dWg), _ptr(dW1), _ptr(dW3), _ptr(dW2), _ptr(fwd_ws),
            fwd_ws.numel() * fwd_ws.element_size(), _ptr(bwd_ws),
            bwd_ws.numel() * bwd_ws.element_size(), _stream(stream)))


def moe_layer_backward_events(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws,
                              events, capacity: int = -1, k: int = 2, stream=None) -> None:
    """``moe_layer_backward`` recording ``events`` (up to 9 created handles, or None to
    skip one) before its first launch and after each stage."""
    T, d, h, E = _backward_dims(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws)
    dev = _dev(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws)
    handles = (ctypes.c_void_p * max(1, len(events)))(*[int(e) if e else None for e in events])
    with torch.cuda.device(dev):
        _check("moe_layer_backward_events", _lib.moe_layer_backward_events(
            _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dy), T, d, h, E, k, _dt(x),
            int(capacity), _ptr(dx), _ptr(dWg), _ptr(dW1), _ptr(dW3), _ptr(dW2), _ptr(fwd_ws),
            fwd_ws.numel() * fwd_ws.element_size(), _ptr(bwd_ws),
            bwd_ws.numel() * bwd_ws.element_size(), ctypes.addressof(handles), len(events),
            _stream(stream)))


def layer_backward(x, Wg, W1, W3, W2, dy, fwd_ws, capacity: int = -1, bwd_ws=None):
    """Allocating convenience wrapper: returns (dx, dWg, dW1, dW3, dW2)."""
    T, d = x.shape
    E, h, _ = W1.shape
    if bwd_ws is None:
        bwd_ws = alloc_backward_workspace(T, d, h, E, 2, x.dtype, x.device)
    dx = torch.empty_like(x)
    f32 = dict(dtype=torch.float32, device=x.device)
    dWg, dW1 = torch.empty(Wg.shape, **f32), torch.empty(W1.shape, **f32)
    dW3, dW2 = torch.empty(W3.shape, **f32), torch.empty(W2.shape, **f32)
    moe_layer_backward(x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, fwd_ws, bwd_ws, capacity)
    return dx, dWg, dW1, dW3, dW2
