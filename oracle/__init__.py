"""CPU oracle of the Mixtral sparse-MoE layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The CUDA library never does.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import __all__  # noqa: F401


def loops_layer(x, Wg, W1, W3, W2):
    """Run the plain-C loop oracle (O3); returns ``(idx int32[T,2], w f64[T,2], y f64[T,d])``."""
    import ctypes

    import numpy as np

    from .build_oracle import build

    lib = ctypes.CDLL(build())
    f = lib.moe_oracle_loops
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    f.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ip, dp, dp]
    f.restype = ctypes.c_int
    arrs = [np.ascontiguousarray(a, dtype=np.float64) for a in (x, Wg, W1, W3, W2)]
    T, d = arrs[0].shape
    E = arrs[1].shape[1]
    h = arrs[2].shape[1]
    idx = np.zeros((T, 2), dtype=np.int32)
    w = np.zeros((T, 2), dtype=np.float64)
    y = np.zeros((T, d), dtype=np.float64)
    rc = f(*[a.ctypes.data_as(dp) for a in arrs], T, d, h, E,
           idx.ctypes.data_as(ip), w.ctypes.data_as(dp), y.ctypes.data_as(dp))
    if rc != 0:
        raise ValueError("moe_oracle_loops rejected its arguments")
    return idx, w, y


def loops_layer_backward(x, Wg, W1, W3, W2, dy):
    """Run the plain-C loop backward (O3); returns ``(dx, dWg, dW1, dW3, dW2)`` in fp64."""
    import ctypes

    import numpy as np

    from .build_oracle import build

    lib = ctypes.CDLL(build())
    f = lib.moe_oracle_loops_backward
    dp = ctypes.POINTER(ctypes.c_double)
    f.argtypes = [dp] * 6 + [ctypes.c_int] * 4 + [dp] * 5
    f.restype = ctypes.c_int
    arrs = [np.ascontiguousarray(a, dtype=np.float64) for a in (x, Wg, W1, W3, W2, dy)]
    T, d = arrs[0].shape
    E = arrs[1].shape[1]
    h = arrs[2].shape[1]
    outs = [np.zeros(s, dtype=np.float64) for s in ((T, d), (d, E), (E, h, d), (E, h, d),
                                                     (E, d, h))]
    rc = f(*[a.ctypes.data_as(dp) for a in arrs], T, d, h, E,
           *[o.ctypes.data_as(dp) for o in outs])
    if rc != 0:
        raise ValueError("moe_oracle_loops_backward rejected its arguments")
    return tuple(outs)
