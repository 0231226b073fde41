"""Host-side checks of the C ABI: the library loads, exports every symbol that
include/moe.h declares, sizes its workspace, and rejects bad arguments before it
touches the GPU (so these run without one)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_moe_build", os.path.join(ROOT, "sparse_mixture_experts_26_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    L = ctypes.CDLL(b.build())
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_workspace_bytes.restype = sz
    L.moe_workspace_bytes.argtypes = [i32] * 6
    L.moe_route.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]
    L.moe_permute.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]
    L.moe_expert_ffn.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, sz, vp]
    L.moe_combine.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp]
    L.moe_layer_forward.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp,
                                    sz, vp]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [i32]
    return L


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine",
                     "moe_layer_forward", "moe_workspace_bytes", "moe_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_exports_the_same_names(lib):
    import sparse_mixture_experts_26_b200 as m
    for name in declared_functions():
        assert callable(getattr(m, name)), name
    assert set(m.EXPORTED_SYMBOLS) == set(declared_functions())


def test_workspace_sizes(lib):
    d, h = 4096, 14336
    n16 = lib.moe_workspace_bytes(16, d, h, 8, 2, BF16)
    n4k = lib.moe_workspace_bytes(4096, d, h, 8, 2, BF16)
    assert 0 < n16 < n4k
    P = 2 * 4096
    # must hold at least x_perm (bf16), H (bf16) and the fp32 expert outputs
    assert n4k >= P * d * 2 + P * h * 2 + P * d * 4
    assert n4k % 1024 == 0
    assert lib.moe_workspace_bytes(16, d, h, 8, 3, BF16) == 0      # k != 2
    assert lib.moe_workspace_bytes(16, 4095, h, 8, 2, BF16) == 0   # d % 8
    assert lib.moe_workspace_bytes(16, d, h, 33, 2, BF16) == 0     # E > 32
    assert lib.moe_workspace_bytes(-1, d, h, 8, 2, BF16) == 0
    # the flattened weight views [E*h, d] / [E*d, h] need 32-bit row coordinates
    assert lib.moe_workspace_bytes(1, 64, 1 << 26, 32, 2, BF16) == 0
    assert lib.moe_workspace_bytes(1, 1 << 26, 64, 32, 2, BF16) == 0
    assert lib.moe_workspace_bytes(1, 64, (1 << 26) - 8, 32, 2, BF16) > 0


@pytest.mark.parametrize("d,h,dt", [(4096, 14336, BF16), (136, 192, BF16), (24, 40, 0)])
def test_workspace_size_never_decreases_with_T(lib, d, h, dt):
    """A workspace sized for T serves every smaller batch: small batches add split-K
    partial sums that larger batches do not need, and the size must not drop there."""
    sizes = [lib.moe_workspace_bytes(T, d, h, 8, 2, dt) for T in range(0, 400)]
    assert all(a <= b for a, b in zip(sizes, sizes[1:]))


FAKE = 1 << 20  # 16-byte aligned, never dereferenced: validation fails first


def test_route_validation(lib):
    p = FAKE
    assert lib.moe_route(None, p, 4, 64, 8, 2, BF16, p, p, None) == INVALID
    assert lib.moe_route(p + 2, p, 4, 64, 8, 2, BF16, p, p, None) == INVALID  # misaligned
    assert lib.moe_route(p, p, 4, 64, 8, 3, BF16, p, p, None) == UNSUPPORTED
    assert lib.moe_route(p, p, 4, 60, 8, 2, BF16, p, p, None) == UNSUPPORTED
    assert lib.moe_route(p, p, 4, 64, 1, 2, BF16, p, p, None) == UNSUPPORTED
    assert lib.moe_route(p, p, -1, 64, 8, 2, BF16, p, p, None) == INVALID
    assert lib.moe_route(p, p, 4, 64, 8, 2, 7, p, p, None) == INVALID
    assert lib.moe_route(None, None, 0, 64, 8, 2, BF16, None, None, None) == OK  # T=0 no-op


def test_layer_validation(lib):
    p = FAKE
    need = lib.moe_workspace_bytes(8, 64, 128, 8, 2, BF16)
    assert lib.moe_layer_forward(p, p, p, p, p, 8, 64, 128, 8, 2, BF16, p, p, need - 1,
                                 None) == WORKSPACE
    assert lib.moe_layer_forward(p, p, p, p, None, 8, 64, 128, 8, 2, BF16, p, p, need,
                                 None) == INVALID
    assert lib.moe_layer_forward(p, p, p, p, p, 8, 64, 100, 8, 2, BF16, p, p, need,
                                 None) == UNSUPPORTED
    assert lib.moe_layer_forward(p, p, p, p, p, 0, 64, 128, 8, 2, BF16, p, p, 0, None) == OK


def test_ffn_permute_combine_validation(lib):
    p = FAKE
    assert lib.moe_expert_ffn(p, p, p, p, p, 7, 64, 128, 8, BF16, p, p, 1 << 30,
                              None) == INVALID  # odd row count
    assert lib.moe_expert_ffn(p, p, p, p, p, 8, 64, 128, 8, BF16, p, p, 16, None) == WORKSPACE
    assert lib.moe_permute(p, p, 8, 64, 8, 2, BF16, p, p, p, p, p, 0, None) == WORKSPACE
    assert lib.moe_permute(p, p, 8, 64, 8, 2, BF16, None, p, p, p, p, 1 << 20,
                           None) == INVALID
    assert lib.moe_combine(p, p, p, 8, 64, 3, BF16, p, None) == UNSUPPORTED
    assert lib.moe_combine(p, None, p, 8, 64, 2, BF16, p, None) == INVALID


def test_status_strings(lib):
    for code in range(6):
        assert lib.moe_status_string(code)
    assert b"unknown" in lib.moe_status_string(99)


def _bind_backward(lib):
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_backward_workspace_bytes.restype = sz
    lib.moe_backward_workspace_bytes.argtypes = [i32] * 6
    args = [vp] * 6 + [i32] * 7 + [vp] * 6 + [sz, vp, sz]
    lib.moe_layer_backward.argtypes = args + [vp]
    lib.moe_layer_backward_events.argtypes = args + [vp, i32, vp]
    return lib


def test_backward_workspace_sizes(lib):
    L = _bind_backward(lib)
    d, h = 4096, 14336
    n = L.moe_backward_workspace_bytes(4096, d, h, 8, 2, BF16)
    P = 2 * 4096
    # dY (bf16), dH (fp32), [du dv] (bf16) and dX (fp32) at least
    assert n >= P * d * 2 + P * h * 4 + P * 2 * h * 2 + P * d * 4
    assert n % 1024 == 0
    assert L.moe_backward_workspace_bytes(16, d, h, 8, 2, F32) == 0      # bf16 only
    assert L.moe_backward_workspace_bytes(16, d, 14344, 8, 2, BF16) == 0  # h % 64
    assert L.moe_backward_workspace_bytes(16, d, h, 8, 3, BF16) == 0      # k != 2


def test_backward_validation(lib):
    L = _bind_backward(lib)
    p = FAKE
    T, d, h, E = 8, 64, 128, 8
    fw = lib.moe_workspace_bytes(T, d, h, E, 2, BF16)
    bw = L.moe_backward_workspace_bytes(T, d, h, E, 2, BF16)

    def call(*, x=p, dy=p, dW2=p, h_=h, dt=BF16, k=2, fws=fw, bws=bw, T_=T):
        return L.moe_layer_backward(x, p, p, p, p, dy, T_, d, h_, E, k, dt, -1, p, p, p, p, dW2,
                                    p, fws, p, bws, None)
    assert call(fws=fw - 1) == WORKSPACE
    assert call(bws=bw - 1) == WORKSPACE
    assert call(dy=None) == INVALID
    assert call(dW2=p + 4) == INVALID          # misaligned
    assert call(h_=96) == UNSUPPORTED           # h % 64 != 0
    assert call(dt=F32) == UNSUPPORTED
    assert call(k=3) == UNSUPPORTED
    assert call(T_=0, x=None, dy=None) == OK    # empty batch: nothing to do
    # the events variant checks its event array too
    assert L.moe_layer_backward_events(p, p, p, p, p, p, T, d, h, E, 2, BF16, -1, p, p, p, p,
                                       p, p, fw, p, bw, None, 3, None) == INVALID


def test_forward_train_validation(lib):
    """moe_layer_forward_train: the forward's checks, plus bf16 only, h % 64 == 0 and a
    backward workspace large enough for the kept pre-activations (2 * 2T * h fp32)."""
    L = _bind_backward(lib)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_layer_forward_train.restype = i32
    L.moe_layer_forward_train.argtypes = [vp] * 5 + [i32] * 6 + [vp, vp, sz, vp, sz, vp]
    p = FAKE
    T, d, h, E = 8, 64, 128, 8
    fw = lib.moe_workspace_bytes(T, d, h, E, 2, BF16)
    bw = L.moe_backward_workspace_bytes(T, d, h, E, 2, BF16)
    assert bw >= 2 * (2 * T) * h * 4  # the kept a and b

    def call(*, W2=p, h_=h, dt=BF16, fws=fw, bws=bw, bptr=p, T_=T, x=p):
        return L.moe_layer_forward_train(x, p, p, p, W2, T_, d, h_, E, 2, dt, p, p, fws, bptr,
                                         bws, None)
    assert call(bws=bw - 1) == WORKSPACE
    assert call(fws=fw - 1) == WORKSPACE
    assert call(bptr=None) == INVALID
    assert call(W2=None) == INVALID
    assert call(h_=96) == UNSUPPORTED           # h % 64 != 0
    assert call(dt=F32) == UNSUPPORTED
    assert call(T_=0, x=None, bptr=None, bws=0, fws=0) == OK  # empty batch: nothing queued


C_PROGRAM = r"""
#include <stdio.h>
#include "moe.h"

int main(void) {
    size_t n = moe_workspace_bytes(16, 4096, 14336, 8, 2, MOE_BF16);
    size_t bad = moe_workspace_bytes(16, 4096, 14336, 8, 3, MOE_BF16);
    moe_status st = moe_route(NULL, NULL, 4, 64, 8, 2, MOE_BF16, NULL, NULL, 0);
    printf("%zu %zu %d %s\n", n, bad, (int)st, moe_status_string(MOE_ERR_WORKSPACE));
    return 0;
}
"""


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """A plain C program (not C++; C11, which the CUDA runtime header itself needs for
    its anonymous unions) includes the header, links against libmoe.so and calls the
    host-only entry points."""
    import shutil
    import subprocess
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    if shutil.which("gcc") is None or not os.path.exists(
            os.path.join(cuda_inc, "cuda_runtime_api.h")):
        pytest.skip("gcc or the CUDA headers are not available")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.join(ROOT, "sparse_mixture_experts_26_b200")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src),
                    "-L", libdir, "-lmoe", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert int(out[0]) == lib.moe_workspace_bytes(16, 4096, 14336, 8, 2, BF16) > 0
    assert int(out[1]) == 0
    assert int(out[2]) == INVALID
    assert " ".join(out[3:]) == lib.moe_status_string(WORKSPACE).decode()
