"""The C-ABI library loads on a host without a GPU, exports every entry point the header
declares, and rejects invalid arguments on the host before any CUDA call."""
import ctypes as C
import os
import re

import pytest

import optimizer_fp8_cast_b200 as fp8
from optimizer_fp8_cast_b200 import _abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fp8train.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([A-Za-z_][A-Za-z0-9_]*)\s*\(", text)
    kw = {"if", "sizeof", "defined"}
    return sorted({n for n in names if n not in kw and not n.isupper()})


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fp8.load()


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("fp8_cast_transpose_amax", "fp8_gemm", "fp8_scale_update", "fused_adamw_multi_tensor"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = C.CDLL(fp8.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), name
    assert lib.fp8t_abi_version() == 1
    for s in range(7):
        assert lib.fp8t_status_string(s).decode() == _abi.status_name(s)


def test_invalid_arguments_rejected_on_host(lib):
    P = C.c_void_p(16 * 1024)          # aligned dummy address: never dereferenced
    U = C.c_void_p(16 * 1024 + 4)      # misaligned dummy address
    z = None
    # cast
    assert lib.fp8_cast_transpose_amax(z, 16, 16, 0, P, P, P, P, P, P, z) == 1
    assert lib.fp8_cast_transpose_amax(P, 16, 16, 7, P, P, P, P, P, P, z) == 1
    assert lib.fp8_cast_transpose_amax(P, 0, 16, 0, P, P, P, P, P, P, z) == 1
    assert lib.fp8_cast_transpose_amax(P, 24, 16, 0, P, P, P, P, P, P, z) == 2
    assert lib.fp8_cast_transpose_amax(U, 16, 16, 0, P, P, P, P, P, P, z) == 3
    assert b"misaligned" in lib.fp8t_last_error_message()
    # grouped cast: validated per tensor before anything runs
    arr = (_abi.CastTensor * 2)()
    arr[0] = _abi.CastTensor(P, 16, 16, 0, P, P, P, P, P, None)
    arr[1] = _abi.CastTensor(P, 16, 24, 1, P, P, P, P, P, None)
    assert lib.fp8_cast_transpose_amax_multi(arr, 2, z) == 2
    assert b"tensor 1" in lib.fp8t_last_error_message()
    assert lib.fp8_cast_transpose_amax_multi(arr, 0, z) == 1
    arr[1] = _abi.CastTensor(P, 16, 16, 1, P, U, P, P, P, None)
    assert lib.fp8_cast_transpose_amax_multi(arr, 2, z) == 3
    # gemm
    assert lib.fp8_gemm(z, 0, P, 0, 16, 16, 16, P, P, P, z) == 1
    assert lib.fp8_gemm(P, 0, P, 9, 16, 16, 16, P, P, P, z) == 1
    assert lib.fp8_gemm(P, 0, P, 0, 16, 20, 16, P, P, P, z) == 2
    assert lib.fp8_gemm(P, 0, P, 0, 16, 16, 1 << 31, P, P, P, z) == 2
    assert lib.fp8_gemm(P, 0, U, 0, 16, 16, 16, P, P, P, z) == 3
    # grouped gemm: validated per problem before anything runs
    g = (_abi.GemmDesc * 2)()
    g[0] = _abi.GemmDesc(P, 0, P, 0, 16, 16, 16, P, P, P)
    g[1] = _abi.GemmDesc(P, 1, P, 0, 16, 16, 24, P, P, P)
    assert lib.fp8_gemm_multi(g, 2, z) == 2 and b"problem 1" in lib.fp8t_last_error_message()
    g[1] = _abi.GemmDesc(P, 1, P, 3, 16, 16, 16, P, P, P)
    assert lib.fp8_gemm_multi(g, 2, z) == 1
    assert lib.fp8_gemm_multi(g, 0, z) == 1
    # scale update
    assert lib.fp8_scale_update(0, P, P, 16, P, 0, 0, P, P, z) == 1
    assert lib.fp8_scale_update(3, P, P, 0, P, 0, 0, P, P, z) == 1
    assert lib.fp8_scale_update(3, P, P, 16, P, 2, 0, P, P, z) == 1
    assert lib.fp8_scale_update(3, P, P, 16, P, 0, 127, P, P, z) == 1
    assert lib.fp8_scale_update(3, C.c_void_p(16 * 1024 + 2), P, 16, P, 0, 0, P, P, z) == 3
    # adamw
    arr = (_abi.AdamWTensor * 1)()
    arr[0] = _abi.AdamWTensor(P, P, P, P, P, 1000)
    need = lib.fused_adamw_workspace_bytes(arr, 1)
    assert need >= 8 and need % 256 == 0
    call = lambda a, n=1, step=1, S=1.0, ws=P, wsb=need, dstep=z: lib.fused_adamw_multi_tensor(
        a, n, 1e-3, 0.9, 0.999, 1e-8, 0.0, step, dstep, S, 1.0, z, z, ws, wsb, z)
    assert call(arr, step=0) == 1
    assert call(arr, step=0, dstep=C.c_void_p(16 * 1024 + 4)) == 3   # misaligned step counter
    assert call(arr, S=0.0) == 1
    assert call(arr, S=float("inf")) == 1
    assert call(arr, ws=None) == 1
    assert call(arr, wsb=need - 1) == 1
    bad = (_abi.AdamWTensor * 1)()
    bad[0] = _abi.AdamWTensor(U, P, P, P, P, 1000)
    assert call(bad) == 3
    bad[0] = _abi.AdamWTensor(P, P, P, P, P, 0)
    assert call(bad) == 1
    assert lib.fused_adamw_workspace_bytes(bad, 1) == 0
    assert b"numel" in lib.fp8t_last_error_message()
    assert lib.fp8t_debug_expire_waits(3) == 1 and lib.fp8t_debug_expire_waits(-1) == 1
