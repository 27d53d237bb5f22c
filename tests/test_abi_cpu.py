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
    assert lib.fp8t_abi_version() == 2
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
    # cast with the scale update in the same launch
    Q = C.c_void_p(32 * 1024)
    arr[1] = _abi.CastTensor(P, 16, 16, 1, P, P, P, P, P, None)
    ups = (_abi.CastUpdate * 2)()
    ups[0] = _abi.CastUpdate(P, Q)
    ups[1] = _abi.CastUpdate(P, Q)
    upd = lambda u=ups, H=16, algo=0, margin=0, ticket=P: lib.fp8_cast_transpose_amax_update_multi(
        arr, u, 2, H, algo, margin, ticket, z)
    assert upd(u=None) == 1
    assert upd(ticket=None) == 1 and upd(ticket=C.c_void_p(16 * 1024 + 2)) == 1
    assert upd(H=0) == 1 and upd(H=65537) == 1
    assert upd(algo=2) == 1 and upd(margin=127) == 1
    ups[1] = _abi.CastUpdate(P, P)                 # the next inverse scale over the used one
    assert upd() == 1 and b"scale_inv_next must differ" in lib.fp8t_last_error_message()
    ups[1] = _abi.CastUpdate(None, Q)
    assert upd() == 1
    ups[1] = _abi.CastUpdate(C.c_void_p(16 * 1024 + 2), Q)
    assert upd() == 3
    ups[1] = _abi.CastUpdate(P, Q)
    arr[1] = _abi.CastTensor(None, 0, 0, 0, P, P, None, P, None, None)   # update only: no outputs
    assert upd() == 1
    assert lib.fp8_cast_transpose_amax_multi(
        (_abi.CastTensor * 1)(_abi.CastTensor(None, 0, 0, 0, P, None, None, P, None, None)), 1, z) == 1
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
    g[1] = _abi.GemmDesc(P, 1, P, 0, 16, 16, 16, P, P, P, 0, 2)     # unknown operand layout
    assert lib.fp8_gemm_multi(g, 2, z) == 1 and b"layout" in lib.fp8t_last_error_message()
    assert lib.fp8_gemm_multi(g, 0, z) == 1
    # grouped gemm with the sum of squares
    g[1] = _abi.GemmDesc(P, 1, P, 0, 16, 16, 16, P, P, P)
    flags = (C.c_int32 * 2)(0, 1)
    need = lib.fp8_gemm_sumsq_workspace_bytes(g, 2, flags)
    assert need == 256 + 8 * 8                          # one 256 x 256 tile, 8 partial slots
    W = C.c_void_p(64 * 1024)                           # 256-byte aligned
    assert lib.fp8_gemm_multi_sumsq(g, 2, None, P, W, need, z) == 1
    assert lib.fp8_gemm_multi_sumsq(g, 2, flags, None, W, need, z) == 1
    assert lib.fp8_gemm_multi_sumsq(g, 2, flags, P, C.c_void_p(16 * 1024 + 16), need, z) == 1  # not 256-aligned
    assert lib.fp8_gemm_multi_sumsq(g, 2, flags, P, W, need - 1, z) == 1
    assert lib.fp8_gemm_sumsq_workspace_bytes(g, 2, (C.c_int32 * 2)(0, 0)) == 0
    assert lib.fp8_gemm_multi_sumsq(g, 2, (C.c_int32 * 2)(0, 0), P, W, need, z) == 1
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
    assert call(bad) == 1 and b"numel" in lib.fp8t_last_error_message()
    pre = lambda a, sumsq=P, dstep=z, ticket=z, casts=None: lib.fused_adamw_multi_tensor_presummed(
        a, casts, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, dstep, 1.0, 1.0, sumsq, z, z, ticket, z)
    assert pre(arr, sumsq=None) == 1
    assert pre(arr, sumsq=C.c_void_p(16 * 1024 + 4)) == 3
    assert pre(arr, dstep=P) == 1                       # a device counter needs a ticket
    assert pre(bad) == 1
    # weight casts inside AdamW: rows x cols must be numel, multiples of 16
    w16 = (_abi.AdamWTensor * 1)()
    w16[0] = _abi.AdamWTensor(P, P, P, P, P, 32 * 48)
    cast = (_abi.AdamWCast * 1)()
    cast[0] = _abi.AdamWCast(32, 40, 0, P, P, P, P)
    assert pre(w16, casts=cast) == 2
    cast[0] = _abi.AdamWCast(32, 48, 5, P, P, P, P)
    assert pre(w16, casts=cast) == 1
    cast[0] = _abi.AdamWCast(32, 48, 0, None, P, P, P)
    assert pre(w16, casts=cast) == 1
    cast[0] = _abi.AdamWCast(32, 48, 0, P, U, P, P)
    assert pre(w16, casts=cast) == 3
    assert lib.fp8t_debug_expire_waits(3) == 1 and lib.fp8t_debug_expire_waits(-1) == 1
