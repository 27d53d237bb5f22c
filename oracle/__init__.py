"""CPU oracle of the FP8 delayed-scaling Linear step and fused AdamW (numpy front end).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package; the product path (``optimizer_fp8_cast_b200``) never
does and shares no code with it. The arithmetic lives in ``fp8_oracle.c`` (plain C, one thread);
this module only marshals numpy arrays into it.

Sources, cited by page title and section:
  [P1] "算子与编译器：FP8 训练与优化器 Kernel"
  [P2] "FP8 混合精度训练工程实践：从 H100 到大模型训练的范式跃迁"
  [P3] "LLM FP8 微调上线生产实战：用 Amax Scaling、层级白名单与 BF16 回退守住收敛"

Every function is pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle_*.py`` against
what the pages and mathematics fix (printed constants, closed forms, brute force, library
special cases). No function here is "parity unpinned".
"""
import ctypes as C

import numpy as np

from .build import build_oracle

E4M3, E5M2 = 0, 1
AMAX_MAX, AMAX_MOST_RECENT = 0, 1
FP8_MAX = {E4M3: 448.0, E5M2: 57344.0}   # [P2 §一]

_lib = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(build_oracle())
        u8p, u16p, f32p, f64p, i64p, u64p = (C.POINTER(t) for t in (
            C.c_uint8, C.c_uint16, C.c_float, C.c_double, C.c_int64, C.c_uint64))
        L.orc_bf16_to_f32.restype = C.c_float
        L.orc_bf16_to_f32.argtypes = [C.c_uint16]
        L.orc_f32_to_bf16.restype = C.c_uint16
        L.orc_f32_to_bf16.argtypes = [C.c_float]
        L.orc_fp8_decode.restype = C.c_double
        L.orc_fp8_decode.argtypes = [C.c_uint8, C.c_int]
        L.orc_fp8_encode.restype = C.c_uint8
        L.orc_fp8_encode.argtypes = [C.c_float, C.c_int]
        L.orc_fp8_encode_array.restype = None
        L.orc_fp8_encode_array.argtypes = [f32p, C.c_int64, C.c_int, u8p]
        L.orc_fp8_is_finite.restype = C.c_int
        L.orc_fp8_is_finite.argtypes = [C.c_uint8, C.c_int]
        L.orc_cast_transpose_amax.restype = None
        L.orc_cast_transpose_amax.argtypes = [u16p, C.c_int64, C.c_int64, C.c_int, C.c_float,
                                              u8p, u8p, f32p, f32p, u64p]
        L.orc_scale_update.restype = None
        L.orc_scale_update.argtypes = [C.c_int32, f32p, f32p, C.c_int32, f32p, C.c_int,
                                       C.c_int32, f32p, f32p]
        L.orc_gemm.restype = None
        L.orc_gemm.argtypes = [u8p, C.c_int, u8p, C.c_int, C.c_int64, C.c_int64, C.c_int64,
                               C.c_float, C.c_float, u16p, f64p]
        L.orc_gemm_at.restype = None
        L.orc_gemm_at.argtypes = [u8p, C.c_int, u8p, C.c_int, C.c_int64, C.c_float, C.c_float,
                                  C.c_int64, i64p, i64p, u16p, f64p]
        pp = C.POINTER(C.c_void_p)
        L.orc_global_norm.restype = C.c_float
        L.orc_global_norm.argtypes = [C.c_int32, pp, i64p, C.c_float]
        L.orc_adamw_update.restype = C.c_int
        L.orc_adamw_update.argtypes = [C.c_int32, pp, pp, pp, pp, pp, i64p, C.c_float,
                                       C.c_float, C.c_float, C.c_float, C.c_float, C.c_int64,
                                       C.c_float, C.c_float, C.c_float]
        L.orc_fused_adamw.restype = C.c_int
        L.orc_fused_adamw.argtypes = [C.c_int32, pp, pp, pp, pp, pp, i64p, C.c_float,
                                      C.c_float, C.c_float, C.c_float, C.c_float, C.c_int64,
                                      C.c_float, C.c_float, f32p]
        L.orc_e8m0_decode.restype = C.c_double
        L.orc_e8m0_decode.argtypes = [C.c_uint8]
        L.orc_mx_quantise.restype = None
        L.orc_mx_quantise.argtypes = [u16p, C.c_int64, C.c_int64, C.c_int, C.c_int, u8p, u8p]
        L.orc_mx_gemm.restype = None
        L.orc_mx_gemm.argtypes = [u8p, u8p, C.c_int, u8p, u8p, C.c_int, C.c_int64, C.c_int64,
                                  C.c_int64, u16p, f64p]
        L.orc_set_threads.restype = C.c_int
        L.orc_set_threads.argtypes = [C.c_int]
        L.orc_get_threads.restype = C.c_int
        L.orc_get_threads.argtypes = []
        L.orc_mx_gemm_at.restype = None
        L.orc_mx_gemm_at.argtypes = [u8p, u8p, C.c_int, u8p, u8p, C.c_int, C.c_int64, C.c_int64,
                                     i64p, i64p, u16p, f64p]
        _lib = L
    return _lib


def _ptr(a, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.POINTER(ctype))


def set_threads(n: int) -> int:
    """Host threads the oracle's loops may use (n <= 0: every core). Results do not depend on
    it: only independent pieces are split, and sums keep their fixed order. Returns the count."""
    return int(lib().orc_set_threads(int(n)))


def get_threads() -> int:
    return int(lib().orc_get_threads())


# ----------------------------------------------------------------------------- scalars
def bf16_to_f32(bits: int) -> float:
    return lib().orc_bf16_to_f32(int(bits))


def f32_to_bf16(x: float) -> int:
    return int(lib().orc_f32_to_bf16(float(x)))


def fp8_decode(code: int, fmt: int) -> float:
    """Value of one FP8 code [P2 §一]."""
    return float(lib().orc_fp8_decode(int(code), int(fmt)))


def fp8_encode(x: float, fmt: int) -> int:
    """FP8 code of an f32 value: round to nearest even, saturate to +-max, NaN -> 0x7F."""
    return int(lib().orc_fp8_encode(float(x), int(fmt)))


def decode_table(fmt: int) -> np.ndarray:
    """All 256 code values as float64 (NaN / inf where the format has them)."""
    return np.array([fp8_decode(c, fmt) for c in range(256)], dtype=np.float64)


def encode_array(x_f32: np.ndarray, fmt: int) -> np.ndarray:
    """Encode every element of an f32 array."""
    x = np.ascontiguousarray(x_f32, dtype=np.float32).reshape(-1)
    out = np.empty(x.size, np.uint8)
    lib().orc_fp8_encode_array(_ptr(x, C.c_float), x.size, int(fmt), _ptr(out, C.c_uint8))
    return out.reshape(np.shape(x_f32))


# ----------------------------------------------------------------------------- cast
def cast_transpose_amax(x_bf16: np.ndarray, fmt: int, scale: float, want_q=True, want_qT=True,
                        amax_in=0.0):
    """Oracle of fp8_cast_transpose_amax on a 2-D uint16 (BF16 bits) array.

    Returns (q, qT, amax, scale_inv, counters[3]); amax is max-accumulated onto amax_in."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.uint8) if want_q else None
    qT = np.empty((cols, rows), np.uint8) if want_qT else None
    amax = np.array([amax_in], np.float32)
    sinv = np.zeros(1, np.float32)
    cnt = np.zeros(3, np.uint64)
    lib().orc_cast_transpose_amax(_ptr(x, C.c_uint16), rows, cols, int(fmt),
                                  float(np.float32(scale)), _ptr(q, C.c_uint8),
                                  _ptr(qT, C.c_uint8), _ptr(amax, C.c_float),
                                  _ptr(sinv, C.c_float), _ptr(cnt, C.c_uint64))
    return q, qT, amax[0], sinv[0], cnt


def cast_current(x_bf16, fmt, margin, prev_scale, want_q=True, want_qT=True):
    """Oracle of fp8_cast_transpose_amax_current_multi for one tensor: current scaling.

    "FP8 混合精度训练工程实践" §四 (FP8Tensor.quantize measures amax = max|x| of the tensor it is
    about to quantise) with the scale rule of "LLM FP8 微调上线生产实战" 核心原理
    (scale = (FP8_MAX / amax) / 2^margin), applied without delay: the amax of x, the scale that
    the scale update forms from a one-entry history holding it (its zero / non-finite / overflow
    readings included), then the cast with that scale.
    Returns (q, qT, amax, scale, scale_inv, counters)."""
    _, _, amax, _, _ = cast_transpose_amax(x_bf16, fmt, 1.0, False, False)
    hist = np.zeros((1, 1), np.float32)
    scale = np.array([prev_scale], np.float32)
    sinv = np.zeros(1, np.float32)
    scale_update(np.array([amax], np.float32), hist, [FP8_MAX[fmt]], AMAX_MOST_RECENT, margin,
                 scale, sinv)
    q, qT, a, si, cnt = cast_transpose_amax(x_bf16, fmt, scale[0], want_q, want_qT)
    return q, qT, a, scale[0], si, cnt


# ----------------------------------------------------------------------------- scale update
def scale_update(amax, hist, fp8_max, algo, margin, scale, scale_inv):
    """Oracle of fp8_scale_update. hist [n, H], scale and scale_inv [n] are updated in place;
    amax is reset to 0 in place when it is a float32 array (a copy is consumed otherwise)."""
    if not (isinstance(amax, np.ndarray) and amax.dtype == np.float32 and amax.flags["C_CONTIGUOUS"]):
        amax = np.ascontiguousarray(amax, np.float32)
    fp8_max = np.ascontiguousarray(fp8_max, np.float32)
    assert hist.dtype == np.float32 and hist.flags["C_CONTIGUOUS"] and hist.ndim == 2
    assert scale.dtype == np.float32 and scale_inv.dtype == np.float32
    n, H = hist.shape
    lib().orc_scale_update(n, _ptr(amax, C.c_float), _ptr(hist, C.c_float), H,
                           _ptr(fp8_max, C.c_float), int(algo), int(margin),
                           _ptr(scale, C.c_float), _ptr(scale_inv, C.c_float))


# ----------------------------------------------------------------------------- GEMM
def gemm(A, afmt, B, bfmt, a_scale_inv, b_scale_inv, want_abs=False):
    """Oracle of fp8_gemm: D = bf16(A . B^T * (sa*sb)), A [M,K] u8, B [N,K] u8 -> D u16 [M,N]."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    D = np.empty((M, N), np.uint16)
    ab = np.empty((M, N), np.float64) if want_abs else None
    lib().orc_gemm(_ptr(A, C.c_uint8), int(afmt), _ptr(B, C.c_uint8), int(bfmt), M, N, K,
                   float(np.float32(a_scale_inv)), float(np.float32(b_scale_inv)),
                   _ptr(D, C.c_uint16), _ptr(ab, C.c_double))
    return (D, ab) if want_abs else D


def gemm_at(A, afmt, B, bfmt, a_scale_inv, b_scale_inv, ii, jj):
    """The oracle GEMM at output positions (ii[s], jj[s]); returns (D_bf16 bits, abs_sum)."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    K = A.shape[1]
    assert B.shape[1] == K
    ii = np.ascontiguousarray(ii, np.int64)
    jj = np.ascontiguousarray(jj, np.int64)
    assert ii.shape == jj.shape
    assert (ii >= 0).all() and (ii < A.shape[0]).all() and (jj >= 0).all() and (jj < B.shape[0]).all()
    out = np.empty(ii.shape, np.uint16)
    ab = np.empty(ii.shape, np.float64)
    lib().orc_gemm_at(_ptr(A, C.c_uint8), int(afmt), _ptr(B, C.c_uint8), int(bfmt), K,
                      float(np.float32(a_scale_inv)), float(np.float32(b_scale_inv)), ii.size,
                      _ptr(ii, C.c_int64), _ptr(jj, C.c_int64), _ptr(out, C.c_uint16),
                      _ptr(ab, C.c_double))
    return out, ab


# ----------------------------------------------------------------------------- MXFP8
def e8m0_decode(code):
    """Value of an E8M0 block-scale code: 2^(code - 127), 0xFF = NaN ("FP8 混合精度训练工程实践" §九)."""
    return lib().orc_e8m0_decode(int(code))


def mx_quantise(x_bf16, axis, fmt):
    """MX block quantisation (blocks of 32 along a row for axis 0, down a column for axis 1) of
    a 2-D uint16 (BF16 bits) array; returns (q [rows, cols], sf) with sf [rows, cols/32] for
    axis 0 and [rows/32, cols] for axis 1."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    assert (cols if axis == 0 else rows) % 32 == 0
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // 32) if axis == 0 else (rows // 32, cols), np.uint8)
    lib().orc_mx_quantise(_ptr(x, C.c_uint16), rows, cols, int(axis), int(fmt), _ptr(q, C.c_uint8),
                          _ptr(sf, C.c_uint8))
    return q, sf


def mx_gemm(A, sfa, afmt, B, sfb, bfmt, want_abs=False):
    """MX GEMM oracle: D = bf16(sum over K of a * b * 2^(Xa + Xb)); A [M, K], B [N, K] codes,
    sfa [M, K/32], sfb [N, K/32] E8M0 codes (all K-contiguous)."""
    A, B = np.ascontiguousarray(A, np.uint8), np.ascontiguousarray(B, np.uint8)
    sfa, sfb = np.ascontiguousarray(sfa, np.uint8), np.ascontiguousarray(sfb, np.uint8)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and K % 32 == 0 and sfa.shape == (M, K // 32) and sfb.shape == (N, K // 32)
    D = np.empty((M, N), np.uint16)
    ab = np.empty((M, N), np.float64) if want_abs else None
    lib().orc_mx_gemm(_ptr(A, C.c_uint8), _ptr(sfa, C.c_uint8), int(afmt), _ptr(B, C.c_uint8),
                      _ptr(sfb, C.c_uint8), int(bfmt), M, N, K, _ptr(D, C.c_uint16),
                      _ptr(ab, C.c_double))
    return (D, ab) if want_abs else D


def mx_gemm_at(A, sfa, afmt, B, sfb, bfmt, ii, jj):
    """The MX GEMM oracle at output positions (ii[s], jj[s]); returns (D bits, abs_sum)."""
    A, B = np.ascontiguousarray(A, np.uint8), np.ascontiguousarray(B, np.uint8)
    sfa, sfb = np.ascontiguousarray(sfa, np.uint8), np.ascontiguousarray(sfb, np.uint8)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and K % 32 == 0 and sfa.shape == (M, K // 32) and sfb.shape == (N, K // 32)
    ii = np.ascontiguousarray(ii, np.int64)
    jj = np.ascontiguousarray(jj, np.int64)
    assert ii.shape == jj.shape
    assert (ii >= 0).all() and (ii < M).all() and (jj >= 0).all() and (jj < N).all()
    out = np.empty(ii.shape, np.uint16)
    ab = np.empty(ii.shape, np.float64)
    lib().orc_mx_gemm_at(_ptr(A, C.c_uint8), _ptr(sfa, C.c_uint8), int(afmt), _ptr(B, C.c_uint8),
                         _ptr(sfb, C.c_uint8), int(bfmt), K, ii.size, _ptr(ii, C.c_int64),
                         _ptr(jj, C.c_int64), _ptr(out, C.c_uint16), _ptr(ab, C.c_double))
    return out, ab


# ----------------------------------------------------------------------------- AdamW
def _ptr_array(arrays):
    arr = (C.c_void_p * len(arrays))()
    for i, a in enumerate(arrays):
        if a is not None:
            assert a.flags["C_CONTIGUOUS"]
            arr[i] = a.ctypes.data
    return arr


def global_norm(grads, loss_scale):
    """Oracle global norm of the unscaled gradient (list of uint16 BF16 arrays)."""
    grads = [np.ascontiguousarray(g, np.uint16).reshape(-1) for g in grads]
    numel = np.array([g.size for g in grads], np.int64)
    return float(lib().orc_global_norm(len(grads), _ptr_array(grads), _ptr(numel, C.c_int64),
                                       float(loss_scale)))


def adamw_update(master, m, v, grads, w, hp, norm):
    """Oracle AdamW given the global norm; lists of arrays updated in place. Returns skipped."""
    n = len(master)
    numel = np.array([a.size for a in master], np.int64)
    return int(lib().orc_adamw_update(
        n, _ptr_array(master), _ptr_array(m), _ptr_array(v), _ptr_array(grads),
        _ptr_array(w) if w is not None else _ptr_array([None] * n), _ptr(numel, C.c_int64),
        hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], int(hp["step"]),
        hp["loss_scale"], hp["max_grad_norm"], float(norm)))


def fused_adamw(master, m, v, grads, w, hp):
    """Oracle of fused_adamw_multi_tensor; arrays updated in place. Returns (norm, skipped)."""
    n = len(master)
    numel = np.array([a.size for a in master], np.int64)
    norm = np.zeros(1, np.float32)
    skipped = lib().orc_fused_adamw(
        n, _ptr_array(master), _ptr_array(m), _ptr_array(v), _ptr_array(grads),
        _ptr_array(w) if w is not None else _ptr_array([None] * n), _ptr(numel, C.c_int64),
        hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], int(hp["step"]),
        hp["loss_scale"], hp["max_grad_norm"], _ptr(norm, C.c_float))
    return float(norm[0]), int(skipped)
