"""B200-native FP8 delayed-scaling Linear training step and fused AdamW.

Thin Python binding of the C ABI in ``include/fp8train.h`` (``libfp8train.so``, built in-tree for
sm_100a). Each function takes torch CUDA tensors, passes their device pointers and the current
CUDA stream to the C entry point of the same name, and raises ``Fp8TrainError`` on a non-OK
status. Every step of the path runs in the library's kernels; there is no CPU or PyTorch
fallback, and a missing library is an error.
"""
import ctypes as C
import os

import torch

from . import _abi

__all__ = ["fp8_cast_transpose_amax", "fp8_cast_transpose_amax_multi",
           "fp8_cast_transpose_amax_update_multi", "fp8_cast_transpose_amax_current_multi",
           "CURRENT_WORKSPACE_BYTES", "fp8_gemm", "fp8_gemm_multi", "fp8_scale_update", "fused_adamw_multi_tensor",
           "fused_adamw_workspace_bytes", "fused_adamw_multi_tensor_noalloc",
           "fp8_gemm_multi_sumsq", "fp8_gemm_sumsq_workspace_bytes",
           "fused_adamw_multi_tensor_presummed", "fp8_mx_cast_multi", "fp8_mx_gemm_multi",
           "fp8_mx_gemm_multi_sumsq", "fp8_mx_gemm_sumsq_workspace_bytes",
           "mx_scale_bytes",
           "fp8t_check_device_error", "fp8t_debug_expire_waits", "fp8t_set_wait_timeout_ns",
           "Fp8TrainError", "E4M3", "E5M2", "K_MAJOR", "MN_MAJOR", "AMAX_MAX", "AMAX_MOST_RECENT", "FP8_MAX", "load",
           "LIB_PATH"]

E4M3, E5M2 = 0, 1
AMAX_MAX, AMAX_MOST_RECENT = 0, 1
K_MAJOR, MN_MAJOR = 0, 1
FP8_MAX = {E4M3: 448.0, E5M2: 57344.0}
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8train.so")


class Fp8TrainError(RuntimeError):
    def __init__(self, status, where, message):
        self.status = status
        super().__init__(f"{where}: {_abi.status_name(status)} ({message})")


_lib = None


def load():
    """Load libfp8train.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m optimizer_fp8_cast_b200.build`")
        _lib = _abi.declare(C.CDLL(LIB_PATH))
    return _lib


def _check(status, where):
    if status != 0:
        raise Fp8TrainError(status, where, load().fp8t_last_error_message().decode())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return C.c_void_p(t.data_ptr())


def fp8_cast_transpose_amax(x, fmt, scale, q=None, qT=None, amax=None, scale_inv=None,
                            counters=None, stream=None):
    """Quantise BF16 ``x`` [rows, cols] with the device scalar ``scale`` (float32 [1]).

    Writes ``q`` [rows, cols] and ``qT`` [cols, rows] (uint8, optional) and ``scale_inv``
    (float32 [1], optional); max-accumulates max|x| into ``amax`` (float32 [1]: start it at 0,
    ``fp8_scale_update`` resets it after use) and adds to ``counters`` (int64 [3], optional:
    saturated, zero, non-finite)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    rows, cols = x.shape
    _check(load().fp8_cast_transpose_amax(_ptr(x), rows, cols, int(fmt), _ptr(scale), _ptr(q),
                                          _ptr(qT), _ptr(amax), _ptr(scale_inv), _ptr(counters),
                                          _stream(stream)), "fp8_cast_transpose_amax")


def _cast_array(casts):
    arr = (_abi.CastTensor * len(casts))()
    for i, c in enumerate(casts):
        x = c["x"]                  # None: a scale-update-only entry (update call only)
        assert x is None or (x.dtype == torch.bfloat16 and x.dim() == 2)
        rows, cols = (0, 0) if x is None else x.shape
        arr[i] = _abi.CastTensor(_ptr(x), rows, cols, int(c["fmt"]), _ptr(c["scale"]),
                                 _ptr(c.get("q")), _ptr(c.get("qT")), _ptr(c.get("amax")),
                                 _ptr(c.get("scale_inv")), _ptr(c.get("counters")))
    return arr


def fp8_cast_transpose_amax_multi(casts, stream=None):
    """Several casts in one launch. ``casts`` is a list of dicts with the keyword arguments of
    fp8_cast_transpose_amax (x, fmt, scale and optionally q, qT, amax, scale_inv, counters)."""
    _check(load().fp8_cast_transpose_amax_multi(_cast_array(casts), len(casts), _stream(stream)),
           "fp8_cast_transpose_amax_multi")


CURRENT_WORKSPACE_BYTES = 64


def fp8_cast_transpose_amax_current_multi(casts, margin, workspace, stream=None):
    """Current scaling: each tensor's scale (written into ``casts[i]["scale"]``) comes from its
    own amax, then the casts of fp8_cast_transpose_amax_multi run with it. ``workspace``: a
    zero-filled uint8 CUDA tensor of CURRENT_WORKSPACE_BYTES, left zero."""
    assert workspace.numel() >= CURRENT_WORKSPACE_BYTES
    _check(load().fp8_cast_transpose_amax_current_multi(_cast_array(casts), len(casts), int(margin),
                                                        _ptr(workspace), _stream(stream)),
           "fp8_cast_transpose_amax_current_multi")


def fp8_cast_transpose_amax_update_multi(casts, updates, algo, margin, ticket, stream=None):
    """The casts of fp8_cast_transpose_amax_multi and, in the same launch, the scale update of
    those tensors: ``updates[i]`` holds ``history`` (this tensor's [H] float32 row, entry 0
    newest) and ``scale_inv_next`` (1 float32, distinct from the cast's ``scale_inv``); the next
    scale is written into ``casts[i]["scale"]``. ``ticket``: one zeroed int32 on the device."""
    assert len(updates) == len(casts) and ticket.dtype == torch.int32
    H = updates[0]["history"].numel()
    arr = (_abi.CastUpdate * len(updates))()
    for i, u in enumerate(updates):
        h = u["history"]
        assert h.dtype == torch.float32 and h.numel() == H and h.is_contiguous()
        arr[i] = _abi.CastUpdate(_ptr(h), _ptr(u["scale_inv_next"]))
    _check(load().fp8_cast_transpose_amax_update_multi(_cast_array(casts), arr, len(casts), H,
                                                       int(algo), int(margin), _ptr(ticket),
                                                       _stream(stream)),
           "fp8_cast_transpose_amax_update_multi")


def fp8_gemm(A, a_fmt, B, b_fmt, a_scale_inv, b_scale_inv, D, stream=None):
    """D [M, N] bf16 = (A [M, K] . B [N, K]^T) * a_scale_inv * b_scale_inv; A, B uint8 FP8 codes."""
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2 and D.shape == (M, N) and D.dtype == torch.bfloat16
    _check(load().fp8_gemm(_ptr(A), int(a_fmt), _ptr(B), int(b_fmt), M, N, K, _ptr(a_scale_inv),
                           _ptr(b_scale_inv), _ptr(D), _stream(stream)), "fp8_gemm")


def _gemm_shape(g):
    """(M, N, K) of a descriptor dict; ``a_mn`` / ``b_mn`` mark operands stored MN-major
    (A as [K, M], B as [K, N])."""
    a_mn, b_mn = bool(g.get("a_mn")), bool(g.get("b_mn"))
    K, M = g["A"].shape if a_mn else g["A"].shape[::-1]
    K2, N = g["B"].shape if b_mn else g["B"].shape[::-1]
    assert K == K2, "inner dimensions differ"
    return M, N, K


def _gemm_array(gemms):
    arr = (_abi.GemmDesc * len(gemms))()
    for i, g in enumerate(gemms):
        M, N, K = _gemm_shape(g)
        D = g["D"]
        assert D.shape == (M, N) and D.dtype == torch.bfloat16
        arr[i] = _abi.GemmDesc(_ptr(g["A"]), int(g["a_fmt"]), _ptr(g["B"]), int(g["b_fmt"]), M, N, K,
                               _ptr(g["a_scale_inv"]), _ptr(g["b_scale_inv"]), _ptr(D),
                               MN_MAJOR if g.get("a_mn") else K_MAJOR,
                               MN_MAJOR if g.get("b_mn") else K_MAJOR)
    return arr


def fp8_gemm_sumsq_workspace_bytes(gemms):
    """Scratch bytes of fp8_gemm_multi_sumsq for these problems (dicts with a ``sumsq`` flag)."""
    flags = (C.c_int32 * len(gemms))(*[1 if g.get("sumsq") else 0 for g in gemms])
    arr = (_abi.GemmDesc * len(gemms))()                 # only the shapes are read
    for i, g in enumerate(gemms):
        arr[i].M, arr[i].N, arr[i].K = _gemm_shape(g)
    return int(load().fp8_gemm_sumsq_workspace_bytes(arr, len(gemms), flags))


def fp8_gemm_multi_sumsq(gemms, sumsq_out, workspace, stream=None):
    """fp8_gemm_multi that also writes into ``sumsq_out`` (float64 [1]) the FP64 sum of f32(D)^2
    over the problems whose dict has ``sumsq=True``. ``workspace``: uint8 CUDA tensor of
    fp8_gemm_sumsq_workspace_bytes, zero-filled once before its first use."""
    flags = (C.c_int32 * len(gemms))(*[1 if g.get("sumsq") else 0 for g in gemms])
    assert sumsq_out.dtype == torch.float64
    _check(load().fp8_gemm_multi_sumsq(_gemm_array(gemms), len(gemms), flags, _ptr(sumsq_out),
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
           "fp8_gemm_multi_sumsq")


def fp8_gemm_multi(gemms, stream=None):
    """Several GEMMs in one persistent launch. ``gemms`` is a list of dicts with the arguments of
    fp8_gemm: A, a_fmt, B, b_fmt, a_scale_inv, b_scale_inv, D."""
    _check(load().fp8_gemm_multi(_gemm_array(gemms), len(gemms), _stream(stream)), "fp8_gemm_multi")


def mx_scale_bytes(mn, k):
    """Bytes of the scale atoms of an MX operand with mn rows (M or N) and contraction k."""
    return (mn // 128) * (k // 128) * 512


def fp8_mx_cast_multi(casts, stream=None):
    """MXFP8 quantisation. ``casts``: dicts with x (BF16 [rows, cols]), fmt and q_row / sf_row
    (row-wise copy: blocks of 32 along rows) and/or q_col / sf_col (column-wise copy: blocks of
    32 down columns); codes are uint8 [rows, cols], scales uint8 tensors of mx_scale_bytes."""
    arr = (_abi.MxCastTensor * len(casts))()
    for i, c in enumerate(casts):
        x = c["x"]
        assert x.dtype == torch.bfloat16 and x.dim() == 2
        rows, cols = x.shape
        arr[i] = _abi.MxCastTensor(_ptr(x), rows, cols, int(c["fmt"]), _ptr(c.get("q_row")),
                                   _ptr(c.get("sf_row")), _ptr(c.get("q_col")), _ptr(c.get("sf_col")))
    _check(load().fp8_mx_cast_multi(arr, len(casts), _stream(stream)), "fp8_mx_cast_multi")


def _mx_gemm_array(gemms):
    arr = (_abi.MxGemmDesc * len(gemms))()
    for i, g in enumerate(gemms):
        M, N, K = _gemm_shape(g)
        D = g["D"]
        assert D.shape == (M, N) and D.dtype == torch.bfloat16
        arr[i] = _abi.MxGemmDesc(_ptr(g["A"]), _ptr(g["a_sf"]), int(g["a_fmt"]),
                                 MN_MAJOR if g.get("a_mn") else K_MAJOR, _ptr(g["B"]), _ptr(g["b_sf"]),
                                 int(g["b_fmt"]), MN_MAJOR if g.get("b_mn") else K_MAJOR, M, N, K,
                                 _ptr(D))
    return arr


def fp8_mx_gemm_multi(gemms, stream=None):
    """Block-scaled FP8 GEMMs in one launch: dicts with A, a_sf, a_fmt, (a_mn), B, b_sf, b_fmt,
    (b_mn), D; D = bf16(A . B^T) with the operands' block scales (no per-tensor scale)."""
    _check(load().fp8_mx_gemm_multi(_mx_gemm_array(gemms), len(gemms), _stream(stream)),
           "fp8_mx_gemm_multi")


def fp8_mx_gemm_sumsq_workspace_bytes(gemms):
    """Scratch bytes of fp8_mx_gemm_multi_sumsq for these problems (dicts with a ``sumsq`` flag;
    only their shapes are read)."""
    flags = (C.c_int32 * len(gemms))(*[1 if g.get("sumsq") else 0 for g in gemms])
    arr = (_abi.MxGemmDesc * len(gemms))()
    for i, g in enumerate(gemms):
        arr[i].M, arr[i].N, arr[i].K = _gemm_shape(g)
    return int(load().fp8_mx_gemm_sumsq_workspace_bytes(arr, len(gemms), flags))


def fp8_mx_gemm_multi_sumsq(gemms, sumsq_out, workspace, stream=None):
    """fp8_mx_gemm_multi that also writes into ``sumsq_out`` (float64 [1]) the FP64 sum of
    f32(D)^2 over the problems whose dict has ``sumsq=True``. ``workspace``: uint8 CUDA tensor of
    fp8_mx_gemm_sumsq_workspace_bytes, zero-filled once before its first use."""
    flags = (C.c_int32 * len(gemms))(*[1 if g.get("sumsq") else 0 for g in gemms])
    assert sumsq_out.dtype == torch.float64
    _check(load().fp8_mx_gemm_multi_sumsq(_mx_gemm_array(gemms), len(gemms), flags, _ptr(sumsq_out),
                                          _ptr(workspace), workspace.numel(), _stream(stream)),
           "fp8_mx_gemm_multi_sumsq")


def fp8_scale_update(amax, history, fp8_max, algo, margin, scale, scale_inv, stream=None):
    """Roll ``history`` [n, H] (entry 0 newest) with ``amax`` [n] (reset to 0 afterwards) and
    write the next scales."""
    n, H = history.shape
    _check(load().fp8_scale_update(n, _ptr(amax), _ptr(history), H, _ptr(fp8_max), int(algo),
                                   int(margin), _ptr(scale), _ptr(scale_inv), _stream(stream)),
           "fp8_scale_update")


def _tensor_table(master, m, v, grads, weights):
    n = len(master)
    arr = (_abi.AdamWTensor * n)()
    for i in range(n):
        for t in (master[i], m[i], v[i]):
            assert t.dtype == torch.float32
        assert grads[i].dtype == torch.bfloat16 and weights[i].dtype == torch.bfloat16
        numel = master[i].numel()
        assert m[i].numel() == v[i].numel() == grads[i].numel() == weights[i].numel() == numel
        arr[i] = _abi.AdamWTensor(_ptr(master[i]), _ptr(m[i]), _ptr(v[i]), _ptr(grads[i]),
                                  _ptr(weights[i]), numel)
    return arr, n


def fused_adamw_workspace_bytes(numels):
    arr = (_abi.AdamWTensor * len(numels))()
    for i, n in enumerate(numels):
        arr[i].numel = int(n)
    return int(load().fused_adamw_workspace_bytes(arr, len(numels)))


def fused_adamw_multi_tensor(master, m, v, grads, weights, *, lr, beta1, beta2, eps,
                             weight_decay, step, loss_scale, max_grad_norm, grad_norm=None,
                             skipped=None, workspace=None, step_counter=None, stream=None):
    """One fused AdamW step over lists of tensors (see include/fp8train.h for the arithmetic).

    ``workspace`` is a uint8 CUDA tensor of at least ``fused_adamw_workspace_bytes`` bytes.
    ``step_counter`` (int64 [1] on the device, completed steps) replaces ``step``: the call
    performs step counter+1 and stores it back unless the update is skipped, which lets a
    captured CUDA graph replay successive steps."""
    arr, n = _tensor_table(master, m, v, grads, weights)
    need = int(load().fused_adamw_workspace_bytes(arr, n))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=master[0].device)
    _check(load().fused_adamw_multi_tensor(arr, n, float(lr), float(beta1), float(beta2),
                                           float(eps), float(weight_decay), int(step),
                                           _ptr(step_counter), float(loss_scale),
                                           float(max_grad_norm),
                                           _ptr(grad_norm), _ptr(skipped), _ptr(workspace),
                                           workspace.numel(), _stream(stream)),
           "fused_adamw_multi_tensor")


def fused_adamw_multi_tensor_presummed(master, m, v, grads, weights, *, lr, beta1, beta2, eps,
                                       weight_decay, step, loss_scale, max_grad_norm, grad_sumsq,
                                       grad_norm=None, skipped=None, step_counter=None,
                                       ticket=None, casts=None, stream=None):
    """The AdamW step without its norm pass: ``grad_sumsq`` (float64 [1] on the device) holds
    the FP64 sum of f32(g)^2 over all gradients. ``ticket`` (zeroed int32 [1]) is required with
    ``step_counter``. ``casts``: None, or one entry per tensor, None or a dict (rows, cols, fmt,
    scale, and optionally q, amax, scale_inv) to cast that tensor's new BF16 weight (row-major
    codes)."""
    arr, n = _tensor_table(master, m, v, grads, weights)
    assert grad_sumsq.dtype == torch.float64
    carr = None
    if casts is not None:
        assert len(casts) == n
        carr = (_abi.AdamWCast * n)()
        for i, c in enumerate(casts):
            if c is not None:
                assert c.get("qT") is None, "weight casts inside AdamW write row-major codes only"
                carr[i] = _abi.AdamWCast(int(c["rows"]), int(c["cols"]), int(c["fmt"]),
                                         _ptr(c["scale"]), _ptr(c.get("q")),
                                         _ptr(c.get("amax")), _ptr(c.get("scale_inv")))
    _check(load().fused_adamw_multi_tensor_presummed(arr, carr, n, float(lr), float(beta1), float(beta2),
                                                     float(eps), float(weight_decay), int(step),
                                                     _ptr(step_counter), float(loss_scale),
                                                     float(max_grad_norm), _ptr(grad_sumsq),
                                                     _ptr(grad_norm), _ptr(skipped), _ptr(ticket),
                                                     _stream(stream)),
           "fused_adamw_multi_tensor_presummed")


def fused_adamw_multi_tensor_noalloc(master, m, v, grads, weights, *, lr, beta1, beta2, eps,
                                     weight_decay, step, loss_scale, max_grad_norm,
                                     grad_norm=None, skipped=None, step_counter=None, stream=None):
    """The same AdamW step, with no scratch buffer from the caller: for code that cannot
    allocate device memory (for instance a plugin that is handed the parameter buffers but not
    the framework's allocator). The library uses a 64 KiB array of its own instead; calls share
    it, so calls that overlap on the GPU race. Allocates nothing."""
    arr, n = _tensor_table(master, m, v, grads, weights)
    _check(load().fused_adamw_multi_tensor_noalloc(arr, n, float(lr), float(beta1), float(beta2),
                                                   float(eps), float(weight_decay), int(step),
                                                   _ptr(step_counter), float(loss_scale),
                                                   float(max_grad_norm),
                                                   _ptr(grad_norm), _ptr(skipped), _stream(stream)),
           "fused_adamw_multi_tensor_noalloc")


def fp8t_check_device_error(stream=None):
    """Synchronise the stream and raise if a bounded wait in a kernel expired."""
    _check(load().fp8t_check_device_error(_stream(stream)), "fp8t_check_device_error")


def fp8t_debug_expire_waits(mode):
    """Test hook: 1 = every bounded kernel wait expires, 2 = only the GEMM epilogue's, 0 = off."""
    _check(load().fp8t_debug_expire_waits(int(mode)), "fp8t_debug_expire_waits")


def fp8t_set_wait_timeout_ns(ns):
    _check(load().fp8t_set_wait_timeout_ns(int(ns)), "fp8t_set_wait_timeout_ns")
