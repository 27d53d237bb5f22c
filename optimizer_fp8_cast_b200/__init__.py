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

__all__ = ["fp8_cast_transpose_amax", "fp8_cast_transpose_amax_multi", "fp8_gemm", "fp8_gemm_multi", "fp8_scale_update", "fused_adamw_multi_tensor",
           "fused_adamw_workspace_bytes", "fused_adamw_multi_tensor_noalloc",
           "fp8t_check_device_error", "fp8t_debug_expire_waits", "fp8t_set_wait_timeout_ns",
           "Fp8TrainError", "E4M3", "E5M2", "AMAX_MAX", "AMAX_MOST_RECENT", "FP8_MAX", "load",
           "LIB_PATH"]

E4M3, E5M2 = 0, 1
AMAX_MAX, AMAX_MOST_RECENT = 0, 1
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


def fp8_cast_transpose_amax_multi(casts, stream=None):
    """Several casts in one launch. ``casts`` is a list of dicts with the keyword arguments of
    fp8_cast_transpose_amax (x, fmt, scale and optionally q, qT, amax, scale_inv, counters)."""
    arr = (_abi.CastTensor * len(casts))()
    for i, c in enumerate(casts):
        x = c["x"]
        assert x.dtype == torch.bfloat16 and x.dim() == 2
        arr[i] = _abi.CastTensor(_ptr(x), x.shape[0], x.shape[1], int(c["fmt"]), _ptr(c["scale"]),
                                 _ptr(c.get("q")), _ptr(c.get("qT")), _ptr(c.get("amax")),
                                 _ptr(c.get("scale_inv")), _ptr(c.get("counters")))
    _check(load().fp8_cast_transpose_amax_multi(arr, len(casts), _stream(stream)),
           "fp8_cast_transpose_amax_multi")


def fp8_gemm(A, a_fmt, B, b_fmt, a_scale_inv, b_scale_inv, D, stream=None):
    """D [M, N] bf16 = (A [M, K] . B [N, K]^T) * a_scale_inv * b_scale_inv; A, B uint8 FP8 codes."""
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2 and D.shape == (M, N) and D.dtype == torch.bfloat16
    _check(load().fp8_gemm(_ptr(A), int(a_fmt), _ptr(B), int(b_fmt), M, N, K, _ptr(a_scale_inv),
                           _ptr(b_scale_inv), _ptr(D), _stream(stream)), "fp8_gemm")


def fp8_gemm_multi(gemms, stream=None):
    """Several GEMMs in one persistent launch. ``gemms`` is a list of dicts with the arguments of
    fp8_gemm: A, a_fmt, B, b_fmt, a_scale_inv, b_scale_inv, D."""
    arr = (_abi.GemmDesc * len(gemms))()
    for i, g in enumerate(gemms):
        A, B, D = g["A"], g["B"], g["D"]
        M, K = A.shape
        N, K2 = B.shape
        assert K == K2 and D.shape == (M, N) and D.dtype == torch.bfloat16
        arr[i] = _abi.GemmDesc(_ptr(A), int(g["a_fmt"]), _ptr(B), int(g["b_fmt"]), M, N, K,
                               _ptr(g["a_scale_inv"]), _ptr(g["b_scale_inv"]), _ptr(D))
    _check(load().fp8_gemm_multi(arr, len(gemms), _stream(stream)), "fp8_gemm_multi")


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
