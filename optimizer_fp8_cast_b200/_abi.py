"""ctypes declarations of the C ABI in include/fp8train.h (argument and return types only)."""
import ctypes as C

STATUS = {0: "FP8T_OK", 1: "FP8T_ERR_INVALID_ARG", 2: "FP8T_ERR_UNSUPPORTED_SHAPE",
          3: "FP8T_ERR_MISALIGNED", 4: "FP8T_ERR_UNSUPPORTED_DEVICE", 5: "FP8T_ERR_CUDA",
          6: "FP8T_ERR_TIMEOUT"}


def status_name(s):
    return STATUS.get(int(s), f"status {int(s)}")


class AdamWTensor(C.Structure):
    """fp8t_adamw_tensor."""
    _fields_ = [("master", C.c_void_p), ("m", C.c_void_p), ("v", C.c_void_p),
                ("grad_bf16", C.c_void_p), ("weight_bf16", C.c_void_p), ("numel", C.c_int64)]


class AdamWCast(C.Structure):
    """fp8t_adamw_cast."""
    _fields_ = [("rows", C.c_int64), ("cols", C.c_int64), ("fmt", C.c_int), ("d_scale", C.c_void_p),
                ("q_rowmajor", C.c_void_p), ("d_amax_inout", C.c_void_p),
                ("d_scale_inv_out", C.c_void_p)]


class CastTensor(C.Structure):
    """fp8t_cast_tensor."""
    _fields_ = [("x_bf16", C.c_void_p), ("rows", C.c_int64), ("cols", C.c_int64),
                ("fmt", C.c_int), ("d_scale", C.c_void_p), ("q_rowmajor", C.c_void_p),
                ("q_transposed", C.c_void_p), ("d_amax_inout", C.c_void_p),
                ("d_scale_inv_out", C.c_void_p), ("d_counters", C.c_void_p)]


class CastUpdate(C.Structure):
    """fp8t_cast_update."""
    _fields_ = [("d_amax_history", C.c_void_p), ("d_scale_inv_next", C.c_void_p)]


class GemmDesc(C.Structure):
    """fp8t_gemm_desc."""
    _fields_ = [("A", C.c_void_p), ("a_fmt", C.c_int), ("B", C.c_void_p), ("b_fmt", C.c_int),
                ("M", C.c_int64), ("N", C.c_int64), ("K", C.c_int64),
                ("d_a_scale_inv", C.c_void_p), ("d_b_scale_inv", C.c_void_p), ("D_bf16", C.c_void_p),
                ("a_layout", C.c_int), ("b_layout", C.c_int)]


class MxCastTensor(C.Structure):
    """fp8t_mx_cast_tensor."""
    _fields_ = [("x_bf16", C.c_void_p), ("rows", C.c_int64), ("cols", C.c_int64), ("fmt", C.c_int),
                ("q_row", C.c_void_p), ("scales_row", C.c_void_p), ("q_col", C.c_void_p),
                ("scales_col", C.c_void_p)]


class MxGemmDesc(C.Structure):
    """fp8t_mx_gemm_desc."""
    _fields_ = [("A", C.c_void_p), ("A_scales", C.c_void_p), ("a_fmt", C.c_int), ("a_layout", C.c_int),
                ("B", C.c_void_p), ("B_scales", C.c_void_p), ("b_fmt", C.c_int), ("b_layout", C.c_int),
                ("M", C.c_int64), ("N", C.c_int64), ("K", C.c_int64), ("D_bf16", C.c_void_p)]


def declare(L):
    vp, i32, i64, f32 = C.c_void_p, C.c_int32, C.c_int64, C.c_float
    L.fp8_cast_transpose_amax.restype = C.c_int
    L.fp8_cast_transpose_amax.argtypes = [vp, i64, i64, C.c_int, vp, vp, vp, vp, vp, vp, vp]
    L.fp8_cast_transpose_amax_multi.restype = C.c_int
    L.fp8_cast_transpose_amax_multi.argtypes = [C.POINTER(CastTensor), i32, vp]
    L.fp8_cast_transpose_amax_update_multi.restype = C.c_int
    L.fp8_cast_transpose_amax_update_multi.argtypes = [C.POINTER(CastTensor), C.POINTER(CastUpdate),
                                                       i32, i32, C.c_int, i32, vp, vp]
    L.fp8_gemm_multi.restype = C.c_int
    L.fp8_gemm_multi.argtypes = [C.POINTER(GemmDesc), i32, vp]
    L.fp8_cast_transpose_amax_current_multi.restype = C.c_int
    L.fp8_cast_transpose_amax_current_multi.argtypes = [C.POINTER(CastTensor), i32, i32, vp, vp]
    L.fp8_gemm_multi_sumsq.restype = C.c_int
    L.fp8_gemm_multi_sumsq.argtypes = [C.POINTER(GemmDesc), i32, C.POINTER(C.c_int32), vp, vp,
                                       C.c_size_t, vp]
    L.fp8_gemm_sumsq_workspace_bytes.restype = C.c_size_t
    L.fp8_gemm_sumsq_workspace_bytes.argtypes = [C.POINTER(GemmDesc), i32, C.POINTER(C.c_int32)]
    L.fused_adamw_multi_tensor_presummed.restype = C.c_int
    L.fused_adamw_multi_tensor_presummed.argtypes = [C.POINTER(AdamWTensor), C.POINTER(AdamWCast),
                                                     i32, f32, f32, f32,
                                                     f32, f32, i64, vp, f32, f32, vp, vp, vp, vp,
                                                     vp]
    L.fp8_mx_cast_multi.restype = C.c_int
    L.fp8_mx_cast_multi.argtypes = [C.POINTER(MxCastTensor), i32, vp]
    L.fp8_mx_gemm_multi.restype = C.c_int
    L.fp8_mx_gemm_multi.argtypes = [C.POINTER(MxGemmDesc), i32, vp]
    L.fp8_mx_gemm_multi_sumsq.restype = C.c_int
    L.fp8_mx_gemm_multi_sumsq.argtypes = [C.POINTER(MxGemmDesc), i32, C.POINTER(C.c_int32), vp, vp,
                                          C.c_size_t, vp]
    L.fp8_mx_gemm_sumsq_workspace_bytes.restype = C.c_size_t
    L.fp8_mx_gemm_sumsq_workspace_bytes.argtypes = [C.POINTER(MxGemmDesc), i32, C.POINTER(C.c_int32)]
    L.fp8_gemm.restype = C.c_int
    L.fp8_gemm.argtypes = [vp, C.c_int, vp, C.c_int, i64, i64, i64, vp, vp, vp, vp]
    L.fp8_scale_update.restype = C.c_int
    L.fp8_scale_update.argtypes = [i32, vp, vp, i32, vp, C.c_int, i32, vp, vp, vp]
    L.fused_adamw_multi_tensor.restype = C.c_int
    L.fused_adamw_multi_tensor.argtypes = [C.POINTER(AdamWTensor), i32, f32, f32, f32, f32, f32,
                                           i64, vp, f32, f32, vp, vp, vp, C.c_size_t, vp]
    L.fused_adamw_multi_tensor_noalloc.restype = C.c_int
    L.fused_adamw_multi_tensor_noalloc.argtypes = [C.POINTER(AdamWTensor), i32, f32, f32, f32, f32,
                                                   f32, i64, vp, f32, f32, vp, vp, vp]
    L.fused_adamw_workspace_bytes.restype = C.c_size_t
    L.fused_adamw_workspace_bytes.argtypes = [C.POINTER(AdamWTensor), i32]
    L.fp8t_check_device_error.restype = C.c_int
    L.fp8t_check_device_error.argtypes = [vp]
    L.fp8t_debug_expire_waits.restype = C.c_int
    L.fp8t_debug_expire_waits.argtypes = [i32]
    L.fp8t_set_wait_timeout_ns.restype = C.c_int
    L.fp8t_set_wait_timeout_ns.argtypes = [C.c_uint64]
    L.fp8t_status_string.restype = C.c_char_p
    L.fp8t_status_string.argtypes = [C.c_int]
    L.fp8t_last_error_message.restype = C.c_char_p
    L.fp8t_last_error_message.argtypes = []
    L.fp8t_abi_version.restype = i32
    L.fp8t_abi_version.argtypes = []
    return L
