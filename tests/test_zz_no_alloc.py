"""The no-allocation AdamW entry point against the regular one, through the C ABI.

Some callers of this library cannot give it scratch memory: a plugin that is handed the
parameter, moment and gradient buffers by its host framework but not that framework's device
allocator, or code that must not allocate after start-up because a pool reserved all device
memory. fused_adamw_multi_tensor_noalloc serves them with a 64 KiB array built into the library.
These checks run two calls in a row (the array keeps the previous call's contents) and compare
every output with fused_adamw_multi_tensor on identical inputs, within the AdamW tolerances of
the other tests (4 f32 ulp for master, m, v; one BF16 step for the weight; 2 ulp for the norm).
"""
import ctypes as C

import numpy as np
import pytest
import torch

from optimizer_fp8_cast_b200 import _abi, synth
from tests._gpu import bf16_bits, f32
from tests._pins import ulp_distance_f32

pytestmark = pytest.mark.gpu

HP = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, loss_scale=1024.0,
          max_grad_norm=1.0)


def _state(sizes, seed):
    cfg = dict(synth.ADAMW4E9, seed=seed)
    P = [synth.adamw_tensor("master", n, i, cfg, "cuda") for i, n in enumerate(sizes)]
    M = [synth.adamw_tensor("m", n, i, cfg, "cuda") for i, n in enumerate(sizes)]
    V = [synth.adamw_tensor("v", n, i, cfg, "cuda") for i, n in enumerate(sizes)]
    G = [synth.adamw_tensor("grad", n, i, cfg, "cuda") for i, n in enumerate(sizes)]
    W = [torch.zeros(n, dtype=torch.bfloat16, device="cuda") for n in sizes]
    return P, M, V, G, W


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_lib):
    sizes = [7, 8193, 100003, 65536, 300]
    A = _state(sizes, seed=11)
    B = tuple([t.clone() for t in group] for group in A)
    ws = torch.empty(cuda_lib.fused_adamw_workspace_bytes(sizes), dtype=torch.uint8, device="cuda")
    for step in (1, 2):
        na = torch.zeros(1, device="cuda"); sa = torch.full((1,), 9, dtype=torch.int32, device="cuda")
        nb = torch.zeros(1, device="cuda"); sb = torch.full((1,), 9, dtype=torch.int32, device="cuda")
        # the gradient of the second call differs, so stale partials would show
        if step == 2:
            for ga, gb in zip(A[3], B[3]):
                ga.mul_(0.5)
                gb.mul_(0.5)
        cuda_lib.fused_adamw_multi_tensor(*A, grad_norm=na, skipped=sa, workspace=ws, step=step, **HP)
        cuda_lib.fused_adamw_multi_tensor_noalloc(*B, grad_norm=nb, skipped=sb, step=step, **HP)
        cuda_lib.fp8t_check_device_error()
        assert sa.item() == sb.item() == 0
        assert ulp_distance_f32(np.float32(na.item()), np.float32(nb.item())) <= 2
        for i in range(len(sizes)):
            for k in range(3):
                assert ulp_distance_f32(f32(A[k][i]), f32(B[k][i])).max() <= 4, (step, i, k)
            wa, wb = bf16_bits(A[4][i]).astype(np.int32), bf16_bits(B[4][i]).astype(np.int32)
            assert np.abs(wa - wb).max() <= 1


def test_noalloc_rejects_calls_beyond_its_array(cuda_lib):
    """A table whose norm partials exceed the built-in array is refused on the host with a
    message, before anything runs (the dummy pointers below are never dereferenced)."""
    lib = cuda_lib.load()
    n = 3584                                   # 14 launch tables x 592 partials > 8192 slots
    arr = (_abi.AdamWTensor * n)()
    P = C.c_void_p(1 << 20)
    for i in range(n):
        arr[i] = _abi.AdamWTensor(P, P, P, P, P, 592 * 8192)
    assert lib.fused_adamw_workspace_bytes(arr, n) > 65536
    st = lib.fused_adamw_multi_tensor_noalloc(arr, n, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None, 1.0,
                                              1.0, None, None, None)
    assert st == 2 and b"built-in array" in lib.fp8t_last_error_message()
