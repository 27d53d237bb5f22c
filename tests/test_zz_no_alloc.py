"""The no-allocation AdamW entry point, through the C ABI, against the oracle.

Some callers of this library cannot give it scratch memory: a plugin that is handed the
parameter, moment and gradient buffers by its host framework but not that framework's device
allocator, or code that must not allocate after start-up because a pool reserved all device
memory. fused_adamw_multi_tensor_noalloc serves them with a 64 KiB array built into the library.
These checks run two calls in a row (the array keeps the previous call's contents: norm partials
and, with a device step counter, the step slot) and compare every output with the oracle's
AdamW on the same inputs, within the AdamW tolerances of the other tests (4 f32 ulp for master,
m, v; the BF16 weight the round-to-nearest-even of the GPU's own master and within one step of
the oracle's; 2 ulp for the norm), and with fused_adamw_multi_tensor given its own workspace.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
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


def _bf16_rne(p):
    b = p.view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


@pytest.mark.parametrize("device_counter", [False, True], ids=["host-step", "device-counter"])
def test_noalloc_matches_oracle_on_two_calls(cuda_lib, device_counter):
    sizes = [7, 8193, 100003, 65536, 300]
    A = _state(sizes, seed=11)
    B = tuple([t.clone() for t in group] for group in A)
    ws = torch.empty(cuda_lib.fused_adamw_workspace_bytes(sizes), dtype=torch.uint8, device="cuda")
    ca = torch.zeros(1, dtype=torch.int64, device="cuda") if device_counter else None
    cb = torch.zeros(1, dtype=torch.int64, device="cuda") if device_counter else None
    for step in (1, 2):
        # the gradient of the second call differs, so stale partials would show
        if step == 2:
            for ga, gb in zip(A[3], B[3]):
                ga.mul_(0.5)
                gb.mul_(0.5)
        P = [f32(t).copy() for t in B[0]]
        M = [f32(t).copy() for t in B[1]]
        V = [f32(t).copy() for t in B[2]]
        Wref = [np.zeros(n, np.uint16) for n in sizes]
        rnorm, rskip = oracle.fused_adamw(P, M, V, [bf16_bits(g) for g in B[3]], Wref,
                                          dict(HP, step=step))
        na = torch.zeros(1, device="cuda"); sa = torch.full((1,), 9, dtype=torch.int32, device="cuda")
        nb = torch.zeros(1, device="cuda"); sb = torch.full((1,), 9, dtype=torch.int32, device="cuda")
        host_step = 0 if device_counter else step       # with a counter the call performs counter+1
        cuda_lib.fused_adamw_multi_tensor(*A, grad_norm=na, skipped=sa, workspace=ws, step=host_step,
                                          step_counter=ca, **HP)
        cuda_lib.fused_adamw_multi_tensor_noalloc(*B, grad_norm=nb, skipped=sb, step=host_step,
                                                  step_counter=cb, **HP)
        cuda_lib.fp8t_check_device_error()
        assert rskip == 0 and sa.item() == sb.item() == 0
        if device_counter:
            assert ca.item() == cb.item() == step
        assert ulp_distance_f32(np.float32(nb.item()), np.float32(rnorm)) <= 2
        assert ulp_distance_f32(np.float32(na.item()), np.float32(nb.item())) <= 2
        for i in range(len(sizes)):
            for k, ref in enumerate((P, M, V)):
                assert ulp_distance_f32(f32(B[k][i]), ref[i]).max() <= 4, (step, i, k)
                assert ulp_distance_f32(f32(A[k][i]), f32(B[k][i])).max() <= 4, (step, i, k)
            wb = bf16_bits(B[4][i])
            assert np.array_equal(wb, _bf16_rne(f32(B[0][i])))
            assert np.abs(wb.astype(np.int32) - Wref[i].astype(np.int32)).max() <= 1


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
