"""Failure detection on the GPU without a fault: the kernels' bounded waits.

Every wait inside the cast and GEMM kernels is bounded in time. The test hook
fp8t_debug_expire_waits makes those waits behave as if their barrier were never signalled (a flag
that nothing sets); with the limit shortened to 1 ms they run out, the kernels record
FP8T_ERR_TIMEOUT in the device error word, drain what they issued and return. The CUDA context
must stay usable: with the hook off and the default limit restored, the next calls are correct.
Mode 2 expires only the GEMM epilogue's waits, so TMA loads and MMAs are genuinely in flight
when the kernel aborts and drains them."""
import numpy as np
import pytest
import torch

import oracle
from optimizer_fp8_cast_b200 import Fp8TrainError
from tests._gpu import bf16_bits, dev_scalar, u8
from tests._pins import gemm_within_tolerance

pytestmark = pytest.mark.gpu


def _run_expired(fp8, mode, launch):
    fp8.fp8t_check_device_error()                   # clean start
    try:
        fp8.fp8t_set_wait_timeout_ns(1_000_000)
        fp8.fp8t_debug_expire_waits(mode)
        launch()
        with pytest.raises(Fp8TrainError) as e:
            fp8.fp8t_check_device_error()
        assert e.value.status == 6                  # FP8T_ERR_TIMEOUT
    finally:
        fp8.fp8t_debug_expire_waits(0)
        fp8.fp8t_set_wait_timeout_ns(0)
    fp8.fp8t_check_device_error()                   # the word was cleared by the read


def test_cast_waits_expire_and_context_survives(cuda_lib):
    x = (torch.randn(8192, 2048) * 3).to(torch.bfloat16)
    xd = x.cuda()
    q = torch.empty(8192, 2048, dtype=torch.uint8, device="cuda")
    qT = torch.empty(2048, 8192, dtype=torch.uint8, device="cuda")
    _run_expired(cuda_lib, 1, lambda: cuda_lib.fp8_cast_transpose_amax(
        xd, oracle.E4M3, dev_scalar(2.0), q, qT, torch.zeros(1, device="cuda")))
    amax = torch.zeros(1, device="cuda")
    cuda_lib.fp8_cast_transpose_amax(xd, oracle.E4M3, dev_scalar(2.0), q, qT, amax)
    cuda_lib.fp8t_check_device_error()
    rq, rqT, ramax, _, _ = oracle.cast_transpose_amax(bf16_bits(x), oracle.E4M3, 2.0)
    assert np.array_equal(u8(q), rq) and np.array_equal(u8(qT), rqT) and amax.item() == ramax


@pytest.mark.parametrize("mode", [1, 2])
def test_gemm_waits_expire_and_context_survives(cuda_lib, mode):
    rng = np.random.default_rng(3 + mode)
    M, N, K = 2048, 2048, 4096
    A = torch.from_numpy(rng.integers(0x20, 0x48, (M, K)).astype(np.uint8)).cuda()
    B = torch.from_numpy(rng.integers(0x20, 0x48, (N, K)).astype(np.uint8)).cuda()
    D = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    one = dev_scalar(1.0)
    _run_expired(cuda_lib, mode, lambda: cuda_lib.fp8_gemm(A, 0, B, 0, one, one, D))
    cuda_lib.fp8_gemm(A, 0, B, 0, one, one, D)
    cuda_lib.fp8t_check_device_error()
    ii = rng.integers(0, M, 512); jj = rng.integers(0, N, 512)
    R, ab = oracle.gemm_at(u8(A), 0, u8(B), 0, 1.0, 1.0, ii, jj)
    assert gemm_within_tolerance(bf16_bits(D)[ii, jj], R, ab).all()
