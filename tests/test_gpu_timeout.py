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


def test_expired_cast_leaves_scale_state_alone(cuda_lib):
    """The cast launch that also updates the scales: when its waits expire, its amax may be
    incomplete, so the last CTA leaves history, scale and amax slot as they were (and resets
    its ticket); the next call performs the update normally."""
    x = (torch.randn(4096, 2048) * 3).to(torch.bfloat16).cuda()
    scale = torch.tensor([2.0], device="cuda")
    hist = torch.full((16,), 5.0, device="cuda")
    amax = torch.zeros(1, device="cuda")
    used, nxt = torch.zeros(1, device="cuda"), torch.zeros(1, device="cuda")
    ticket = torch.zeros(1, dtype=torch.int32, device="cuda")
    # with q^T requested the tiled kernel runs (the streaming one has no waits to expire)
    casts = [dict(x=x, fmt=oracle.E4M3, scale=scale, q=torch.empty(4096, 2048, dtype=torch.uint8, device="cuda"),
                  qT=torch.empty(2048, 4096, dtype=torch.uint8, device="cuda"), amax=amax, scale_inv=used)]
    ups = [dict(history=hist, scale_inv_next=nxt)]
    _run_expired(cuda_lib, 1, lambda: cuda_lib.fp8_cast_transpose_amax_update_multi(
        casts, ups, oracle.AMAX_MAX, 0, ticket))
    assert scale.item() == 2.0 and nxt.item() == 0.0 and ticket.item() == 0
    assert torch.equal(hist, torch.full((16,), 5.0, device="cuda"))
    amax.zero_()
    cuda_lib.fp8_cast_transpose_amax_update_multi(casts, ups, oracle.AMAX_MAX, 0, ticket)
    cuda_lib.fp8t_check_device_error()
    a = float(x.float().abs().max())
    assert hist[0].item() == a and hist[1].item() == 5.0 and amax.item() == 0.0
    assert scale.item() == np.float32(448.0) / np.float32(max(a, 5.0))


def test_expired_gemm_sum_of_squares_is_nan(cuda_lib):
    """fp8_gemm_multi_sumsq with expired epilogue waits reports a NaN sum (so a following AdamW
    skips its update) and leaves its workspace ticket at zero."""
    rng = np.random.default_rng(9)
    A = torch.from_numpy(rng.integers(0x20, 0x48, (1024, 2048)).astype(np.uint8)).cuda()
    B = torch.from_numpy(rng.integers(0x20, 0x48, (1024, 2048)).astype(np.uint8)).cuda()
    one = dev_scalar(1.0)
    g = [dict(A=A, a_fmt=0, B=B, b_fmt=0, a_scale_inv=one, b_scale_inv=one, sumsq=True,
              D=torch.empty(1024, 1024, dtype=torch.bfloat16, device="cuda"))]
    ws = torch.zeros(cuda_lib.fp8_gemm_sumsq_workspace_bytes(g), dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    _run_expired(cuda_lib, 2, lambda: cuda_lib.fp8_gemm_multi_sumsq(g, out, ws))
    assert np.isnan(out.item()) and not ws[:8].any()      # ticket and abort word back at zero
    cuda_lib.fp8_gemm_multi_sumsq(g, out, ws)
    cuda_lib.fp8t_check_device_error()
    d = g[0]["D"].float().double()
    assert abs(out.item() - float((d * d).sum())) <= 1e-12 * float((d * d).sum())


def _mx_problem(M, N, K, seed):
    """K-major E4M3 codes and atom-ordered scales of A [M, K] and B [N, K] (plain copies too)."""
    rng = np.random.default_rng(seed)
    qa = rng.integers(0x20, 0x48, (M, K)).astype(np.uint8)
    qb = rng.integers(0x20, 0x48, (N, K)).astype(np.uint8)
    sa = rng.integers(120, 134, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(120, 134, (N, K // 32)).astype(np.uint8)

    def atoms(plain):
        mn, kk = plain.shape
        a = plain.reshape(mn // 128, 4, 32, kk // 4, 4).transpose(0, 3, 2, 1, 4)
        return torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    return qa, qb, sa, sb, atoms(sa), atoms(sb)


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("N", [1024, 256])
def test_mx_gemm_waits_expire_and_context_survives(cuda_lib, mode, N):
    """Both block-scaled kernels (256 x 384 tiles for N >= 512, 256 x 256 below): expired waits,
    then a correct launch."""
    M, K = 1024, 2048
    qa, qb, sa, sb, sa_d, sb_d = _mx_problem(M, N, K, 40 + mode + N)
    D = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    g = [dict(A=torch.from_numpy(qa).cuda(), a_sf=sa_d, a_fmt=oracle.E4M3,
              B=torch.from_numpy(qb).cuda(), b_sf=sb_d, b_fmt=oracle.E4M3, D=D)]
    _run_expired(cuda_lib, mode, lambda: cuda_lib.fp8_mx_gemm_multi(g))
    cuda_lib.fp8_mx_gemm_multi(g)
    cuda_lib.fp8t_check_device_error()
    rng = np.random.default_rng(7)
    ii = rng.integers(0, M, 512); jj = rng.integers(0, N, 512)
    R, ab = oracle.mx_gemm_at(qa, sa, oracle.E4M3, qb, sb, oracle.E4M3, ii, jj)
    assert gemm_within_tolerance(bf16_bits(D)[ii, jj], R, ab).all()


def test_mx_cast_waits_expire_and_context_survives(cuda_lib):
    x = (torch.randn(1024, 2048) * 3).to(torch.bfloat16)
    xd = x.cuda()
    q = torch.empty(1024, 2048, dtype=torch.uint8, device="cuda")
    sf = torch.empty(cuda_lib.mx_scale_bytes(1024, 2048), dtype=torch.uint8, device="cuda")
    cast = lambda: cuda_lib.fp8_mx_cast_multi([dict(x=xd, fmt=oracle.E4M3, q_row=q, sf_row=sf)])
    _run_expired(cuda_lib, 1, cast)
    cast()
    cuda_lib.fp8t_check_device_error()
    rq, _ = oracle.mx_quantise(bf16_bits(x), 0, oracle.E4M3)
    assert np.array_equal(u8(q), rq)


@pytest.mark.parametrize("N", [1024, 256])
def test_expired_mx_gemm_sum_of_squares_is_nan(cuda_lib, N):
    """fp8_mx_gemm_multi_sumsq (both block-scaled kernels) with expired epilogue waits reports a
    NaN sum and leaves its workspace words at zero; the next call gives the exact sum again."""
    M, K = 1024, 1024
    qa, qb, sa, sb, sa_d, sb_d = _mx_problem(M, N, K, 60 + N)
    g = [dict(A=torch.from_numpy(qa).cuda(), a_sf=sa_d, a_fmt=oracle.E4M3,
              B=torch.from_numpy(qb).cuda(), b_sf=sb_d, b_fmt=oracle.E4M3, sumsq=True,
              D=torch.empty(M, N, dtype=torch.bfloat16, device="cuda"))]
    ws = torch.zeros(cuda_lib.fp8_mx_gemm_sumsq_workspace_bytes(g), dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    _run_expired(cuda_lib, 2, lambda: cuda_lib.fp8_mx_gemm_multi_sumsq(g, out, ws))
    assert np.isnan(out.item()) and not ws[:8].any()
    cuda_lib.fp8_mx_gemm_multi_sumsq(g, out, ws)
    cuda_lib.fp8t_check_device_error()
    d = g[0]["D"].float().double()
    assert abs(out.item() - float((d * d).sum())) <= 1e-12 * float((d * d).sum())
