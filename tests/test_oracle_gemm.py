"""Pins of the oracle's per-tensor scaled FP8 GEMM.

[P2] "FP8 混合精度训练工程实践", §三 (FP8 GEMM with higher-precision accumulation and a 16-bit
output), §四 (dequantize divides by the scale), §五 (per-tensor mode: FP8 x FP8, FP32 accumulate,
BF16 output).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests._pins import bf16_to_f32, bf16_ulp, nearest_f32

PAIRS = [(oracle.E4M3, oracle.E4M3), (oracle.E5M2, oracle.E4M3), (oracle.E4M3, oracle.E5M2),
         (oracle.E5M2, oracle.E5M2)]


def _finite_codes(rng, fmt, shape):
    t = oracle.decode_table(fmt)
    ok = np.flatnonzero(np.isfinite(t)).astype(np.uint8)
    return rng.choice(ok, size=shape)


def _lib_decode(codes, fmt):
    dt = torch.float8_e4m3fn if fmt == oracle.E4M3 else torch.float8_e5m2
    return [Fraction(float(v)) for v in torch.from_numpy(codes.reshape(-1)).view(dt).double()]


def _bf16_rne_of_rational(fr: Fraction) -> float:
    """Exact rational -> nearest f32 -> BF16 round-to-nearest-even (torch as the library)."""
    f = nearest_f32(fr)
    return float(torch.tensor([f], dtype=torch.float32).to(torch.bfloat16).float()[0])


@pytest.mark.parametrize("afmt,bfmt", PAIRS)
def test_brute_force_exact_rationals(afmt, bfmt):
    """Tiny shapes: the exact rational sum of products (operands decoded by torch's float8
    dtypes), times the f32 product of the scale inverses, rounded once to f32 then BF16."""
    rng = np.random.default_rng(afmt * 2 + bfmt)
    M, N, K = 5, 7, 48
    A = _finite_codes(rng, afmt, (M, K))
    B = _finite_codes(rng, bfmt, (N, K))
    sa, sb = np.float32(0.37), np.float32(1.0 / 3.0)
    D, ab = oracle.gemm(A, afmt, B, bfmt, sa, sb, want_abs=True)
    Ad = np.array(_lib_decode(A, afmt), dtype=object).reshape(M, K)
    Bd = np.array(_lib_decode(B, bfmt), dtype=object).reshape(N, K)
    alpha = Fraction(float(sa * sb))
    exact_hits = 0
    for i in range(M):
        for j in range(N):
            s = sum(Ad[i, k] * Bd[j, k] for k in range(K)) * alpha
            want = _bf16_rne_of_rational(s)
            got = float(bf16_to_f32(D[i, j]))
            # the oracle rounds acc -> double -> float -> bf16; allow one bf16 step for that
            assert abs(got - want) <= bf16_ulp(want), (i, j, got, want)
            exact_hits += got == want
            sabs = sum(abs(Ad[i, k] * Bd[j, k]) for k in range(K)) * alpha
            assert abs(ab[i, j] - float(sabs)) <= 1e-12 * float(sabs)
    assert exact_hits >= M * N - 1


def test_closed_form_all_ones():
    """A, B all 1.0 (E4M3 code 0x38): D = bf16(K * sa * sb)."""
    for K in (16, 48, 4096):
        A = np.full((3, K), 0x38, np.uint8)
        B = np.full((4, K), 0x38, np.uint8)
        sa, sb = np.float32(0.5), np.float32(0.25)
        D = oracle.gemm(A, oracle.E4M3, B, oracle.E4M3, sa, sb)
        want = torch.tensor([K * 0.125], dtype=torch.float32).to(torch.bfloat16).float().item()
        assert np.all(bf16_to_f32(D) == want)


def test_closed_form_permutation_gathers_rows():
    """A = permutation matrix (1.0 at A[i, p[i]]): D[i, j] = bf16(B[j, p[i]] * sa * sb)."""
    rng = np.random.default_rng(3)
    K = 64
    p = rng.permutation(K)[:32]
    A = np.zeros((32, K), np.uint8)
    A[np.arange(32), p] = 0x38
    B = _finite_codes(rng, oracle.E5M2, (16, K))
    sa, sb = np.float32(1.0), np.float32(2.0 ** -4)
    D = oracle.gemm(A, oracle.E4M3, B, oracle.E5M2, sa, sb)
    bval = torch.from_numpy(B).view(torch.float8_e5m2).float() * float(sa * sb)
    want = bval[:, p].T.to(torch.bfloat16).float().numpy()
    assert np.array_equal(bf16_to_f32(D), want)


def test_transposition_and_operand_order_matter():
    """D = A.B^T, not A^T.B or B.A^T: a non-symmetric case distinguishes them."""
    A = np.zeros((16, 16), np.uint8); B = np.zeros((16, 16), np.uint8)
    A[0, 1] = 0x38        # a[0][1] = 1
    B[2, 1] = 0x40        # b[2][1] = 2
    D = bf16_to_f32(oracle.gemm(A, oracle.E4M3, B, oracle.E4M3, 1.0, 1.0))
    assert D[0, 2] == 2.0 and np.count_nonzero(D) == 1


def test_nonfinite_operand_gives_nan():
    A = np.full((16, 16), 0x38, np.uint8); B = np.full((16, 16), 0x38, np.uint8)
    A[3, 7] = 0x7F        # NaN
    D = bf16_to_f32(oracle.gemm(A, oracle.E4M3, B, oracle.E4M3, 1.0, 1.0))
    assert np.all(np.isnan(D[3])) and np.all(np.isfinite(np.delete(D, 3, axis=0)))


def test_gemm_at_matches_full():
    rng = np.random.default_rng(9)
    A = _finite_codes(rng, oracle.E4M3, (32, 96)); B = _finite_codes(rng, oracle.E5M2, (48, 96))
    D, ab = oracle.gemm(A, oracle.E4M3, B, oracle.E5M2, 0.01, 3.0, want_abs=True)
    ii = rng.integers(0, 32, 200); jj = rng.integers(0, 48, 200)
    d2, ab2 = oracle.gemm_at(A, oracle.E4M3, B, oracle.E5M2, 0.01, 3.0, ii, jj)
    assert np.array_equal(d2, D[ii, jj]) and np.array_equal(ab2, ab[ii, jj])


def test_large_k_exact_accumulation():
    """K = 16384 of +-max products that cancel except for one small term: an f32 accumulator
    would lose the small term, the exact accumulator keeps it."""
    K = 16384
    A = np.full((1, K), 0x7E, np.uint8)               # 448
    B = np.full((1, K), 0x7B, np.uint8)               # 57344
    B[0, K // 2:] = 0xFB                              # -57344: pairs cancel exactly
    A[0, 0] = 0x01                                    # 2^-9 instead of 448 at k = 0
    D = oracle.gemm(A, oracle.E4M3, B, oracle.E5M2, 1.0, 1.0)
    want = 2.0 ** -9 * 57344 - 448 * 57344            # k = 0 term replaces one positive 448 term
    assert bf16_to_f32(D)[0, 0] == torch.tensor([want]).to(torch.bfloat16).float().item()
