"""Pins of the MXFP8 oracle ("FP8 混合精度训练工程实践" §九: 32 values share one E8M0 scale,
each stored as FP8; §三: micro scaling with E4M3 elements), independent of its own code:

* E8M0 decodes as 2^(code - 127) with 0xFF = NaN (the format's definition), checked on all codes;
* the shared exponent is the published MX rule X = floor(log2 amax) - emax (emax 8 for E4M3,
  15 for E5M2: 448 = 1.75 * 2^8, 57344 = 1.75 * 2^15, page values): for every block amax / 2^X
  lies in [2^emax, 2^(emax+1)), checked by brute force on random blocks and on every power of two;
* with every scale at 2^0 the MX quantisation reduces to the per-tensor cast at scale 1 and the MX
  GEMM to the per-tensor GEMM at unit scales (special cases, both pinned elsewhere);
* exact rational sums (fractions) on small GEMMs with mixed block scales;
* all-ones and power-of-two closed forms."""
from fractions import Fraction

import numpy as np
import torch

import oracle
from optimizer_fp8_cast_b200.synth import bf16_bits

EMAX = {oracle.E4M3: 8, oracle.E5M2: 15}


def test_e8m0_decode_every_code():
    for c in range(255):
        assert oracle.e8m0_decode(c) == 2.0 ** (c - 127)
    assert np.isnan(oracle.e8m0_decode(255))


def test_shared_exponent_rule_by_brute_force():
    rng = np.random.default_rng(5)
    for fmt in (oracle.E4M3, oracle.E5M2):
        x = (rng.standard_normal((64, 256)) * 10.0 ** rng.uniform(-20, 20, (64, 1))).astype(np.float32)
        bits = bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
        vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        for axis in (0, 1):
            q, sf = oracle.mx_quantise(bits, axis, fmt)
            blocks = vals.reshape(64, 8, 32) if axis == 0 else vals.T.reshape(256, 2, 32)
            scales = sf if axis == 0 else sf.T
            for idx in np.ndindex(blocks.shape[:2]):
                amax = np.abs(blocks[idx]).max()
                X = int(scales[idx]) - 127
                assert 2.0 ** EMAX[fmt] <= amax / 2.0 ** X < 2.0 ** (EMAX[fmt] + 1)
            # decode(q) * 2^X is the element rounded to the format (within half a step of x)
            dec = np.vectorize(lambda c: oracle.fp8_decode(int(c), fmt))(q).astype(np.float64)
            rep = np.repeat(sf.astype(np.int64) - 127, 32, axis=1) if axis == 0 else \
                np.repeat(sf.astype(np.int64) - 127, 32, axis=0)
            back = dec * np.exp2(rep)
            top = 448.0 if fmt == oracle.E4M3 else 57344.0
            rel_step = 2.0 ** -(3 if fmt == oracle.E4M3 else 2)
            unsat = np.abs(vals) <= top * np.exp2(rep)
            err = np.abs(back - vals)[unsat]
            assert (err <= np.abs(vals)[unsat] * rel_step / 2 + np.exp2(rep)[unsat] * 2.0 ** -10).all()


def test_powers_of_two_and_zero_blocks():
    for fmt in (oracle.E4M3, oracle.E5M2):
        for k in range(-100, 101, 7):
            x = np.full((1, 32), 2.0 ** k, np.float32)
            q, sf = oracle.mx_quantise(bf16_bits(torch.from_numpy(x).to(torch.bfloat16)), 0, fmt)
            assert sf[0, 0] == k - EMAX[fmt] + 127
            # 2^emax is exponent field emax + bias, mantissa 0
            assert q[0, 0] == ((EMAX[fmt] + (7 if fmt == oracle.E4M3 else 15)) << (3 if fmt == oracle.E4M3 else 2))
        q, sf = oracle.mx_quantise(np.zeros((32, 32), np.uint16), 1, fmt)
        assert (sf == 0).all() and not q.any()


def test_unit_scales_reduce_to_the_per_tensor_cast_and_gemm():
    rng = np.random.default_rng(6)
    # blocks whose amax lies in [2^8, 2^9): the shared exponent is 0 for E4M3
    x = rng.uniform(-300, 300, (32, 64)).astype(np.float32)
    x[:, ::32] = 300.0
    bits = bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    q, sf = oracle.mx_quantise(bits, 0, oracle.E4M3)
    assert (sf == 127).all()
    rq, _, _, _, _ = oracle.cast_transpose_amax(bits, oracle.E4M3, 1.0)
    assert np.array_equal(q, rq)
    B = rng.integers(0, 0x7E, (48, 64)).astype(np.uint8)
    D = oracle.mx_gemm(q, sf, oracle.E4M3, B, np.full((48, 2), 127, np.uint8), oracle.E4M3)
    assert np.array_equal(D, oracle.gemm(q, oracle.E4M3, B, oracle.E4M3, 1.0, 1.0))


def test_exact_rational_sums_with_block_scales():
    rng = np.random.default_rng(7)
    M, N, K = 3, 4, 96
    A = rng.integers(0, 0x7E, (M, K)).astype(np.uint8) | (rng.integers(0, 2, (M, K)) << 7).astype(np.uint8)
    B = rng.integers(0, 0x7B, (N, K)).astype(np.uint8)
    sfa = rng.integers(100, 150, (M, K // 32)).astype(np.uint8)
    sfb = rng.integers(110, 140, (N, K // 32)).astype(np.uint8)
    D = oracle.mx_gemm(A, sfa, oracle.E4M3, B, sfb, oracle.E5M2)
    for i in range(M):
        for j in range(N):
            s = sum(Fraction(oracle.fp8_decode(int(A[i, k]), oracle.E4M3)) *
                    Fraction(oracle.fp8_decode(int(B[j, k]), oracle.E5M2)) *
                    Fraction(2) ** (int(sfa[i, k // 32]) + int(sfb[j, k // 32]) - 254)
                    for k in range(K))
            ref = oracle.f32_to_bf16(np.float32(float(s)))
            assert abs(int(D[i, j]) - int(ref)) <= 1 or D[i, j] == ref


def test_all_ones_closed_form():
    one = 0x38                                        # 1.0 in E4M3: exponent 7 (bias 7), mantissa 0
    A = np.full((2, 128), one, np.uint8)
    B = np.full((3, 128), one, np.uint8)
    sfa = np.array([[127, 128, 126, 127]] * 2, np.uint8)
    sfb = np.array([[130, 127, 127, 125]] * 3, np.uint8)
    D = oracle.mx_gemm(A, sfa, oracle.E4M3, B, sfb, oracle.E4M3)
    want = 32 * (2.0 ** 3 + 2.0 ** 1 + 2.0 ** -1 + 2.0 ** -2)
    assert (D == oracle.f32_to_bf16(np.float32(want))).all()


def test_subnormal_blocks_clamp_the_exponent():
    """A block whose amax is a BF16 subnormal: floor(log2) is taken from the mantissa's top bit
    (2^-130 = 8 * 2^-133), X = -130 - 8 clamps to -127 (scale code 0), and the elements come out
    as 2^-130 * 2^127 = 2^-3, the E4M3 code 0x20 (exponent field 4, bias 7)."""
    v = np.uint16(8)                                   # BF16 bits of 2^-130 (subnormal)
    bits = np.full((1, 32), v, np.uint16)
    q, sf = oracle.mx_quantise(bits, 0, oracle.E4M3)
    assert sf[0, 0] == 0 and (q == 0x20).all()
    bits[0, 0] = 0x0001                                # 2^-133, the smallest subnormal
    q, sf = oracle.mx_quantise(bits, 0, oracle.E5M2)   # X = -130 - 15 clamps to -127 as well
    assert sf[0, 0] == 0
    assert oracle.fp8_decode(int(q[0, 0]), oracle.E5M2) == 2.0 ** -6   # 2^-133 * 2^127


def _exact_mx(A, sfa, afmt, B, sfb, bfmt, i, j):
    """sum_k a_ik b_jk 2^(Xa + Xb) as an exact rational, operands decoded from the code tables."""
    K = A.shape[1]
    return sum(Fraction(oracle.fp8_decode(int(A[i, k]), afmt)) *
               Fraction(oracle.fp8_decode(int(B[j, k]), bfmt)) *
               Fraction(2) ** (int(sfa[i, k // 32]) + int(sfb[j, k // 32]) - 254)
               for k in range(K))


def test_mx_gemm_at_matches_full_gemm_and_exact_sums():
    """The sampled MX GEMM (the oracle behind the full-size MX GEMM checks) against the full one
    at random positions, with M != N, a distinct scale row for every row of A and of B and mixed
    E4M3 x E5M2 operands, so that swapping the row and column indices, or taking one operand's
    scale row for the other's, gives different values; a few positions also against the exact
    rational sum."""
    rng = np.random.default_rng(8)
    M, N, K = 37, 53, 160
    ta, tb = oracle.decode_table(oracle.E4M3), oracle.decode_table(oracle.E5M2)
    A = rng.choice(np.flatnonzero(np.isfinite(ta)).astype(np.uint8), (M, K))
    B = rng.choice(np.flatnonzero(np.isfinite(tb)).astype(np.uint8), (N, K))
    sfa = rng.integers(110, 145, (M, K // 32)).astype(np.uint8)
    sfb = rng.integers(115, 140, (N, K // 32)).astype(np.uint8)
    D, ab = oracle.mx_gemm(A, sfa, oracle.E4M3, B, sfb, oracle.E5M2, want_abs=True)
    ii = rng.integers(0, M, 400)
    jj = rng.integers(0, N, 400)
    got, gab = oracle.mx_gemm_at(A, sfa, oracle.E4M3, B, sfb, oracle.E5M2, ii, jj)
    assert np.array_equal(got, D[ii, jj]) and np.array_equal(gab, ab[ii, jj])
    # the sampled values are not those of transposed indices or of swapped scale rows
    Dsw = oracle.mx_gemm(A, np.roll(sfa, 1, axis=0), oracle.E4M3, B, sfb, oracle.E5M2)
    assert (Dsw[ii, jj] != got).mean() > 0.5
    for s in range(12):
        ref = oracle.f32_to_bf16(np.float32(float(_exact_mx(A, sfa, oracle.E4M3, B, sfb,
                                                            oracle.E5M2, ii[s], jj[s]))))
        assert abs(int(got[s]) - int(ref)) <= 1


def test_nan_block_keeps_unit_scale_and_nan_code():
    """A block holding a NaN has no finite amax: its E8M0 scale is the NaN code 0xFF (the only
    non-numeric E8M0 code), and its other elements are encoded at unit scale, X = 0. Hand-worked
    values: 1.0 -> 0x38 and -2.0 -> 0xC0 in E4M3 (bias 7), 1.0 -> 0x3C and 3.0 -> 0x42 in E5M2
    (bias 15), 1000.0 saturates to 448 (0x7E) in E4M3; the NaN itself is the byte 0x7F."""
    nan = np.uint16(0x7FC1)                                  # a NaN with a payload
    for fmt, vals, codes in ((oracle.E4M3, [1.0, -2.0, 1000.0], [0x38, 0xC0, 0x7E]),
                             (oracle.E5M2, [1.0, 3.0, -0.0], [0x3C, 0x42, 0x80])):
        x = np.zeros((1, 32), np.float32)
        x[0, 1:4] = vals
        bits = bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
        bits[0, 17] = nan
        q, sf = oracle.mx_quantise(bits, 0, fmt)
        assert sf[0, 0] == 0xFF
        assert list(q[0, 1:4]) == codes and q[0, 17] == 0x7F
        assert q[0, 0] == 0x00 and (q[0, 4:17] == 0).all() and (q[0, 18:] == 0).all()
        # column-wise blocks follow the same rule: only the column holding the NaN
        cols = np.zeros((32, 4), np.uint16)
        cols[:, 2] = bits[0]
        cols[:, 0] = bits[0, 1]                               # a column of 1.0 / 1.0
        qc, sfc = oracle.mx_quantise(cols, 1, fmt)
        assert sfc[0, 2] == 0xFF and list(qc[1:4, 2]) == codes and qc[17, 2] == 0x7F
        assert sfc[0, 0] == 127 - (8 if fmt == oracle.E4M3 else 15) and sfc[0, 1] == 0


def test_infinite_amax_takes_the_largest_exponent():
    """A block whose amax is +-inf: X = 127, the largest finite E8M0 exponent (code 254). The
    infinity then saturates to the format's largest code (0x7E = 448 in E4M3, 0x7B = 57344 in
    E5M2; sign kept), and finite elements times 2^-127 fall below the smallest subnormal and
    encode as signed zeros."""
    for fmt, top in ((oracle.E4M3, 0x7E), (oracle.E5M2, 0x7B)):
        x = np.full((2, 32), 3.5, np.float32)
        x[0, 5] = np.inf
        x[1, 9] = -np.inf
        x[1, 0] = -1.0e30
        bits = bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
        q, sf = oracle.mx_quantise(bits, 0, fmt)
        assert (sf[:, 0] == 254).all()
        assert q[0, 5] == top and q[1, 9] == 0x80 | top
        assert (np.delete(q[0], 5) == 0x00).all()
        # -1e30 * 2^-127 ~ -5.9e-9: far below the smallest subnormal, a negative zero
        assert q[1, 0] == 0x80 and (np.delete(q[1], [0, 9]) == 0x00).all()
