"""Pins of the oracle's cast / transpose / amax and counters.

[P2] "FP8 混合精度训练工程实践", §四 (FP8Tensor.quantize: amax = max(abs(x)); x * scale, clamp,
store as FP8); [P3] "LLM FP8 微调上线生产实战", 工程落地 第四步 (saturation and zero fractions).
"""
import numpy as np
import pytest

import oracle
from tests._pins import SPEC, bf16_to_f32, brute_encode

ALL_BF16 = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
SCALES = [1.0, 2.0 ** -3, 3.7, 1.0 / 3.0, 16384.0, 2.0 ** 100, 2.0 ** -100]


def _independent_cast(x_bits, fmt, scale):
    xf = bf16_to_f32(x_bits)
    s = np.float32(scale)
    with np.errstate(over="ignore", invalid="ignore"):
        prod = (xf * s).astype(np.float32)          # one IEEE f32 multiply
    q = brute_encode(prod, fmt).reshape(x_bits.shape)
    with np.errstate(invalid="ignore"):
        sat = int(np.sum(np.abs(prod) > SPEC[fmt]["max"]))
    zero = int(np.sum((q & 0x7F) == 0))
    nonfin = int(np.sum(~np.isfinite(xf)))
    with np.errstate(invalid="ignore"):
        amax = np.float32(np.max(np.abs(xf)))       # numpy's max propagates NaN
    return q, amax, sat, zero, nonfin


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("scale", SCALES)
def test_cast_every_bf16_pattern(fmt, scale):
    """All 65,536 BF16 inputs: codes, transpose, counters and scale_inv against independent
    numpy arithmetic plus the brute-force encoder."""
    q, qT, amax, sinv, cnt = oracle.cast_transpose_amax(ALL_BF16, fmt, scale)
    q2, amax2, sat, zero, nonfin = _independent_cast(ALL_BF16, fmt, scale)
    assert np.array_equal(q, q2)
    assert np.array_equal(qT, q.T)
    assert np.isnan(amax) and np.isnan(amax2)       # the table contains NaN patterns
    assert list(cnt) == [sat, zero, nonfin]
    assert sinv == np.float32(1.0) / np.float32(scale)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_amax_brute_force(fmt):
    rng = np.random.default_rng(11)
    for shape in [(16, 16), (48, 80), (128, 32)]:
        x = rng.standard_normal(shape).astype(np.float32) * rng.uniform(1e-3, 1e3)
        bits = (x.view(np.uint32) >> 16).astype(np.uint16)   # any BF16 patterns will do
        _, _, amax, _, _ = oracle.cast_transpose_amax(bits, fmt, 1.0)
        assert amax == np.max(np.abs(bf16_to_f32(bits)))


def test_amax_special_cases():
    E = oracle.E4M3
    z = np.zeros((16, 16), np.uint16)
    assert oracle.cast_transpose_amax(z, E, 1.0)[2] == 0.0
    negz = np.full((16, 16), 0x8000, np.uint16)                 # -0 counts as 0
    a = oracle.cast_transpose_amax(negz, E, 1.0)[2]
    assert a == 0.0 and not np.signbit(a)
    x = z.copy(); x[3, 5] = 0xFF80                               # -inf
    assert oracle.cast_transpose_amax(x, E, 1.0)[2] == np.inf
    x[7, 1] = 0x7FC1                                              # a NaN with payload
    a = oracle.cast_transpose_amax(x, E, 1.0)[2]
    assert np.isnan(a) and np.float32(a).view(np.uint32) == 0x7FC00000   # canonical NaN
    x = z.copy(); x[0, 0] = 0x0001; x[1, 1] = 0x8003             # BF16 subnormals
    assert oracle.cast_transpose_amax(x, E, 1.0)[2] == bf16_to_f32(np.uint16(0x0003))


def test_amax_slot_is_max_accumulated():
    x = np.full((16, 16), 0x4000, np.uint16)                      # all 2.0
    E = oracle.E4M3
    assert oracle.cast_transpose_amax(x, E, 1.0, amax_in=0.0)[2] == 2.0
    assert oracle.cast_transpose_amax(x, E, 1.0, amax_in=5.0)[2] == 5.0
    assert oracle.cast_transpose_amax(x, E, 1.0, amax_in=1.5)[2] == 2.0
    assert np.isnan(oracle.cast_transpose_amax(x, E, 1.0, amax_in=float("nan"))[2])
    assert oracle.cast_transpose_amax(x, E, 1.0, amax_in=float("inf"))[2] == np.inf


def test_counters_accumulate_and_hand_case():
    """Counters add to what the caller passes in; a hand-made 16x16 case."""
    x = np.zeros((16, 16), np.uint16)
    x[0, 0] = 0x43E0      # 448.0 exactly: not saturated (strictly greater than max counts)
    x[0, 1] = 0x43E1      # 450.0: saturated
    x[0, 2] = 0x7F80      # inf: saturated and non-finite
    x[0, 3] = 0x7FC0      # NaN: non-finite only, code 0x7F
    x[0, 4] = 0x3F80      # 1.0
    q, qT, amax, sinv, cnt = oracle.cast_transpose_amax(x, oracle.E4M3, 1.0)
    assert list(q[0, :5]) == [0x7E, 0x7E, 0x7E, 0x7F, 0x38]
    assert list(cnt) == [2, 256 - 5, 2]
