"""Pins of the oracle's FP8 / BF16 codec against the pages and independent definitions.

[P2] "FP8 混合精度训练工程实践：从 H100 到大模型训练的范式跃迁", §一 FP8 格式设计.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from tests._pins import SPEC, brute_encode, positive_values

GOLD = os.path.join(os.path.dirname(__file__), "golden")
FMTS = [oracle.E4M3, oracle.E5M2]


def test_page_constants():
    """Bias, range and the E4M3 step near 1 printed on the page."""
    c = json.load(open(os.path.join(GOLD, "page_constants.json")))
    for name, fmt in (("E4M3", oracle.E4M3), ("E5M2", oracle.E5M2)):
        t = oracle.decode_table(fmt)
        fin = t[np.isfinite(t)]
        assert fin.max() == c[name]["max"] and fin.min() == -c[name]["max"]
        # exponent field == bias with mantissa 0 is exactly 1.0
        one = c[name]["bias"] << c[name]["mantissa_bits"]
        assert t[one] == 1.0
        assert c[name]["exponent_bits"] + c[name]["mantissa_bits"] + 1 == 8
    t = oracle.decode_table(oracle.E4M3)
    assert t[0x39] - t[0x38] == c["E4M3_step_near_1"]
    assert oracle.FP8_MAX[oracle.E4M3] == 448.0 and oracle.FP8_MAX[oracle.E5M2] == 57344.0


@pytest.mark.parametrize("fmt", FMTS)
def test_decode_table_matches_field_definition(fmt):
    """Every positive code decodes to the exact rational its fields give; negatives mirror."""
    t = oracle.decode_table(fmt)
    pv = dict(positive_values(fmt))
    for code in range(128):
        if code in pv:
            assert t[code] == float(pv[code])
            assert t[code | 0x80] == -float(pv[code]) or (code == 0 and t[0x80] == 0.0)
        else:
            assert not np.isfinite(t[code])
    # special codes: E4M3 has NaN only at S.1111.111; E5M2 has inf at S.11111.00, NaN above
    if fmt == oracle.E4M3:
        assert np.isnan(t[0x7F]) and np.isnan(t[0xFF]) and np.isfinite(t).sum() == 254
    else:
        assert t[0x7C] == np.inf and t[0xFC] == -np.inf
        assert all(np.isnan(t[c]) for c in (0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF))
        assert np.isfinite(t).sum() == 248
    # closed forms: smallest subnormal and normal
    s = SPEC[fmt]
    assert t[0x01] == 2.0 ** (1 - s["bias"] - s["mbits"])
    assert t[1 << s["mbits"]] == 2.0 ** (1 - s["bias"])
    # strictly increasing over the positive finite codes
    fin = [t[c] for c in range(128) if np.isfinite(t[c])]
    assert all(a < b for a, b in zip(fin, fin[1:]))


@pytest.mark.parametrize("fmt", FMTS)
def test_decode_matches_torch_float8(fmt):
    """Library special case: torch's float8 dtypes use the same layouts for finite values."""
    dt = torch.float8_e4m3fn if fmt == oracle.E4M3 else torch.float8_e5m2
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(dt).to(torch.float64).numpy()
    t = oracle.decode_table(fmt)
    fin = np.isfinite(t)
    assert np.array_equal(lib[fin], t[fin])
    assert np.array_equal(np.isnan(lib), np.isnan(t))


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_decode_identity(fmt):
    t = oracle.decode_table(fmt)
    for code in range(256):
        if np.isfinite(t[code]):
            assert oracle.fp8_encode(np.float32(t[code]), fmt) == code


def _structured_f32():
    """Every f32 exponent from 2^-30 to 2^17 with all 2^11 leading mantissa patterns and the
    trailing 12 bits set to the rounding-relevant patterns, both signs; plus specials."""
    exps = np.arange(127 - 30, 127 + 18, dtype=np.uint32)
    top = np.arange(1 << 11, dtype=np.uint32) << 12
    low = np.array([0, 1, 0x7FF, 0x800, 0x801, 0xFFF], np.uint32)
    bits = (exps[:, None, None] << 23) | top[None, :, None] | low[None, None, :]
    bits = bits.reshape(-1)
    sub = np.array([0, 1, 0x400000, 0x7FFFFF, 0x800000], np.uint32)
    specials = np.array([0x7F800000, 0x7FC00000, 0x7F800001], np.uint32)
    bits = np.concatenate([bits, sub, specials])
    bits = np.concatenate([bits, bits | 0x80000000])
    return bits.view(np.float32)


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_matches_brute_force(fmt):
    """The bit-manipulation encoder agrees with nearest-value search on every rounding case and
    on two million random f32 bit patterns."""
    xs = _structured_f32()
    assert np.array_equal(oracle.encode_array(xs, fmt), brute_encode(xs, fmt))
    rng = np.random.default_rng(1234 + fmt)
    r = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    assert np.array_equal(oracle.encode_array(r, fmt), brute_encode(r, fmt))


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_matches_torch_within_range(fmt):
    """Library special case: torch's round-to-nearest-even cast agrees for |x| <= max (torch does
    not saturate, so values beyond max are not compared)."""
    xs = _structured_f32()
    keep = np.isfinite(xs) & (np.abs(xs) <= SPEC[fmt]["max"])
    xs = xs[keep]
    dt = torch.float8_e4m3fn if fmt == oracle.E4M3 else torch.float8_e5m2
    lib = torch.from_numpy(xs).to(dt).view(torch.uint8).numpy()
    assert np.array_equal(oracle.encode_array(xs, fmt), lib)


def test_saturation_and_nan():
    for fmt, maxc in ((oracle.E4M3, 0x7E), (oracle.E5M2, 0x7B)):
        m = SPEC[fmt]["max"]
        assert oracle.fp8_encode(m * 1.01, fmt) == maxc
        assert oracle.fp8_encode(-m * 1.01, fmt) == 0x80 | maxc
        assert oracle.fp8_encode(float("inf"), fmt) == maxc
        assert oracle.fp8_encode(float("-inf"), fmt) == 0x80 | maxc
        assert oracle.fp8_encode(float("nan"), fmt) == 0x7F
        assert oracle.fp8_encode(-1e-30, fmt) == 0x80   # sign of an underflowed value is kept


def test_bf16_conversions_match_torch():
    """BF16 widening is exact; narrowing is round-to-nearest-even (torch as the library case)."""
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    lib = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([oracle.f32_to_bf16(v) for v in f[:20000]], np.uint16)
    assert np.array_equal(ours, lib[:20000])
    for h in (0x0000, 0x8000, 0x3F80, 0x7F7F, 0x0001, 0xFF80):
        assert oracle.bf16_to_f32(h) == np.uint32(h << 16).view(np.float32)
    assert oracle.f32_to_bf16(float("nan")) == 0x7FC0
