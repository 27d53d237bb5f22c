"""Independent checks used to pin the oracle (and shared comparison helpers).

Nothing here calls the oracle or the CUDA library. The FP8 encoder below is a second,
independent statement of "round to nearest, ties to even, saturate": it searches the sorted list
of representable values instead of manipulating bits, and builds that list from the page's
field widths and biases with exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np

FMT = {"E4M3": 0, "E5M2": 1}
SPEC = {  # [P2 §一]: field widths, bias, largest finite value
    0: dict(ebits=4, mbits=3, bias=7, max=448.0),
    1: dict(ebits=5, mbits=2, bias=15, max=57344.0),
}


def positive_values(fmt):
    """All non-negative finite values with their codes, from exact rationals: subnormals
    m/2^mb * 2^(1-bias), normals (1 + m/2^mb) * 2^(e-bias), up to the page's maximum."""
    s = SPEC[fmt]
    out = []
    for code in range(128):
        e, m = code >> s["mbits"], code & ((1 << s["mbits"]) - 1)
        if e == 0:
            v = Fraction(m, 1 << s["mbits"]) * Fraction(2) ** (1 - s["bias"])
        else:
            v = (1 + Fraction(m, 1 << s["mbits"])) * Fraction(2) ** (e - s["bias"])
        if v <= Fraction(s["max"]):
            out.append((code, v))
    return out


def brute_encode(x, fmt):
    """Nearest representable value by search; ties go to the even code; |x| > max saturates;
    NaN -> 0x7F. x: float32 array. Returns uint8 codes."""
    x = np.asarray(x, np.float32).reshape(-1)
    pv = positive_values(fmt)
    codes = np.array([c for c, _ in pv], np.int64)
    vals = np.array([float(v) for _, v in pv], np.float64)   # exact in float64
    with np.errstate(invalid="ignore"):
        a = np.abs(x.astype(np.float64))
    sign = (x.view(np.uint32) >> 31).astype(np.int64)
    idx = np.searchsorted(vals, a, side="left")            # vals[idx-1] < a <= vals[idx]
    idx_hi = np.clip(idx, 0, len(vals) - 1)
    idx_lo = np.clip(idx - 1, 0, len(vals) - 1)
    d_hi = np.abs(vals[idx_hi] - a)
    d_lo = np.abs(a - vals[idx_lo])
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (codes[idx_lo] % 2 == 0))
    code = np.where(pick_lo, codes[idx_lo], codes[idx_hi])
    code = np.where(a > SPEC[fmt]["max"], codes[-1], code)   # saturation (inf included)
    out = (sign << 7) | code
    out = np.where(np.isnan(x), 0x7F, out)
    return out.astype(np.uint8)


def f32_ordered(x):
    """Map float32 bit patterns to integers whose order is the float order (for ulp distance)."""
    b = np.asarray(x, np.float32).view(np.int32).astype(np.int64)
    return np.where(b < 0, -(b & 0x7FFFFFFF), b)


def ulp_distance_f32(a, b):
    """Number of representable float32 values between a and b (0 = identical)."""
    return np.abs(f32_ordered(a) - f32_ordered(b))


def bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_ulp(v):
    """Spacing of BF16 values at |v| (float64 array): 2^(e-7) for normals, 2^-133 at and below
    the smallest normal (zero included)."""
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(v > 0, v, 2.0 ** -126)))
    e = np.maximum(e, -126)
    return np.where(np.isfinite(v), np.exp2(e - 7), np.inf)


def gemm_within_tolerance(d_gpu_bits, d_ref_bits, abs_sum):
    """|D_gpu - D_ref| <= 2 BF16 ulp of D_ref + 1e-5 * sum_k |a_k b_k| * scale, per element;
    NaN where and only where the reference is NaN. Returns the boolean mask of passing elements."""
    g = bf16_to_f32(d_gpu_bits).astype(np.float64)
    r = bf16_to_f32(d_ref_bits).astype(np.float64)
    tol = 2 * bf16_ulp(r) + 1e-5 * np.asarray(abs_sum, np.float64)
    with np.errstate(invalid="ignore"):
        ok = (np.abs(g - r) <= tol) | (g == r)
    both_nan = np.isnan(g) & np.isnan(r)
    return (ok & ~np.isnan(g) & ~np.isnan(r)) | both_nan


def nearest_f32(fr: Fraction) -> float:
    """Exact rational -> nearest float32 (ties to even), by bracketing with numpy.nextafter."""
    f = np.float32(float(fr))            # within one f32 ulp of the answer
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - fr)
        key = (d, int(np.float32(c).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return float(best[1])
