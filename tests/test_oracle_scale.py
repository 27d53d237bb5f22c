"""Pins of the oracle's amax-history roll and scale update.

[P3] "LLM FP8 微调上线生产实战", 核心原理: scale = (FP8_MAX / amax) / 2^margin; Delayed Scaling
records amax into a history window, takes its max or most recent entry, and the scale is used by
the next iteration.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._pins import nearest_f32

GOLD = os.path.join(os.path.dirname(__file__), "golden")
FLT_MAX = float(np.finfo(np.float32).max)


def _one(amax, fmt, margin, prev, algo=oracle.AMAX_MAX, H=1):
    hist = np.zeros((1, H), np.float32)
    scale = np.array([prev], np.float32)
    sinv = np.zeros(1, np.float32)
    oracle.scale_update(np.array([amax], np.float32), hist, [oracle.FP8_MAX[fmt]], algo, margin,
                        scale, sinv)
    return scale[0], sinv[0], hist


def test_hand_worked_cases():
    cases = json.load(open(os.path.join(GOLD, "scale_cases.json")))["cases"]
    for c in cases:
        fmt = oracle.E4M3 if c["fmt"] == "E4M3" else oracle.E5M2
        amax = float(c["amax"]) if not isinstance(c["amax"], str) else float(c["amax"])
        s, sinv, _ = _one(amax, fmt, c["margin"], c["prev"])
        if c["expected"] is None:
            a32 = Fraction(float(np.float32(amax)))
            q = nearest_f32(Fraction(oracle.FP8_MAX[fmt]) / a32)      # IEEE quotient
            exp = float(np.float32(q) * np.float32(2.0 ** -c["margin"]))
        elif c["expected"] == "flt_max":
            exp = FLT_MAX
        else:
            exp = c["expected"]
        assert s == np.float32(exp), c["why"]
        assert sinv == np.float32(nearest_f32(1 / Fraction(float(s)))), c["why"]


def test_history_sequence_h4():
    g = json.load(open(os.path.join(GOLD, "history_h4.json")))
    H = g["H"]
    for algo, key in ((oracle.AMAX_MAX, "rep_max"), (oracle.AMAX_MOST_RECENT, "rep_most_recent")):
        hist = np.zeros((1, H), np.float32)
        scale = np.ones(1, np.float32)
        sinv = np.ones(1, np.float32)
        for t, a in enumerate(g["amax_sequence"]):
            oracle.scale_update(np.array([a], np.float32), hist, [448.0], algo, 0, scale, sinv)
            assert hist[0].tolist() == g["history_after"][t]
            assert scale[0] == np.float32(nearest_f32(Fraction(448) / Fraction(g[key][t])))


def test_consumed_amax_is_reset():
    amax = np.array([3.0, np.nan, 0.5], np.float32)
    hist = np.zeros((3, 4), np.float32)
    s = np.ones(3, np.float32); si = np.ones(3, np.float32)
    oracle.scale_update(amax, hist, [448.0] * 3, oracle.AMAX_MAX, 0, s, si)
    assert np.all(amax == 0) and hist[0, 0] == 3.0 and np.isnan(hist[1, 0])


def test_h1_max_equals_most_recent():
    rng = np.random.default_rng(5)
    seq = rng.uniform(0, 10, 20).astype(np.float32)
    out = []
    for algo in (oracle.AMAX_MAX, oracle.AMAX_MOST_RECENT):
        hist = np.zeros((1, 1), np.float32); s = np.ones(1, np.float32); si = np.ones(1, np.float32)
        trace = []
        for a in seq:
            oracle.scale_update(np.array([a], np.float32), hist, [448.0], algo, 0, s, si)
            trace.append(float(s[0]))
        out.append(trace)
    assert out[0] == out[1]


def test_window_drops_oldest_and_nan_propagates():
    H = 3
    hist = np.zeros((2, H), np.float32)
    s = np.ones(2, np.float32); si = np.ones(2, np.float32)
    fm = [448.0, 57344.0]
    for a in ([100.0, 1.0], [1.0, np.nan], [1.0, 1.0], [1.0, 1.0]):
        oracle.scale_update(np.array(a, np.float32), hist, fm, oracle.AMAX_MAX, 0, s, si)
    # tensor 0: window after four pushes is [1, 1, 1]: the 100 fell out after H pushes
    assert s[0] == np.float32(448.0)
    # tensor 1: NaN still in the window -> scale kept from before the NaN arrived (57344/1)
    assert s[1] == np.float32(57344.0)
    oracle.scale_update(np.array([1.0, 2.0], np.float32), hist, fm, oracle.AMAX_MAX, 0, s, si)
    assert s[1] == np.float32(57344.0 / 2.0)   # NaN has left the window


@pytest.mark.parametrize("margin", [0, 1, 5, 126])
def test_margin_is_power_of_two(margin):
    s0, _, _ = _one(3.0, oracle.E4M3, 0, 1.0)
    s, _, _ = _one(3.0, oracle.E4M3, margin, 1.0)
    assert s == np.float32(Fraction(float(s0)) / 2 ** margin)
