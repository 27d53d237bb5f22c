"""Pins of the current-scaling oracle (cast_current) against values the pages fix.

"LLM FP8 微调上线生产实战" 核心原理: scale = (FP8_MAX / amax) / 2^margin — the hand-worked cases
of tests/golden/scale_cases.json (amax 3.5 -> 128 for E4M3, -> 16384 for E5M2) — applied to the
amax of the tensor being cast ("FP8 混合精度训练工程实践" §四 quantize). The largest element then
lands on the format's largest code (448 = 0x7E for E4M3, 57344 = 0x7B for E5M2, values fixed
in §一)."""
import json
import os

import numpy as np
import torch

import oracle
from optimizer_fp8_cast_b200.synth import bf16_bits

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scale_cases.json")))


def bits_of(values, shape=(16, 16)):
    x = np.zeros(shape, np.float32).reshape(-1)
    x[:len(values)] = values
    return bf16_bits(torch.from_numpy(x.reshape(shape)).to(torch.bfloat16))


def test_scale_and_top_code_from_the_hand_worked_cases():
    for case in GOLD["cases"]:
        if not isinstance(case["amax"], float) or not isinstance(case["expected"], float) or case["amax"] == 0:
            continue
        fmt = oracle.E4M3 if case["fmt"] == "E4M3" else oracle.E5M2
        a = case["amax"]
        if np.float32(a) != np.float32(torch.tensor(a).to(torch.bfloat16).float().item()):
            continue                                   # amax must be a BF16 value to appear in x
        x = bits_of([a, -a / 4, a / 1000, 0.0])
        q, qT, amax, scale, sinv, cnt = oracle.cast_current(x, fmt, case["margin"], 3.0)
        assert amax == np.float32(a)
        assert scale == np.float32(case["expected"]), case["why"]
        top = 0x7E if fmt == oracle.E4M3 else 0x7B
        if case["margin"] == 0:
            assert q[0, 0] == top and cnt[0] == 0     # the amax element hits the largest code
        assert np.array_equal(qT, q.T)


def test_zero_and_nonfinite_tensors():
    q, _, amax, scale, _, _ = oracle.cast_current(bits_of([0.0]), oracle.E4M3, 0, 5.0)
    assert amax == 0.0 and scale == 1.0 and not q.any()
    for bad in (np.nan, np.inf):
        _, _, amax, scale, _, _ = oracle.cast_current(bits_of([1.0, bad]), oracle.E5M2, 0, 5.0)
        assert scale == np.float32(5.0)               # previous scale kept


def test_random_tensor_never_saturates_more_than_its_amax_elements():
    rng = np.random.default_rng(0)
    for fmt in (oracle.E4M3, oracle.E5M2):
        for margin in (0, 1, 2):
            x = bf16_bits(torch.from_numpy((rng.standard_normal((64, 48)) * 37).astype(np.float32)).to(torch.bfloat16))
            q, _, amax, scale, _, cnt = oracle.cast_current(x, fmt, margin, 1.0)
            mag = (x & 0x7FFF).astype(np.uint32)
            n_top = int((mag == (np.float32(amax).view(np.uint32) >> 16)).sum())
            assert cnt[0] <= n_top and (q & 0x7F).max() <= (0x7E if fmt == oracle.E4M3 else 0x7B)
            if margin:
                assert cnt[0] == 0
