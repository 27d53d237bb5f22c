"""The benchmark's CPU baseline on CPU: the oracle timed stage by stage on samples (one thread and
several), the host description, and the whole-step time those rates give."""
import os

import numpy as np

import bench
import oracle
from optimizer_fp8_cast_b200 import synth


def _host(wl):
    X, dY = synth.linear_inputs(wl, 0, 0, "cpu")
    W = synth.linear_weight(wl, 0, "cpu")
    h = dict(X=synth.bf16_bits(X), dY=synth.bf16_bits(dY), W=synth.bf16_bits(W))
    for name, fmt in (("X", oracle.E4M3), ("W", oracle.E4M3), ("dY", oracle.E5M2)):
        q, qT, _, _, _ = oracle.cast_transpose_amax(h[name], fmt, 1.0)
        h[name + "q"], h[name + "qT"] = q, qT
    h["master"] = W.float().numpy().reshape(-1)
    h["dW"] = h["W"].reshape(-1).copy()
    return {k: np.ascontiguousarray(v) for k, v in h.items()}


def test_stage_rates_on_one_and_several_threads():
    wl = synth.LINEAR256
    host = _host(wl)
    before = oracle.get_threads()
    try:
        for threads in (1, 2):
            r = bench.oracle_stage_rates(oracle, host, wl, threads, budget_s=0.02)
            assert oracle.get_threads() == threads
            assert r["cast"]["gbs"] > 0 and r["gemm"]["tflops"] > 0 and r["adamw"]["gbs"] > 0
            assert r["scale_update"]["us"] > 0
            assert all(r[k]["sample"] for k in r)
    finally:
        oracle.set_threads(before)
    h = bench.cpu_host()
    assert h["nproc"] == os.cpu_count()


def test_step_value_adds_the_stage_times_of_a_whole_step():
    wl = synth.LINEAR4096
    nums = bench.workload_numbers(wl)
    flop = 3 * sum(nums["gemm_flop"])
    rates = {"cast": {"gbs": 2.0}, "gemm": {"tflops": 0.5}, "scale_update": {"us": 100.0},
             "adamw": {"gbs": 4.0}}
    v, t = bench.oracle_step_value(rates, nums, flop)
    cast_s = 3 * (8192 * 4096 * 2 + 4096 * 4096) / 2e9       # X, W, dY at 3 B per element
    want = cast_s + flop / 0.5e12 + 100e-6 + 30 * 4096 * 4096 / 4e9
    assert abs(t - want) <= 1e-9 * want and abs(v - flop / want / 1e12) <= 1e-9 * v
