"""Host-side logic of the step driver and the benchmark's accounting (no GPU, no kernel runs):
which launches each step configuration makes, and the algorithmic bytes the bench divides by."""
import torch

import bench
from optimizer_fp8_cast_b200 import synth
from optimizer_fp8_cast_b200.step import Fp8LinearStep

HP = dict(lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1024.0,
          max_grad_norm=1.0)


def make(layers=1, **kw):
    shapes = [(256, 128)] * layers
    return Fp8LinearStep(shapes, 128, 16, adamw=HP, w_init=[torch.zeros(256, 128)] * layers,
                         device="cpu", **kw)


def test_launch_counts_per_configuration():
    assert make().kernels_per_step() == 3                                 # all fused
    assert make(counters=True).kernels_per_step() == 3                    # W cast back in the cast launch
    assert make(fused_update=False, fused_norm=False, fused_wcast=False).kernels_per_step() == 5
    assert make(recipe="current").kernels_per_step() == 4                 # amax launch + cast
    assert make(recipe="mxfp8").kernels_per_step() == 3                   # MX cast, GEMM (+ dW^2), AdamW
    assert make(recipe="mxfp8", fused_norm=False).kernels_per_step() == 4  # AdamW with its norm pass
    assert make(layers=3).kernels_per_step() == 4                         # 9 casts: two cast launches
    assert make(layers=9).kernels_per_step() == 4 + 2 + 1                 # 27 casts, 27 GEMMs: 4 + 2 launches


def test_fused_weight_cast_needs_its_preconditions():
    assert make().fused_wcast
    assert not make(counters=True).fused_wcast
    assert not make(transposes=True).fused_wcast
    assert not make(fused_norm=False).fused_wcast
    assert not make(recipe="current").fused_wcast and not make(recipe="current").fused_update
    st = make(transposes=True)
    assert st.layers[0].XqT is not None and make().layers[0].XqT is None


def test_grouped_gemm_descriptors_use_mn_major_operands():
    st = make()
    fprop, dgrad, wgrad = st._gemm_descs(sumsq=True)
    L = st.layers[0]
    assert fprop["A"] is L.Xq and fprop["B"] is L.Wq and fprop["b_mn"] and not fprop.get("a_mn")
    assert dgrad["A"] is L.dYq and dgrad["B"] is L.Wq and not dgrad.get("b_mn")
    assert wgrad["A"] is L.Xq and wgrad["a_mn"] and wgrad["B"] is L.dYq and wgrad["b_mn"]
    assert wgrad.get("sumsq") and not fprop.get("sumsq") and not dgrad.get("sumsq")
    t = make(transposes=True)._gemm_descs()
    assert not any(d.get("a_mn") or d.get("b_mn") for d in t)


def test_bench_workload_numbers():
    n = bench.workload_numbers(synth.LINEAR4096)
    assert n["gemm_flop"] == [2 * 8192 * 4096 * 4096]
    assert 3 * sum(n["gemm_flop"]) == 824633720832                       # 824.6 GFLOP per step
    assert n["cast_bytes"] == 4 * (8192 * 4096 * 2 + 4096 * 4096)         # 4 B/element with q^T
    assert n["params"] == 4096 * 4096 and n["adamw_bytes"] == 30 * 4096 * 4096
    assert n["h2d"] == n["d2h"] == 2 * 2 * 8192 * 4096
    assert bench.throughput(1e12, 10, 2, 1000.0) == 20.0                  # 2 ranks x 10 steps x 1 TFLOP in 1 s
