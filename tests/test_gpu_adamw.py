"""Parity of fused_adamw_multi_tensor (C ABI, sm_100a) with the oracle: m, v and master within
4 f32 ulp (bit-exact expected), BF16 weight = RNE of the GPU's own master and within one BF16
step of the oracle's, global norm within 2 f32 ulp.

[P1] "算子与编译器：FP8 训练与优化器 Kernel", Fused Optimizer 的意义 / 优化器 kernel 的带宽账;
[P2] "FP8 混合精度训练工程实践" §四 (loss scale, un-scaling, FP32 AdamW)."""
import numpy as np
import pytest
import torch

import oracle
from optimizer_fp8_cast_b200 import synth
from tests._gpu import bf16_bits, f32
from tests._pins import ulp_distance_f32

pytestmark = pytest.mark.gpu

HP = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, loss_scale=1024.0,
          max_grad_norm=1.0)


def make(sizes, seed, device="cuda", grad_std=1e-3):
    cfg = dict(synth.ADAMW4E9, seed=seed, grad_std=grad_std)
    P = [synth.adamw_tensor("master", n, i, cfg, device) for i, n in enumerate(sizes)]
    M = [synth.adamw_tensor("m", n, i, cfg, device) for i, n in enumerate(sizes)]
    V = [synth.adamw_tensor("v", n, i, cfg, device) for i, n in enumerate(sizes)]
    G = [synth.adamw_tensor("grad", n, i, cfg, device) for i, n in enumerate(sizes)]
    W = [torch.zeros(n, dtype=torch.bfloat16, device=device) for n in sizes]
    return P, M, V, G, W


def run_both(fp8, P, M, V, G, W, hp, steps=1):
    host = [[f32(t) for t in P], [f32(t) for t in M], [f32(t) for t in V]]
    for step in range(1, steps + 1):
        hpp = dict(hp, step=step + 999)
        norm = torch.zeros(1, device="cuda"); skipped = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        fp8.fused_adamw_multi_tensor(P, M, V, G, W, grad_norm=norm, skipped=skipped, **hpp)
        fp8.fp8t_check_device_error()
        gbits = [bf16_bits(g) for g in G]
        wref = [np.zeros(g.size, np.uint16) for g in gbits]
        rnorm, rskip = oracle.fused_adamw(host[0], host[1], host[2], gbits, wref, hpp)
        assert skipped.item() == rskip
        n = norm.item()
        assert ulp_distance_f32(np.float32(n), np.float32(rnorm)) <= 2 or (np.isnan(n) and np.isnan(rnorm))
        for i in range(len(P)):
            for got, ref in ((P[i], host[0][i]), (M[i], host[1][i]), (V[i], host[2][i])):
                d = ulp_distance_f32(f32(got), ref)
                assert d.max() <= 4, f"tensor {i}: {d.max()} ulp"
            wg = bf16_bits(W[i])
            assert np.array_equal(wg, bf16_bits(P[i].to(torch.bfloat16)))     # RNE of own master
            diff = np.abs(wg.astype(np.int32) - wref[i].astype(np.int32))
            assert diff.max() <= 1
    return host


def test_single_tensor_linear256(cuda_lib):
    P, M, V, G, W = make([65536], seed=0)
    run_both(cuda_lib, P, M, V, G, W, dict(HP, lr=1e-4, beta2=0.999, weight_decay=0.01), steps=3)


def test_ragged_multi_tensor(cuda_lib):
    sizes = [1, 7, 8, 9, 15, 8191, 8192, 8193, 100003, 262144 + 5]
    P, M, V, G, W = make(sizes, seed=1)
    run_both(cuda_lib, P, M, V, G, W, HP, steps=2)


def test_more_tensors_than_one_launch_table(cuda_lib):
    rng = np.random.default_rng(2)
    sizes = [int(s) for s in rng.integers(1, 20000, 300)]
    P, M, V, G, W = make(sizes, seed=2)
    run_both(cuda_lib, P, M, V, G, W, HP, steps=1)


def test_no_clip_and_clip_inactive(cuda_lib):
    P, M, V, G, W = make([4096, 5000], seed=3)
    run_both(cuda_lib, P, M, V, G, W, dict(HP, max_grad_norm=0.0), steps=1)
    run_both(cuda_lib, P, M, V, G, W, dict(HP, max_grad_norm=1e9), steps=1)


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_nonfinite_gradient_skips_update(cuda_lib, bad):
    P, M, V, G, W = make([1000, 3000], seed=4)
    G[1][1234] = bad
    before = [f32(t) for t in P + M + V]
    norm = torch.zeros(1, device="cuda"); skipped = torch.zeros(1, dtype=torch.int32, device="cuda")
    cuda_lib.fused_adamw_multi_tensor(P, M, V, G, W, grad_norm=norm, skipped=skipped, step=5, **HP)
    cuda_lib.fp8t_check_device_error()
    assert skipped.item() == 1 and not np.isfinite(norm.item())
    after = [f32(t) for t in P + M + V]
    assert all(np.array_equal(a, b) for a, b in zip(before, after))
    assert all(int(w.abs().sum().item()) == 0 for w in W)


def test_device_step_counter(cuda_lib):
    """With a device step counter the call performs counter+1, stores it back, and leaves it
    unchanged on a skipped step; results match the oracle at that step within 4 ulp."""
    P, M, V, G, W = make([5000, 70000], seed=6)
    counter = torch.tensor([41], dtype=torch.int64, device="cuda")
    host = [[f32(t) for t in P], [f32(t) for t in M], [f32(t) for t in V]]
    for k in range(3):
        norm = torch.zeros(1, device="cuda")
        cuda_lib.fused_adamw_multi_tensor(P, M, V, G, W, grad_norm=norm, step_counter=counter,
                                          step=0, **HP)
        cuda_lib.fp8t_check_device_error()
        assert counter.item() == 42 + k
        gbits = [bf16_bits(g) for g in G]
        oracle.fused_adamw(host[0], host[1], host[2], gbits, [np.zeros(g.size, np.uint16) for g in gbits],
                           dict(HP, step=42 + k))
        for i in range(2):
            for got, ref in ((P[i], host[0][i]), (M[i], host[1][i]), (V[i], host[2][i])):
                assert ulp_distance_f32(f32(got), ref).max() <= 4
    G[0][3] = float("nan")
    skipped = torch.zeros(1, dtype=torch.int32, device="cuda")
    cuda_lib.fused_adamw_multi_tensor(P, M, V, G, W, skipped=skipped, step_counter=counter, step=0, **HP)
    cuda_lib.fp8t_check_device_error()
    assert skipped.item() == 1 and counter.item() == 44


def test_adamw4e9_full_size_sampled(cuda_lib):
    """The 4.0e9-parameter, 512-tensor workload at full size in the benchmark's launch
    configuration. The oracle computes the global norm over every gradient (host copies) and
    the update of a seeded sample of tensors, compared element by element."""
    cfg = synth.ADAMW4E9
    sizes = synth.adamw_sizes(cfg["n_tensors"], cfg["total"], cfg["seed"], cfg["min_bytes"] // 4,
                              cfg["max_bytes"] // 4)
    free, _ = torch.cuda.mem_get_info()
    if free < 70e9:
        pytest.skip("needs ~64 GB of free device memory")
    P, M, V, G, W = make([int(s) for s in sizes], seed=cfg["seed"])
    hp = dict(cfg["hp"])
    rng = np.random.default_rng(0)
    pick = sorted(set(rng.choice(len(sizes), 6, replace=False).tolist()) | {int(np.argmax(sizes)), len(sizes) - 1})
    host = {i: (f32(P[i]), f32(M[i]), f32(V[i])) for i in pick}
    norm = torch.zeros(1, device="cuda"); skipped = torch.zeros(1, dtype=torch.int32, device="cuda")
    cuda_lib.fused_adamw_multi_tensor(P, M, V, G, W, grad_norm=norm, skipped=skipped, **hp)
    cuda_lib.fp8t_check_device_error()
    gbits_all = [bf16_bits(g) for g in G]
    rnorm = oracle.global_norm(gbits_all, hp["loss_scale"])
    assert ulp_distance_f32(np.float32(norm.item()), np.float32(rnorm)) <= 2
    assert skipped.item() == 0
    for i in pick:
        p, m, v = host[i]
        w = np.zeros(p.size, np.uint16)
        oracle.adamw_update([p], [m], [v], [gbits_all[i]], [w], hp, rnorm)
        for got, ref in ((P[i], p), (M[i], m), (V[i], v)):
            assert ulp_distance_f32(f32(got), ref).max() <= 4
        assert np.abs(bf16_bits(W[i]).astype(np.int32) - w.astype(np.int32)).max() <= 1
