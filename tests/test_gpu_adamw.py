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


def sumsq_of(G):
    """FP64 sum of f32(g)^2 over all gradients: the input the presummed call expects (squares of
    BF16 values are exact in FP64; numpy's pairwise sum rounds ~1e-16 relative)."""
    return torch.tensor([sum(float(np.sum(np.square(f32(g.float()).astype(np.float64)))) for g in G)],
                        dtype=torch.float64, device="cuda")


def run_both(fp8, P, M, V, G, W, hp, steps=1, presummed=False):
    host = [[f32(t) for t in P], [f32(t) for t in M], [f32(t) for t in V]]
    for step in range(1, steps + 1):
        hpp = dict(hp, step=step + 999)
        norm = torch.zeros(1, device="cuda"); skipped = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        if presummed:
            fp8.fused_adamw_multi_tensor_presummed(P, M, V, G, W, grad_sumsq=sumsq_of(G),
                                                   grad_norm=norm, skipped=skipped, **hpp)
        else:
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


def test_presummed_matches_oracle(cuda_lib):
    """fused_adamw_multi_tensor_presummed (sum of squares given, no norm pass) against the oracle,
    which forms the norm itself: ragged tensors, two steps, clip active."""
    P, M, V, G, W = make([1, 7, 8193, 100003], seed=11)
    run_both(cuda_lib, P, M, V, G, W, HP, steps=2, presummed=True)


def test_presummed_device_counter_over_two_launch_tables(cuda_lib):
    """300 tensors (two launches) with a device step counter: every call performs counter+1 in
    both launches, the last CTA of the last launch advances the counter, the ticket returns to
    zero; a NaN sum of squares skips the update and leaves the counter alone."""
    rng = np.random.default_rng(12)
    sizes = [int(x) for x in rng.integers(1, 5000, 300)]
    P, M, V, G, W = make(sizes, seed=12)
    counter = torch.tensor([99], dtype=torch.int64, device="cuda")
    ticket = torch.zeros(1, dtype=torch.int32, device="cuda")
    host = [[f32(t) for t in P], [f32(t) for t in M], [f32(t) for t in V]]
    for k in range(3):
        cuda_lib.fused_adamw_multi_tensor_presummed(P, M, V, G, W, grad_sumsq=sumsq_of(G), step=0,
                                                    step_counter=counter, ticket=ticket, **HP)
        cuda_lib.fp8t_check_device_error()
        assert counter.item() == 100 + k and ticket.item() == 0
        gbits = [bf16_bits(g) for g in G]
        oracle.fused_adamw(host[0], host[1], host[2], gbits,
                           [np.zeros(g.size, np.uint16) for g in gbits], dict(HP, step=100 + k))
        for i in (0, 150, 299):
            for got, ref in ((P[i], host[0][i]), (M[i], host[1][i]), (V[i], host[2][i])):
                assert ulp_distance_f32(f32(got), ref).max() <= 4
    before = [f32(t) for t in P[:3]]
    skipped = torch.zeros(1, dtype=torch.int32, device="cuda")
    nan = torch.tensor([float("nan")], dtype=torch.float64, device="cuda")
    cuda_lib.fused_adamw_multi_tensor_presummed(P, M, V, G, W, grad_sumsq=nan, skipped=skipped,
                                                step=0, step_counter=counter, ticket=ticket, **HP)
    cuda_lib.fp8t_check_device_error()
    assert skipped.item() == 1 and counter.item() == 102 and ticket.item() == 0
    assert all(np.array_equal(a, f32(b)) for a, b in zip(before, P[:3]))


def _weight_casts(shapes, fmts, scales):
    casts = []
    for (r, c), f, s in zip(shapes, fmts, scales):
        if r == 0:
            casts.append(None)
            continue
        casts.append(dict(rows=r, cols=c, fmt=f, scale=torch.tensor([s], device="cuda"),
                          q=torch.full((r, c), 0xAB, dtype=torch.uint8, device="cuda"),
                          amax=torch.zeros(1, device="cuda"), scale_inv=torch.zeros(1, device="cuda")))
    return casts


def _check_weight_casts(W, casts, scales):
    from tests._gpu import u8
    for w, c, s in zip(W, casts, scales):
        if c is None:
            continue
        bits = bf16_bits(w).reshape(c["rows"], c["cols"])
        q, _, a, si, _ = oracle.cast_transpose_amax(bits, c["fmt"], s, True, False)
        assert np.array_equal(u8(c["q"]), q)
        assert np.float32(c["amax"].item()).view(np.uint32) == np.float32(a).view(np.uint32)
        assert np.float32(c["scale_inv"].item()).view(np.uint32) == np.float32(si).view(np.uint32)


def test_presummed_with_weight_casts(cuda_lib):
    """The next step's weight cast inside AdamW ("算子与编译器" 优化器 kernel 的带宽账: one pass over
    the parameters): the update matches the oracle, and the row-major codes, amax and scale
    inverse of each new BF16 weight match the oracle's cast of it. Both formats, a tensor
    without a cast among them, and 40 casts (two launch tables). Then a skipped step (NaN sum of
    squares): weights unchanged and cast again with a new scale."""
    rng = np.random.default_rng(13)
    shapes = [(272, 400), (16, 16), (0, 0), (4096 // 8, 128 * 3), (64, 2064)]
    shapes += [(16 * int(rng.integers(1, 9)), 16 * int(rng.integers(1, 9))) for _ in range(38)]
    sizes = [r * c if r else 7777 for r, c in shapes]
    fmts = [oracle.E4M3 if i % 5 else oracle.E5M2 for i in range(len(shapes))]
    scales = [float(np.float32(2.0 ** rng.uniform(2, 12))) for _ in shapes]
    P, M, V, G, W = make(sizes, seed=13)
    casts = _weight_casts(shapes, fmts, scales)
    host = [[f32(t) for t in P], [f32(t) for t in M], [f32(t) for t in V]]
    hp = dict(HP, step=7)
    cuda_lib.fused_adamw_multi_tensor_presummed(P, M, V, G, W, grad_sumsq=sumsq_of(G), casts=casts, **hp)
    cuda_lib.fp8t_check_device_error()
    gbits = [bf16_bits(g) for g in G]
    wref = [np.zeros(g.size, np.uint16) for g in gbits]
    oracle.fused_adamw(host[0], host[1], host[2], gbits, wref, hp)
    for i in range(len(P)):
        assert ulp_distance_f32(f32(P[i]), host[0][i]).max() <= 4
        assert np.array_equal(bf16_bits(W[i]), bf16_bits(P[i].to(torch.bfloat16)))
    _check_weight_casts(W, casts, scales)

    # skipped step: nothing updated, the unchanged weights cast again with new scales
    before = [bf16_bits(w).copy() for w in W]
    scales2 = [s * 0.5 for s in scales]
    for c, s in zip(casts, scales2):
        if c is not None:
            c["scale"].fill_(s)
            c["amax"].zero_()
    skipped = torch.zeros(1, dtype=torch.int32, device="cuda")
    nan = torch.tensor([float("nan")], dtype=torch.float64, device="cuda")
    cuda_lib.fused_adamw_multi_tensor_presummed(P, M, V, G, W, grad_sumsq=nan, casts=casts,
                                                skipped=skipped, **dict(HP, step=8))
    cuda_lib.fp8t_check_device_error()
    assert skipped.item() == 1
    assert all(np.array_equal(b, bf16_bits(w)) for b, w in zip(before, W))
    _check_weight_casts(W, casts, scales2)
