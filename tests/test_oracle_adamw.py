"""Pins of the oracle's global norm and fused AdamW.

[P1] "算子与编译器：FP8 训练与优化器 Kernel", Fused Optimizer 的意义 (grad -> moments -> bias
correction -> weight decay -> parameter update) and FP8 训练主路径图 (unscale / clip before the
optimizer); [P2] "FP8 混合精度训练工程实践", §四 (loss scale x1024, un-scaling, FP32 AdamW).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests._pins import bf16_to_f32, ulp_distance_f32

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _run(master, m, v, g_bits, hp):
    w = [np.zeros(a.size, np.uint16) for a in master]
    norm, skipped = oracle.fused_adamw(master, m, v, g_bits, w, hp)
    return norm, skipped, w


def test_two_step_hand_expansion():
    gold = json.load(open(os.path.join(GOLD, "adamw_two_step.json")))
    hp = dict(gold["hp"]); hp["loss_scale"] = gold["loss_scale"]
    p = [np.array([gold["p0"]], np.float32)]
    m = [np.zeros(1, np.float32)]; v = [np.zeros(1, np.float32)]
    for t, (gs, want) in enumerate(zip(gold["scaled_grads"], gold["p_expected"]), start=1):
        hp["step"] = t
        _run(p, m, v, [_bf16([gs])], hp)
        # bias-corrected moments equal the hand-expanded closed forms
        # (the hyperparameters reach the optimizer as f32, so correct with the f32 betas)
        mhat = m[0][0] / (1 - float(np.float32(hp["beta1"])) ** t)
        vhat = v[0][0] / (1 - float(np.float32(hp["beta2"])) ** t)
        assert math.isclose(mhat, gold["m_hat"][t - 1], rel_tol=1e-6)
        assert math.isclose(vhat, gold["v_hat"][t - 1], rel_tol=1e-6)
        assert ulp_distance_f32(p[0][0], np.float32(want)) <= 4, (t, p[0][0], want)


@pytest.mark.parametrize("seed", [0, 1])
def test_first_step_closed_form(seed):
    """With m = v = 0 at step 1 the bias corrections cancel: the update is
    p1 = p0 (1 - lr wd) - lr g / (|g| + eps) for the unscaled, clipped g."""
    rng = np.random.default_rng(seed)
    n = 4096
    p0 = rng.normal(0, 0.02, n).astype(np.float32)
    gs = _bf16(rng.normal(0, 1e-3, n) * 1024)
    hp = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, loss_scale=1024.0,
              max_grad_norm=0.0, step=1)
    p = [p0.copy()]; m = [np.zeros(n, np.float32)]; v = [np.zeros(n, np.float32)]
    _run(p, m, v, [gs], hp)
    g = bf16_to_f32(gs).astype(np.float64) / 1024
    decayed = p0.astype(np.float64) * (1 - 3e-4 * 0.1)
    step = 3e-4 * g / (np.abs(g) + 1e-8)
    want = decayed - step
    # a handful of f32 roundings of operands of size |decayed| + |step|; near cancellation the
    # result's own ulp is smaller, so the bound is taken on the operands
    bound = 4 * np.spacing((np.abs(decayed) + np.abs(step)).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(p[0].astype(np.float64) - want) <= bound)


def test_clip_coefficient_closed_form():
    """Four gradients of 2 (scaled by 1024) have unscaled norm 4; with clip 1 the effective
    gradient is 0.5, and the returned norm is exactly 4."""
    gs = _bf16([2048.0] * 4)
    hp = dict(lr=0.1, beta1=0.9, beta2=0.999, eps=0.0, weight_decay=0.0, loss_scale=1024.0,
              max_grad_norm=1.0, step=1)
    p = [np.ones(4, np.float32)]; m = [np.zeros(4, np.float32)]; v = [np.zeros(4, np.float32)]
    norm, skipped, w = _run(p, m, v, [gs], hp)
    assert norm == 4.0 and skipped == 0
    omb1 = np.float32(1.0 - float(np.float32(0.9)))                      # 1 - f32(beta1)
    assert np.all(m[0] == np.float32(omb1 * np.float32(0.5)))             # (1-b1) * 0.5
    assert np.all(p[0] == np.float32(0.9))                                 # 1 - lr * sign(g)


def test_lr_zero_keeps_weights():
    rng = np.random.default_rng(2)
    p0 = rng.normal(0, 1, 1000).astype(np.float32)
    hp = dict(lr=0.0, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.5, loss_scale=1.0,
              max_grad_norm=0.0, step=3)
    p = [p0.copy()]; m = [np.zeros(1000, np.float32)]; v = [np.zeros(1000, np.float32)]
    _, _, w = _run(p, m, v, [_bf16(rng.normal(0, 1, 1000))], hp)
    assert np.array_equal(p[0], p0) and np.count_nonzero(m[0]) > 900
    assert np.array_equal(w[0], _bf16(p0))


@pytest.mark.parametrize("bad", [np.nan, np.inf])
def test_nonfinite_gradient_skips(bad):
    g = np.ones(64, np.float32); g[17] = bad
    hp = dict(lr=0.1, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, loss_scale=1.0,
              max_grad_norm=1.0, step=1)
    p = [np.ones(64, np.float32)]; m = [np.zeros(64, np.float32)]; v = [np.zeros(64, np.float32)]
    norm, skipped, w = _run(p, m, v, [_bf16(g)], hp)
    assert skipped == 1 and not np.isfinite(norm)
    assert np.all(p[0] == 1) and np.all(m[0] == 0) and np.all(w[0] == 0)


def test_global_norm_against_numpy():
    rng = np.random.default_rng(4)
    gs = [_bf16(rng.normal(0, 1e-3, n) * 1024) for n in (1, 7, 1000, 65537)]
    norm = oracle.global_norm(gs, 1024.0)
    G = sum(np.sum(bf16_to_f32(g).astype(np.float64) ** 2) for g in gs)   # pairwise order
    assert ulp_distance_f32(norm, np.float32(math.sqrt(G) / 1024)) <= 1


def test_matches_torch_adamw_three_steps():
    """Library cross-check: torch.optim.AdamW (FP32, CPU, single-tensor path) on the unscaled,
    clipped gradient agrees within 4 f32 ulp (its operation order differs slightly)."""
    rng = np.random.default_rng(6)
    n = 20000
    p0 = rng.normal(0, 0.02, n).astype(np.float32)
    hp = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, loss_scale=1024.0,
              max_grad_norm=1.0)
    p = [p0.copy()]; m = [np.zeros(n, np.float32)]; v = [np.zeros(n, np.float32)]
    tp = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([tp], lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]), eps=hp["eps"],
                            weight_decay=hp["weight_decay"], foreach=False, fused=False)
    for step in (1, 2, 3):
        prev = p[0].copy()
        gs = _bf16(rng.normal(0, 1e-3, n) * 1024)
        hp["step"] = step
        norm, _, _ = _run(p, m, v, [gs], hp)
        coef = np.float32(1.0) if norm <= 1.0 else np.float32(np.float32(1.0) / np.float32(norm))
        f = np.float32(coef * np.float32(1 / 1024))
        tp.grad = torch.from_numpy(bf16_to_f32(gs) * f)
        opt.step()
        # within 4 ulp of the operands (|p| and the step size): the two differ in rounding order
        # only, and near cancellation the result's own ulp is smaller than the operands'
        ops = np.abs(prev) + np.float32(hp["lr"] / (1 - hp["beta1"] ** step))
        bound = 4 * np.spacing(ops.astype(np.float32)).astype(np.float64)
        diff = np.abs(p[0].astype(np.float64) - tp.detach().numpy().astype(np.float64))
        assert np.all(diff <= bound)
        assert np.mean(ulp_distance_f32(p[0], tp.detach().numpy()) == 0) > 0.9
