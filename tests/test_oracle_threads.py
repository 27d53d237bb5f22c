"""The oracle gives the same bits on one thread and on several.

Its loops are split over host threads only where the pieces are independent (output elements,
rows, blocks) or are combined by integer sums and maxima; the global-norm sum keeps its fixed
order (65,536-element chunks, each summed in order, combined pairwise). So the all-core timing
of the CPU baseline runs the same program as the single-thread one."""
import numpy as np
import pytest
import torch

import oracle
from optimizer_fp8_cast_b200.synth import bf16_bits


@pytest.fixture
def threads():
    before = oracle.get_threads()
    yield
    oracle.set_threads(before)


def _both(fn):
    oracle.set_threads(1)
    a = fn()
    n = oracle.set_threads(4)
    assert n == 4
    b = fn()
    return a, b


def _same(a, b):
    if isinstance(a, tuple):
        assert len(a) == len(b)
        for x, y in zip(a, b):
            _same(x, y)
    elif isinstance(a, np.ndarray):
        assert a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8))
    else:
        assert np.float64(a).tobytes() == np.float64(b).tobytes()


def test_cast_gemm_and_mx_are_thread_count_independent(threads):
    rng = np.random.default_rng(21)
    x = bf16_bits((torch.randn(300, 256) * 40).to(torch.bfloat16))
    x[5, 7] = 0x7FC1                                  # a NaN: amax and counters see it
    for fmt in (oracle.E4M3, oracle.E5M2):
        _same(*_both(lambda: oracle.cast_transpose_amax(x, fmt, 3.7)))
    A = rng.integers(0, 0x7E, (70, 96)).astype(np.uint8)
    B = rng.integers(0, 0x7B, (50, 96)).astype(np.uint8)
    _same(*_both(lambda: oracle.gemm(A, 0, B, 1, 0.25, 3.0, want_abs=True)))
    ii, jj = rng.integers(0, 70, 300), rng.integers(0, 50, 300)
    _same(*_both(lambda: oracle.gemm_at(A, 0, B, 1, 0.25, 3.0, ii, jj)))
    for axis in (0, 1):
        _same(*_both(lambda: oracle.mx_quantise(x[:288], axis, oracle.E4M3)))
    sfa = rng.integers(120, 135, (70, 3)).astype(np.uint8)
    sfb = rng.integers(120, 135, (50, 3)).astype(np.uint8)
    _same(*_both(lambda: oracle.mx_gemm(A, sfa, 0, B, sfb, 1, want_abs=True)))


def test_norm_and_adamw_are_thread_count_independent(threads):
    rng = np.random.default_rng(22)
    sizes = [3, 65536, 65537, 200001, 131072 * 3 + 5]      # chunk edges and ragged tails
    g = [bf16_bits(torch.from_numpy(rng.standard_normal(n).astype(np.float32) * 30).to(torch.bfloat16))
         for n in sizes]
    _same(*_both(lambda: oracle.global_norm(g, 1024.0)))
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, step=3,
              loss_scale=1024.0, max_grad_norm=1.0)

    def run():
        P = [rng2.standard_normal(n).astype(np.float32) for n in sizes]
        M = [np.full(n, 1e-3, np.float32) for n in sizes]
        V = [np.full(n, 1e-6, np.float32) for n in sizes]
        W = [np.zeros(n, np.uint16) for n in sizes]
        norm, skip = oracle.fused_adamw(P, M, V, g, W, hp)
        return (np.float64(norm), np.float64(skip), *P, *M, *V, *W)

    rng2 = np.random.default_rng(1)
    a = run()
    oracle.set_threads(4)
    rng2 = np.random.default_rng(1)
    b = run()
    oracle.set_threads(1)
    rng2 = np.random.default_rng(1)
    c = run()
    _same(a, b)
    _same(a, c)
