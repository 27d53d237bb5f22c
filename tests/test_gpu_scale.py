"""Parity of fp8_scale_update (C ABI, sm_100a) with the oracle: bit-exact history, scales and
scale inverses. [P3] "LLM FP8 微调上线生产实战", 核心原理 (scale formula, delayed history)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H", [1, 2, 16, 255, 256, 257, 1024, 4097])
@pytest.mark.parametrize("algo", [oracle.AMAX_MAX, oracle.AMAX_MOST_RECENT])
@pytest.mark.parametrize("margin", [0, 1, 7])
def test_random_histories(cuda_lib, H, algo, margin):
    rng = np.random.default_rng(H * 10 + algo * 3 + margin)
    n = 21
    hist = (rng.lognormal(0, 3, (n, H))).astype(np.float32)
    hist[rng.random((n, H)) < 0.05] = 0.0
    scale = rng.uniform(0.5, 2.0, n).astype(np.float32)
    sinv = np.zeros(n, np.float32)
    fp8_max = np.array([448.0, 448.0, 57344.0] * 7, np.float32)
    dh, ds, dsi, dm = (torch.from_numpy(a.copy()).cuda() for a in (hist, scale, sinv, fp8_max))
    for step in range(3):
        amax = rng.lognormal(0, 3, n).astype(np.float32)
        amax[:3] = [0.0, np.nan, np.inf] if step == 1 else amax[:3]
        amax[3] = 1e-40
        damax = torch.from_numpy(amax.copy()).cuda()
        cuda_lib.fp8_scale_update(damax, dh, dm, algo, margin, ds, dsi)
        oracle.scale_update(amax, hist, fp8_max, algo, margin, scale, sinv)
        cuda_lib.fp8t_check_device_error()
        assert not damax.any().item() and not amax.any()         # consumed slots reset to 0
        assert np.array_equal(dh.cpu().numpy().view(np.uint32), hist.view(np.uint32))
        assert np.array_equal(ds.cpu().numpy().view(np.uint32), scale.view(np.uint32))
        assert np.array_equal(dsi.cpu().numpy().view(np.uint32), sinv.view(np.uint32))
