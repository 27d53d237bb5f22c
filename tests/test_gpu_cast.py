"""Parity of fp8_cast_transpose_amax (C ABI, sm_100a) with the oracle: bit-exact codes,
transpose, amax, scale_inv and counters.

[P2] "FP8 混合精度训练工程实践" §四 quantize; [P3] "LLM FP8 微调上线生产实战" 核心原理 (HYBRID) and
工程落地 第四步 (saturation / zero metrics)."""
import numpy as np
import pytest
import torch

import oracle
from optimizer_fp8_cast_b200 import synth
from tests._gpu import bf16_bits, bf16_from_bits, dev_scalar, f32, u8

pytestmark = pytest.mark.gpu

SCALES = [1.0, 2.0 ** -3, 3.7, 1.0 / 3.0, 16384.0, 2.0 ** 100, 2.0 ** -100]


def run_gpu(fp8, x, fmt, scale, want_q=True, want_qT=True, counters=True):
    rows, cols = x.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda") if want_q else None
    qT = torch.empty(cols, rows, dtype=torch.uint8, device="cuda") if want_qT else None
    amax = torch.zeros(1, device="cuda")                            # max-accumulated from 0
    sinv = torch.zeros(1, device="cuda")
    cnt = torch.zeros(3, dtype=torch.int64, device="cuda") if counters else None
    fp8.fp8_cast_transpose_amax(x, fmt, dev_scalar(scale), q, qT, amax, sinv, cnt)
    fp8.fp8t_check_device_error()
    return (u8(q) if want_q else None, u8(qT) if want_qT else None,
            np.float32(amax.item()), np.float32(sinv.item()),
            cnt.cpu().numpy().astype(np.uint64) if counters else None)


def check(fp8, x_bits, fmt, scale):
    """Both kernels: the tiled one (q and q^T) and the streaming one (q only)."""
    x = bf16_from_bits(x_bits)
    rq, rqT, ramax, rsinv, rcnt = oracle.cast_transpose_amax(x_bits, fmt, scale)
    for want_qT in (True, False):
        q, qT, amax, sinv, cnt = run_gpu(fp8, x, fmt, scale, want_qT=want_qT)
        assert np.array_equal(q, rq), "row-major codes differ"
        assert not want_qT or np.array_equal(qT, rqT), "transposed codes differ"
        assert amax.view(np.uint32) == np.float32(ramax).view(np.uint32), (amax, ramax)
        assert sinv.view(np.uint32) == np.float32(rsinv).view(np.uint32)
        assert np.array_equal(cnt, rcnt), (cnt, rcnt)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("scale", SCALES)
def test_every_bf16_pattern(cuda_lib, fmt, scale):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    check(cuda_lib, bits, fmt, scale)
    # the same values in a different arrangement (rows and columns swapped, tail tiles)
    check(cuda_lib, np.ascontiguousarray(bits.reshape(128, 512)), fmt, scale)


@pytest.mark.parametrize("shape", [(16, 16), (48, 80), (144, 272), (128, 128), (256, 384),
                                   (1040, 2064), (16, 4096), (4096, 16)])
@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_ragged_shapes(cuda_lib, shape, fmt):
    g = torch.Generator().manual_seed(hash(shape) & 0xFFFF)
    x = torch.randn(shape, generator=g) * 3
    x[torch.rand(shape, generator=g) < 0.01] *= 1000
    bits = bf16_bits(x.to(torch.bfloat16))
    for scale in (1.0, 0.37, 200.0):
        check(cuda_lib, bits, fmt, scale)


def test_optional_outputs(cuda_lib):
    x = torch.randn(272, 144).to(torch.bfloat16)
    bits = bf16_bits(x)
    xd = bf16_from_bits(bits)
    rq, rqT, ramax, _, _ = oracle.cast_transpose_amax(bits, oracle.E4M3, 2.0)
    q, qT, amax, _, _ = run_gpu(cuda_lib, xd, oracle.E4M3, 2.0, want_qT=False, counters=False)
    assert qT is None and np.array_equal(q, rq) and amax == ramax
    q, qT, amax, _, _ = run_gpu(cuda_lib, xd, oracle.E4M3, 2.0, want_q=False)
    assert q is None and np.array_equal(qT, rqT)
    q, qT, amax, _, _ = run_gpu(cuda_lib, xd, oracle.E4M3, 2.0, want_q=False, want_qT=False)
    assert amax == ramax


def test_counters_accumulate(cuda_lib):
    x = torch.randn(512, 256) * 100
    xd = x.to(torch.bfloat16).cuda()
    cnt = torch.zeros(3, dtype=torch.int64, device="cuda")
    amax = torch.zeros(1, device="cuda")
    for _ in range(3):
        cuda_lib.fp8_cast_transpose_amax(xd, oracle.E4M3, dev_scalar(4.0), None, None, amax, None, cnt)
    _, _, _, _, rc = oracle.cast_transpose_amax(bf16_bits(xd), oracle.E4M3, 4.0)
    assert np.array_equal(cnt.cpu().numpy(), 3 * rc.astype(np.int64))


def test_amax_is_max_accumulated(cuda_lib):
    """The amax slot keeps the larger of its content and max|x|; NaN dominates."""
    x = (torch.randn(64, 64) * 3).to(torch.bfloat16)
    bits = bf16_bits(x)
    xd = bf16_from_bits(bits)
    for start in (0.0, 1e-3, 1e6, float("inf"), float("nan")):
        amax = torch.tensor([start], device="cuda")
        cuda_lib.fp8_cast_transpose_amax(xd, oracle.E4M3, dev_scalar(1.0), None, None, amax)
        _, _, ref, _, _ = oracle.cast_transpose_amax(bits, oracle.E4M3, 1.0, False, False, amax_in=start)
        got = np.float32(amax.item())
        assert got.view(np.uint32) == np.float32(ref).view(np.uint32), (start, got, ref)


def test_special_values_and_nan_amax(cuda_lib):
    bits = np.zeros((32, 32), np.uint16)
    bits[0, :8] = [0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x0001, 0x8001]
    for fmt in (oracle.E4M3, oracle.E5M2):
        check(cuda_lib, bits, fmt, 1.0)
    bits2 = np.full((32, 32), 0x8000, np.uint16)      # all -0: amax +0
    check(cuda_lib, bits2, oracle.E4M3, 1.0)


@pytest.mark.parametrize("name,rows,cols,fmt", [
    ("X linear4096", 8192, 4096, oracle.E4M3),
    ("W linear4096", 4096, 4096, oracle.E4M3),
    ("dY linear4096", 8192, 4096, oracle.E5M2),
    ("X of down, block7b", 16384, 11008, oracle.E4M3),
    ("dY of gate, block7b", 16384, 11008, oracle.E5M2),
])
def test_full_size_workload_shapes(cuda_lib, name, rows, cols, fmt):
    """Full-size tensors of the 4096 x 4096 / 8192-token Linear and the 7B-block projections,
    compared element by element."""
    std = 1e-3 if fmt == oracle.E5M2 else (0.02 if name.startswith("W") else 1.0)
    x = synth.normal_f32((rows, cols), std, synth.tensor_seed(0, name, 0), "cuda")
    if fmt == oracle.E5M2:
        x[torch.rand(rows, cols, device="cuda") < 1e-3] *= 1000
    xb = x.to(torch.bfloat16)
    del x
    scale = 448.0 / 4.5 if fmt == oracle.E4M3 else 57344.0 / 1.1
    check(cuda_lib, bf16_bits(xb), fmt, scale)


def test_multi_tensor_launch(cuda_lib):
    """Several casts in one launch (mixed shapes, formats and optional outputs) equal the
    per-tensor oracle, including more tensors than one launch table holds."""
    rng = np.random.default_rng(21)
    specs = [((272, 144), oracle.E4M3, 3.0, True, True), ((16, 4096), oracle.E5M2, 1000.0, True, True),
             ((1040, 48), oracle.E4M3, 0.5, False, True), ((128, 128), oracle.E5M2, 7.0, True, False)]
    specs = specs * 3                                   # 12 tensors: two launch tables
    casts, refs = [], []
    for (shape, fmt, scale, want_q, want_qT) in specs:
        x = torch.from_numpy((rng.standard_normal(shape) * 3).astype(np.float32)).to(torch.bfloat16)
        bits = bf16_bits(x)
        rows, cols = shape
        c = dict(x=bf16_from_bits(bits), fmt=fmt, scale=dev_scalar(scale),
                 q=torch.empty(rows, cols, dtype=torch.uint8, device="cuda") if want_q else None,
                 qT=torch.empty(cols, rows, dtype=torch.uint8, device="cuda") if want_qT else None,
                 amax=torch.zeros(1, device="cuda"), scale_inv=torch.zeros(1, device="cuda"),
                 counters=torch.zeros(3, dtype=torch.int64, device="cuda"))
        casts.append(c)
        refs.append(oracle.cast_transpose_amax(bits, fmt, scale))
    cuda_lib.fp8_cast_transpose_amax_multi(casts)
    cuda_lib.fp8t_check_device_error()
    for c, (rq, rqT, ramax, rsinv, rcnt) in zip(casts, refs):
        if c["q"] is not None:
            assert np.array_equal(u8(c["q"]), rq)
        if c["qT"] is not None:
            assert np.array_equal(u8(c["qT"]), rqT)
        assert np.float32(c["amax"].item()).view(np.uint32) == np.float32(ramax).view(np.uint32)
        assert np.float32(c["scale_inv"].item()) == rsinv
        assert np.array_equal(c["counters"].cpu().numpy().astype(np.uint64), rcnt)


@pytest.mark.parametrize("n,H,algo,margin", [(3, 1, oracle.AMAX_MAX, 0), (3, 16, oracle.AMAX_MAX, 1),
                                             (21, 16, oracle.AMAX_MOST_RECENT, 0),
                                             (5, 1024, oracle.AMAX_MAX, 0), (9, 3000, oracle.AMAX_MAX, 3)])
@pytest.mark.parametrize("with_qT", [True, False], ids=["tiled", "streaming"])
def test_cast_with_fused_scale_update(cuda_lib, n, H, algo, margin, with_qT):
    """fp8_cast_transpose_amax_update_multi equals the oracle's cast followed by its scale
    update ("LLM FP8 微调上线生产实战" 核心原理: history roll, representative amax, next scale), bit
    for bit: codes, inverse of the scale used, history, next scale and its inverse, amax slots
    reset, ticket left at zero. 21 tensors take three launches; H = 3000 needs several chunks of
    the warp roll. One tensor carries a NaN (its scale is kept) and one is all zero."""
    rng = np.random.default_rng(1000 + n + H)
    shapes = [(16 * int(rng.integers(1, 20)), 16 * int(rng.integers(1, 20))) for _ in range(n)]
    fmts = [oracle.E4M3 if i % 3 != 2 else oracle.E5M2 for i in range(n)]
    xs = []
    for i, (r, c) in enumerate(shapes):
        x = (rng.standard_normal((r, c)) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        if i == 1:
            x[r // 2, c // 3] = np.nan
        if i == n - 1:
            x[:] = 0.0
        xs.append(bf16_bits(torch.from_numpy(x).to(torch.bfloat16)))
    scale0 = (2.0 ** rng.uniform(-8, 8, n)).astype(np.float32)
    hist0 = np.abs(rng.standard_normal((n, H)) * 10.0 ** rng.uniform(-2, 2, (n, 1))).astype(np.float32)
    fp8_max = np.array([448.0 if f == oracle.E4M3 else 57344.0 for f in fmts], np.float32)

    scale = torch.from_numpy(scale0.copy()).cuda()
    hist = torch.from_numpy(hist0.copy()).cuda()
    amax = torch.zeros(n, device="cuda")
    sinv_used = torch.zeros(n, device="cuda")
    sinv_next = torch.zeros(n, device="cuda")
    ticket = torch.zeros(1, dtype=torch.int32, device="cuda")
    casts, ups = [], []
    for i, ((r, c), f) in enumerate(zip(shapes, fmts)):
        casts.append(dict(x=bf16_from_bits(xs[i]), fmt=f, scale=scale[i:i + 1],
                          q=torch.empty(r, c, dtype=torch.uint8, device="cuda"),
                          qT=torch.empty(c, r, dtype=torch.uint8, device="cuda") if with_qT else None,
                          amax=amax[i:i + 1], scale_inv=sinv_used[i:i + 1]))
        ups.append(dict(history=hist[i], scale_inv_next=sinv_next[i:i + 1]))
    cuda_lib.fp8_cast_transpose_amax_update_multi(casts, ups, algo, margin, ticket)
    cuda_lib.fp8t_check_device_error()

    amax_ref = np.zeros(n, np.float32)
    for i, f in enumerate(fmts):
        rq, rqT, ra, rsinv, _ = oracle.cast_transpose_amax(xs[i], f, scale0[i])
        assert np.array_equal(u8(casts[i]["q"]), rq)
        assert not with_qT or np.array_equal(u8(casts[i]["qT"]), rqT)
        assert np.float32(sinv_used[i].item()).view(np.uint32) == np.float32(rsinv).view(np.uint32)
        amax_ref[i] = ra
    h_ref, s_ref, si_ref = hist0.copy(), scale0.copy(), np.zeros(n, np.float32)
    oracle.scale_update(amax_ref, h_ref, fp8_max, algo, margin, s_ref, si_ref)
    assert np.array_equal(f32(hist).view(np.uint32), h_ref.view(np.uint32))
    assert np.array_equal(f32(scale).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(f32(sinv_next).view(np.uint32), si_ref.view(np.uint32))
    assert np.isnan(h_ref[1, 0]) and s_ref[1] == scale0[1]          # the NaN tensor kept its scale
    assert not amax.any().item() and ticket.item() == 0


def test_fused_scale_update_equals_separate_launch(cuda_lib):
    """Ten consecutive steps of three tensors: the fused launch and cast + fp8_scale_update in
    separate launches leave identical scale state and codes."""
    rng = np.random.default_rng(77)
    H, n = 16, 3
    shapes = [(512, 256), (256, 256), (512, 256)]
    fmts = [oracle.E4M3, oracle.E4M3, oracle.E5M2]
    fp8_max = torch.tensor([448.0, 448.0, 57344.0], device="cuda")
    state = [dict(scale=torch.ones(n, device="cuda"), hist=torch.zeros(n, H, device="cuda"),
                  amax=torch.zeros(n, device="cuda"), used=torch.zeros(n, device="cuda"),
                  nxt=torch.zeros(n, device="cuda")) for _ in range(2)]
    ticket = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(10):
        xs = [torch.from_numpy((rng.standard_normal(s) * 10.0 ** rng.uniform(-2, 2)).astype(np.float32))
              .to(torch.bfloat16).cuda() for s in shapes]
        outs = []
        for k, S in enumerate(state):
            casts = [dict(x=xs[i], fmt=fmts[i], scale=S["scale"][i:i + 1],
                          q=torch.empty(shapes[i], dtype=torch.uint8, device="cuda"),
                          amax=S["amax"][i:i + 1], scale_inv=S["used"][i:i + 1]) for i in range(n)]
            if k == 0:
                ups = [dict(history=S["hist"][i], scale_inv_next=S["nxt"][i:i + 1]) for i in range(n)]
                cuda_lib.fp8_cast_transpose_amax_update_multi(casts, ups, oracle.AMAX_MAX, 0, ticket)
            else:
                cuda_lib.fp8_cast_transpose_amax_multi(casts)
                cuda_lib.fp8_scale_update(S["amax"], S["hist"], fp8_max, oracle.AMAX_MAX, 0,
                                          S["scale"], S["nxt"])
            outs.append([c["q"] for c in casts])
        cuda_lib.fp8t_check_device_error()
        for a, b in zip(*outs):
            assert torch.equal(a, b)
        for key in ("scale", "hist", "amax", "used", "nxt"):
            assert torch.equal(state[0][key], state[1][key]), (t, key)


def test_current_scaling_multi(cuda_lib):
    """fp8_cast_transpose_amax_current_multi against the oracle's current scaling (amax of the
    tensor itself, then scale = (FP8_MAX / amax) / 2^margin, then the cast), bit for bit: scale
    written in place, codes, transposed codes, inverse scale, amax slot; 11 tensors (two amax
    launches), an all-zero tensor (scale 1) and one with an infinity (previous scale kept); the
    workspace is left zeroed."""
    rng = np.random.default_rng(31)
    n, margin = 11, 1
    shapes = [(16 * int(rng.integers(1, 40)), 16 * int(rng.integers(1, 40))) for _ in range(n)]
    shapes[0] = (4096, 2048)                             # a tensor large enough for many CTAs
    fmts = [oracle.E4M3 if i % 2 else oracle.E5M2 for i in range(n)]
    xs = []
    for i, (r, c) in enumerate(shapes):
        x = (rng.standard_normal((r, c)) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        if i == 3:
            x[:] = 0.0
        if i == 5:
            x[r - 1, c - 1] = np.inf
        xs.append(bf16_bits(torch.from_numpy(x).to(torch.bfloat16)))
    prev = [float(np.float32(2.0 ** rng.uniform(-4, 4))) for _ in range(n)]
    ws = torch.zeros(cuda_lib.CURRENT_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    casts = []
    for i, ((r, c), f) in enumerate(zip(shapes, fmts)):
        casts.append(dict(x=bf16_from_bits(xs[i]), fmt=f, scale=dev_scalar(prev[i]),
                          q=torch.empty(r, c, dtype=torch.uint8, device="cuda"),
                          qT=torch.empty(c, r, dtype=torch.uint8, device="cuda"),
                          amax=torch.zeros(1, device="cuda"), scale_inv=torch.zeros(1, device="cuda")))
    cuda_lib.fp8_cast_transpose_amax_current_multi(casts, margin, ws)
    cuda_lib.fp8t_check_device_error()
    for i, c in enumerate(casts):
        rq, rqT, ra, rs, rsinv, _ = oracle.cast_current(xs[i], fmts[i], margin, prev[i])
        assert np.float32(c["scale"].item()).view(np.uint32) == np.float32(rs).view(np.uint32), i
        assert np.array_equal(u8(c["q"]), rq) and np.array_equal(u8(c["qT"]), rqT), i
        assert np.float32(c["scale_inv"].item()).view(np.uint32) == np.float32(rsinv).view(np.uint32)
        assert np.float32(c["amax"].item()).view(np.uint32) == np.float32(ra).view(np.uint32)
    assert casts[3]["scale"].item() == 1.0 and casts[5]["scale"].item() == np.float32(prev[5])
    assert not ws.any().item()
