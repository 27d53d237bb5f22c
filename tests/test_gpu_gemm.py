"""Parity of fp8_gemm (C ABI, tcgen05 on sm_100a) with the oracle's exact GEMM:
|D - D_ref| <= 2 BF16 ulp + 1e-5 * sum_k |a_k b_k| * scale for every compared element.

[P2] "FP8 混合精度训练工程实践" §三 (FP8 GEMM, FP32 accumulation, 16-bit output), §五 (per-tensor
mode)."""
import numpy as np
import pytest
import torch

import oracle
from optimizer_fp8_cast_b200 import synth
from tests._gpu import bf16_bits, dev_scalar, f32, sample_positions, u8
from tests._pins import gemm_within_tolerance

pytestmark = pytest.mark.gpu
PAIRS = [(oracle.E4M3, oracle.E4M3), (oracle.E5M2, oracle.E4M3), (oracle.E4M3, oracle.E5M2),
         (oracle.E5M2, oracle.E5M2)]


def codes_from_normal(fp8, rows, cols, fmt, std, seed):
    """FP8 operand made by the library's own cast of seeded normal data (realistic codes)."""
    x = synth.normal_f32((rows, cols), std, seed, "cuda").to(torch.bfloat16)
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    amax = torch.zeros(1, device="cuda")
    scale = (448.0 if fmt == oracle.E4M3 else 57344.0) / (5.0 * std)
    fp8.fp8_cast_transpose_amax(x, fmt, dev_scalar(scale), q, None, amax)
    return q


def random_codes(rows, cols, fmt, seed):
    rng = np.random.default_rng(seed)
    t = oracle.decode_table(fmt)
    ok = np.flatnonzero(np.isfinite(t) & (np.abs(t) <= (64 if fmt == oracle.E5M2 else 448)))
    return torch.from_numpy(rng.choice(ok, size=(rows, cols)).astype(np.uint8)).cuda()


def run(fp8, A, af, B, bf, sa, sb):
    M, N = A.shape[0], B.shape[0]
    D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    fp8.fp8_gemm(A, af, B, bf, dev_scalar(sa), dev_scalar(sb), D)
    fp8.fp8t_check_device_error()
    return bf16_bits(D)


@pytest.mark.parametrize("af,bf", PAIRS)
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (512, 256, 256), (256, 256, 512),
                                   (16, 16, 16), (144, 272, 48), (400, 528, 1040),
                                   (128, 256, 4096)])
def test_full_compare_small(cuda_lib, af, bf, M, N, K):
    A = random_codes(M, K, af, M * 7 + K)
    B = random_codes(N, K, bf, N * 13 + K)
    sa, sb = 0.013, 0.7
    D = run(cuda_lib, A, af, B, bf, sa, sb)
    R, ab = oracle.gemm(u8(A), af, u8(B), bf, sa, sb, want_abs=True)
    ok = gemm_within_tolerance(D, R, ab)
    assert ok.all(), f"{(~ok).sum()} of {ok.size} outside tolerance, first at {np.argwhere(~ok)[:3]}"


def test_realistic_codes_and_step_shapes(cuda_lib):
    """The three GEMMs of the 256 x 256 / 512-token Linear with codes from the library cast."""
    T, fin, fout = 512, 256, 256
    Xq = codes_from_normal(cuda_lib, T, fin, oracle.E4M3, 1.0, 1)
    WqT = codes_from_normal(cuda_lib, fout, fin, oracle.E4M3, 0.02, 2)
    dYq = codes_from_normal(cuda_lib, T, fout, oracle.E5M2, 1e-3, 3)
    for A, af, B, bf in ((Xq, 0, WqT, 0), (dYq, 1, WqT.t().contiguous(), 0),
                         (Xq.t().contiguous(), 0, dYq.t().contiguous(), 1)):
        D = run(cuda_lib, A, af, B, bf, 0.01, 0.002)
        R, ab = oracle.gemm(u8(A), af, u8(B), bf, 0.01, 0.002, want_abs=True)
        assert gemm_within_tolerance(D, R, ab).all()


def test_output_overwritten_and_nan_propagates(cuda_lib):
    A = random_codes(128, 128, 0, 5)
    B = random_codes(256, 128, 0, 6)
    A[3, 7] = 0x7F                       # NaN code
    D = run(cuda_lib, A, 0, B, 0, 1.0, 1.0)
    R = oracle.gemm(u8(A), 0, u8(B), 0, 1.0, 1.0)
    Df = (D.astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.isnan(Df[3])) and not np.isnan(np.delete(Df, 3, 0)).any()
    assert gemm_within_tolerance(D, R, np.zeros(R.shape)).sum() > 0


@pytest.mark.parametrize("M,N,K,af,bf,label", [
    (8192, 4096, 4096, 0, 0, "fprop linear4096"),
    (8192, 4096, 4096, 1, 0, "dgrad linear4096"),
    (4096, 4096, 8192, 0, 1, "wgrad linear4096"),
    (16384, 11008, 4096, 0, 0, "fprop gate/up block7b"),
    (16384, 4096, 11008, 0, 0, "fprop down block7b"),
    (4096, 11008, 16384, 0, 1, "wgrad gate/up block7b"),
    (11008, 4096, 16384, 0, 1, "wgrad down block7b"),
])
def test_full_size_sampled(cuda_lib, M, N, K, af, bf, label):
    """Full-size GEMMs of the benchmark workloads in the launch configuration the benchmark uses,
    checked on ~6,000 seeded output positions including tile edges."""
    A = codes_from_normal(cuda_lib, M, K, af, 1.0 if af == 0 else 1e-3, M + K)
    B = codes_from_normal(cuda_lib, N, K, bf, 0.02 if bf == 0 else 1e-3, N + 3 * K)
    sa, sb = 1.0 / 89.6, 1.0 / 4480.0
    D = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    cuda_lib.fp8_gemm(A, af, B, bf, dev_scalar(sa), dev_scalar(sb), D)
    cuda_lib.fp8t_check_device_error()
    ii, jj = sample_positions(M, N, 4096, seed=M ^ N ^ K)
    Dh = bf16_bits(D)[ii, jj]
    R, ab = oracle.gemm_at(u8(A), af, u8(B), bf, sa, sb, ii, jj)
    ok = gemm_within_tolerance(Dh, R, ab)
    assert ok.all(), f"{label}: {(~ok).sum()} of {ok.size} samples outside tolerance"


def test_grouped_launch_mixed_problems(cuda_lib):
    """Problems of different shapes and formats in one launch (and more than one launch table)
    each equal the oracle within the GEMM tolerance."""
    rng = np.random.default_rng(42)
    shapes = [(144, 272, 48), (512, 256, 256), (16, 16, 16), (400, 528, 1040), (256, 768, 128)]
    probs = []
    for i in range(26):                                  # 26 problems: two launch tables
        M, N, K = shapes[i % len(shapes)]
        af, bf = PAIRS[i % 4]
        A = random_codes(M, K, af, 100 + i)
        B = random_codes(N, K, bf, 200 + i)
        sa, sb = float(rng.uniform(0.01, 1)), float(rng.uniform(0.01, 1))
        probs.append(dict(A=A, a_fmt=af, B=B, b_fmt=bf, a_scale_inv=dev_scalar(sa),
                          b_scale_inv=dev_scalar(sb), D=torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda"),
                          sa=sa, sb=sb))
    cuda_lib.fp8_gemm_multi([{k: v for k, v in p.items() if k not in ("sa", "sb")} for p in probs])
    cuda_lib.fp8t_check_device_error()
    for p in probs:
        R, ab = oracle.gemm(u8(p["A"]), p["a_fmt"], u8(p["B"]), p["b_fmt"], p["sa"], p["sb"], want_abs=True)
        assert gemm_within_tolerance(bf16_bits(p["D"]), R, ab).all()


def test_grouped_launch_with_sum_of_squares(cuda_lib):
    """fp8_gemm_multi_sumsq: D as in fp8_gemm_multi, plus the FP64 sum of f32(D)^2 over the
    flagged problems only (the AdamW global-norm input, "算子与编译器" FP8 训练主路径图), across two
    launch tables and ragged tiles; a repeated call gives the identical bits and the workspace
    ticket is left at zero."""
    rng = np.random.default_rng(43)
    shapes = [(144, 272, 48), (512, 256, 256), (16, 16, 16), (400, 528, 1040), (256, 768, 128)]
    probs = []
    for i in range(27):                                  # 27 problems: two launch tables
        M, N, K = shapes[i % len(shapes)]
        af, bf = PAIRS[i % 4]
        A = random_codes(M, K, af, 300 + i)
        B = random_codes(N, K, bf, 400 + i)
        sa, sb = float(rng.uniform(0.01, 1)), float(rng.uniform(0.01, 1))
        probs.append(dict(A=A, a_fmt=af, B=B, b_fmt=bf, a_scale_inv=dev_scalar(sa),
                          b_scale_inv=dev_scalar(sb), sumsq=(i % 3 == 1) or i == 26,
                          D=torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda"),
                          sa=sa, sb=sb))
    descs = [{k: v for k, v in p.items() if k not in ("sa", "sb")} for p in probs]
    ws = torch.zeros(cuda_lib.fp8_gemm_sumsq_workspace_bytes(descs), dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    cuda_lib.fp8_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    first = out.item()
    for p in probs:
        R, ab = oracle.gemm(u8(p["A"]), p["a_fmt"], u8(p["B"]), p["b_fmt"], p["sa"], p["sb"], want_abs=True)
        assert gemm_within_tolerance(bf16_bits(p["D"]), R, ab).all()
    squares = np.concatenate([np.square(f32(p["D"].float()).astype(np.float64)).reshape(-1)
                              for p in probs if p["sumsq"]])
    exact = float(np.sum(np.sort(squares)))
    assert abs(first - exact) <= 1e-13 * exact
    assert ws[:4].view(torch.int32).item() == 0
    cuda_lib.fp8_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    assert np.float64(out.item()).view(np.uint64) == np.float64(first).view(np.uint64)


@pytest.mark.parametrize("a_mn,b_mn", [(False, True), (True, False), (True, True)],
                         ids=["B-MN-major", "A-MN-major", "both-MN-major"])
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (144, 272, 48), (400, 528, 1040),
                                   (256, 768, 4096), (16, 16, 16)])
def test_mn_major_operands(cuda_lib, a_mn, b_mn, M, N, K):
    """Operands stored MN-major (A as K x M, B as K x N, row-major) give the product of the same
    logical matrices: the tensor cores read 8-bit operands in either order, which is what lets
    the step skip the transposed FP8 copies. All four format pairs, ragged tiles."""
    for i, (af, bf) in enumerate(PAIRS):
        A = random_codes(M, K, af, 1000 + M + K + i)
        B = random_codes(N, K, bf, 2000 + N + K + i)
        sa, sb = 0.021, 0.37
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        cuda_lib.fp8_gemm_multi([dict(A=A.t().contiguous() if a_mn else A, a_mn=a_mn, a_fmt=af,
                                      B=B.t().contiguous() if b_mn else B, b_mn=b_mn, b_fmt=bf,
                                      a_scale_inv=dev_scalar(sa), b_scale_inv=dev_scalar(sb), D=D)])
        cuda_lib.fp8t_check_device_error()
        R, ab = oracle.gemm(u8(A), af, u8(B), bf, sa, sb, want_abs=True)
        ok = gemm_within_tolerance(bf16_bits(D), R, ab)
        assert ok.all(), f"pair {i}: {(~ok).sum()} of {ok.size} outside tolerance"


def test_step_layouts_full_size_sampled(cuda_lib):
    """The 4096-class step's GEMMs exactly as the step issues them, in one grouped launch: fprop
    (Xq K-major, Wq MN-major), dgrad (dYq, Wq both K-major), wgrad (Xq, dYq both MN-major, K =
    8192 tokens), each on 4096 sampled outputs against the oracle's transposed operands."""
    T, fin, fout = 8192, 4096, 4096
    Xq = random_codes(T, fin, oracle.E4M3, 1)
    Wq = random_codes(fin, fout, oracle.E4M3, 2)
    dYq = random_codes(T, fout, oracle.E5M2, 3)
    s = [dev_scalar(v) for v in (0.011, 0.023, 0.5)]
    Y = torch.empty(T, fout, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(T, fin, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(fin, fout, dtype=torch.bfloat16, device="cuda")
    cuda_lib.fp8_gemm_multi([
        dict(A=Xq, a_fmt=0, B=Wq, b_mn=True, b_fmt=0, a_scale_inv=s[0], b_scale_inv=s[1], D=Y),
        dict(A=dYq, a_fmt=1, B=Wq, b_fmt=0, a_scale_inv=s[2], b_scale_inv=s[1], D=dX),
        dict(A=Xq, a_mn=True, a_fmt=0, B=dYq, b_mn=True, b_fmt=1, a_scale_inv=s[0],
             b_scale_inv=s[2], D=dW)])
    cuda_lib.fp8t_check_device_error()
    hX, hW, hdY = u8(Xq), u8(Wq), u8(dYq)
    for D, A, af, B, bf, sa, sb in ((Y, hX, 0, hW.T, 0, 0.011, 0.023), (dX, hdY, 1, hW, 0, 0.5, 0.023),
                                    (dW, hX.T, 0, hdY.T, 1, 0.011, 0.5)):
        ii, jj = sample_positions(D.shape[0], D.shape[1], 4096, seed=D.shape[1])
        R, ab = oracle.gemm_at(np.ascontiguousarray(A), af, np.ascontiguousarray(B), bf, sa, sb, ii, jj)
        assert gemm_within_tolerance(bf16_bits(D)[ii, jj], R, ab).all()


@pytest.mark.parametrize("shapes", [[(256, 512, 256)], [(400, 528, 1040)],
                                    [(512, 1024, 4096), (256, 768, 128), (1040, 1552, 272),
                                     (128, 512, 64)]],
                         ids=["one-tile-in-halves", "ragged", "grouped"])
def test_wide_tiles_with_sum_of_squares(cuda_lib, shapes):
    """Launches whose every problem is at least 512 wide run 256 x 512 tiles, and the schedule
    splits tiles into their two 256-column halves on different clusters where that evens out the
    load (a launch with fewer tiles than clusters is split throughout). Every output against the
    oracle, mixed formats and operand layouts, and the FP64 sum of squares of the flagged
    problems against numpy's; a repeat gives identical bits and leaves the workspace at zero."""
    rng = np.random.default_rng(len(shapes) * 7)
    probs = []
    for i, (M, N, K) in enumerate(shapes):
        af, bf = PAIRS[(i + 1) % 4]
        A = random_codes(M, K, af, 500 + i)
        B = random_codes(N, K, bf, 600 + i)
        a_mn, b_mn = bool(i % 2), bool((i // 2) % 2)
        sa, sb = float(rng.uniform(0.01, 1)), float(rng.uniform(0.01, 1))
        probs.append(dict(A=A.t().contiguous() if a_mn else A, a_mn=a_mn, a_fmt=af,
                          B=B.t().contiguous() if b_mn else B, b_mn=b_mn, b_fmt=bf,
                          a_scale_inv=dev_scalar(sa), b_scale_inv=dev_scalar(sb), sumsq=i != 1,
                          D=torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda"),
                          sa=sa, sb=sb, Ah=u8(A), Bh=u8(B)))
    descs = [{k: v for k, v in p.items() if k not in ("sa", "sb", "Ah", "Bh")} for p in probs]
    ws = torch.zeros(cuda_lib.fp8_gemm_sumsq_workspace_bytes(descs), dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    cuda_lib.fp8_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    first = out.item()
    for p in probs:
        R, ab = oracle.gemm(p["Ah"], p["a_fmt"], p["Bh"], p["b_fmt"], p["sa"], p["sb"], want_abs=True)
        ok = gemm_within_tolerance(bf16_bits(p["D"]), R, ab)
        assert ok.all(), f"{(~ok).sum()} of {ok.size} outside tolerance"
    squares = np.concatenate([np.square(f32(p["D"].float()).astype(np.float64)).reshape(-1)
                              for p in probs if p["sumsq"]])
    exact = float(np.sum(np.sort(squares)))
    assert abs(first - exact) <= 1e-13 * exact
    assert not ws[:8].any()
    cuda_lib.fp8_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    assert np.float64(out.item()).view(np.uint64) == np.float64(first).view(np.uint64)


def tile_samples(M, N, per_tile, seed):
    """per_tile positions inside every 256 x 512 output tile (so split tiles are always hit)."""
    rng = np.random.default_rng(seed)
    ti, tj = np.meshgrid(np.arange(-(-M // 256)), np.arange(-(-N // 512)), indexing="ij")
    ti, tj = np.repeat(ti.reshape(-1), per_tile), np.repeat(tj.reshape(-1), per_tile)
    ii = np.minimum(ti * 256 + rng.integers(0, 256, ti.size), M - 1)
    jj = np.minimum(tj * 512 + rng.integers(0, 512, tj.size), N - 1)
    return ii, jj


def test_step_gemms_summed_full_size_every_tile_sampled(cuda_lib):
    """The 4096-class step's three GEMMs as the step issues them with the wgrad sum of squares
    (fp8_gemm_multi_sumsq): the schedule gives some clusters 256-column halves of tiles, so
    eight outputs of every 256 x 512 tile of every problem are checked against the oracle, and
    the sum of squares against numpy's over the whole of dW. A second call with other X codes
    gives the same agreement (nothing carried over from the first)."""
    T, fin, fout = 8192, 4096, 4096
    Wq = random_codes(fin, fout, oracle.E4M3, 2)
    dYq = random_codes(T, fout, oracle.E5M2, 3)
    s = [dev_scalar(v) for v in (0.011, 0.023, 0.5)]
    Y = torch.empty(T, fout, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(T, fin, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(fin, fout, dtype=torch.bfloat16, device="cuda")
    ws, out = None, torch.zeros(1, dtype=torch.float64, device="cuda")
    hW, hdY = u8(Wq), u8(dYq)
    for call, xseed in enumerate((1, 11)):
        Xq = random_codes(T, fin, oracle.E4M3, xseed)
        descs = [
            dict(A=Xq, a_fmt=0, B=Wq, b_mn=True, b_fmt=0, a_scale_inv=s[0], b_scale_inv=s[1], D=Y),
            dict(A=dYq, a_fmt=1, B=Wq, b_fmt=0, a_scale_inv=s[2], b_scale_inv=s[1], D=dX),
            dict(A=Xq, a_mn=True, a_fmt=0, B=dYq, b_mn=True, b_fmt=1, a_scale_inv=s[0],
                 b_scale_inv=s[2], D=dW, sumsq=True)]
        if ws is None:
            ws = torch.zeros(cuda_lib.fp8_gemm_sumsq_workspace_bytes(descs), dtype=torch.uint8,
                             device="cuda")
        cuda_lib.fp8_gemm_multi_sumsq(descs, out, ws)
        cuda_lib.fp8t_check_device_error()
        hX = u8(Xq)
        for D, A, af, B, bf, sa, sb in ((Y, hX, 0, hW.T, 0, 0.011, 0.023), (dX, hdY, 1, hW, 0, 0.5, 0.023),
                                        (dW, hX.T, 0, hdY.T, 1, 0.011, 0.5)):
            ii, jj = tile_samples(D.shape[0], D.shape[1], 8, seed=D.shape[1] + call)
            R, ab = oracle.gemm_at(np.ascontiguousarray(A), af, np.ascontiguousarray(B), bf, sa, sb, ii, jj)
            ok = gemm_within_tolerance(bf16_bits(D)[ii, jj], R, ab)
            assert ok.all(), f"call {call}: {(~ok).sum()} of {ok.size} outside tolerance"
        sq = np.square(f32(dW.float()).astype(np.float64)).reshape(-1)
        exact = float(np.sum(np.sort(sq)))
        assert abs(out.item() - exact) <= 1e-13 * exact
        assert ws[:8].view(torch.int32).eq(0).all()
