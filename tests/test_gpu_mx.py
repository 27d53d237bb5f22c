"""MXFP8 through the C ABI against the oracle ("FP8 混合精度训练工程实践" §九: 32 values share one
E8M0 scale, each stored as FP8; §三: micro scaling with E4M3 elements).

The cast's codes and scales are compared bit for bit in both orientations (scales converted from
the 512-byte atom order the tensor cores read to a plain [rows, blocks] array); the block-scaled
GEMM within the GEMM tolerance (2 BF16 ulp + 1e-5 of the sum of |a b 2^(Xa+Xb)|) on full outputs
of small problems in every operand layout and on sampled outputs of the 4096-class shapes."""
import numpy as np
import pytest
import torch

import oracle
from optimizer_fp8_cast_b200 import synth
from tests._gpu import bf16_bits, bf16_from_bits, sample_positions, u8
from tests._pins import gemm_within_tolerance

pytestmark = pytest.mark.gpu


def from_atoms(atoms, mn, k):
    """Atom-ordered scales (bytes of [mn/128][k/128][512]) -> plain [mn, k/32]."""
    a = u8(atoms).reshape(mn // 128, k // 128, 32, 4, 4)      # [mb][kb4][i%32][i/32][kb]
    return np.ascontiguousarray(a.transpose(0, 3, 2, 1, 4).reshape(mn, k // 32))


def to_atoms(plain):
    mn, kk = plain.shape
    a = plain.reshape(mn // 128, 4, 32, kk // 4, 4).transpose(0, 3, 2, 1, 4)
    return torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()


def mx_cast(fp8, x_bits, fmt):
    rows, cols = x_bits.shape
    x = bf16_from_bits(x_bits)
    qr = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    qc = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    sr = torch.empty(fp8.mx_scale_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    sc = torch.empty(fp8.mx_scale_bytes(cols, rows), dtype=torch.uint8, device="cuda")
    fp8.fp8_mx_cast_multi([dict(x=x, fmt=fmt, q_row=qr, sf_row=sr, q_col=qc, sf_col=sc)])
    fp8.fp8t_check_device_error()
    return qr, sr, qc, sc


def check_cast(fp8, x_bits, fmt):
    rows, cols = x_bits.shape
    qr, sr, qc, sc = mx_cast(fp8, x_bits, fmt)
    rq, rs = oracle.mx_quantise(x_bits, 0, fmt)
    assert np.array_equal(u8(qr), rq) and np.array_equal(from_atoms(sr, rows, cols), rs)
    cq, cs = oracle.mx_quantise(x_bits, 1, fmt)                  # cs: [rows/32, cols]
    assert np.array_equal(u8(qc), cq) and np.array_equal(from_atoms(sc, cols, rows), cs.T)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("shape", [(128, 128), (256, 384), (1024, 512)])
def test_mx_cast_random_and_special(cuda_lib, fmt, shape):
    rng = np.random.default_rng(shape[0] + shape[1] + fmt)
    x = (rng.standard_normal(shape) * 10.0 ** rng.uniform(-30, 30, (shape[0], 1))).astype(np.float32)
    x[0, :32] = 0.0                                              # a zero block
    x[1, 5] = np.nan                                             # a NaN block
    x[2, 40] = np.inf                                            # an infinite amax
    x[3, 64:96] = 3e-41                                          # subnormal BF16 values
    x[:32, 100] = -0.0
    check_cast(cuda_lib, bf16_bits(torch.from_numpy(x).to(torch.bfloat16)), fmt)


def test_mx_cast_every_bf16_pattern(cuda_lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(256, 256)
    for fmt in (oracle.E4M3, oracle.E5M2):
        check_cast(cuda_lib, bits, fmt)
        check_cast(cuda_lib, np.ascontiguousarray(bits.T), fmt)


def test_mx_cast_full_size(cuda_lib):
    wl = synth.LINEAR4096
    X, dY = synth.linear_inputs(wl, 0, 0, "cuda")
    check_cast(cuda_lib, bf16_bits(X), oracle.E4M3)
    check_cast(cuda_lib, bf16_bits(dY), oracle.E4M3)


def mx_operands(rows, cols, fmt, seed, spread=8.0):
    """Codes and plain scales (both orientations) of a random matrix with varied block ranges."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, cols)) * 2.0 ** rng.uniform(-spread, spread, (rows, 1))
         * 2.0 ** rng.uniform(-spread, spread, (1, cols))).astype(np.float32)
    bits = bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    return oracle.mx_quantise(bits, 0, fmt), oracle.mx_quantise(bits, 1, fmt)


@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (False, True), (True, False), (True, True)])
@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (256, 256, 256), (384, 640, 512),
                                   (256, 512, 256), (128, 896, 384), (256, 1152, 128)])
def test_mx_gemm_small_full(cuda_lib, a_mn, b_mn, M, N, K):
    """Every output against the oracle. N < 512 runs the 256 x 256 kernel; N >= 512 the 256 x 384
    one, whose last column tile may have no rows for its N = 128 MMA (640, 896: 256 and 128 rows
    left) or only part of its N = 256 MMA's rows (512, 896), and 1152 = 3 x 384 has no such tile."""
    for bf in (oracle.E4M3, oracle.E5M2):
        (qa_r, sa_r), (qa_c, sa_c) = mx_operands(M, K, oracle.E4M3, M + K) if not a_mn else \
            mx_operands(K, M, oracle.E4M3, M + K)
        (qb_r, sb_r), (qb_c, sb_c) = mx_operands(N, K, bf, N + K + bf) if not b_mn else \
            mx_operands(K, N, bf, N + K + bf)
        # logical A [M, K] with K-contiguous plain scales [M, K/32] for the oracle
        if a_mn:                        # stored [K, M], blocks down columns (K)
            A_dev, A_log, sa_log = qa_c, qa_c.T, sa_c.T
        else:
            A_dev, A_log, sa_log = qa_r, qa_r, sa_r
        if b_mn:
            B_dev, B_log, sb_log = qb_c, qb_c.T, sb_c.T
        else:
            B_dev, B_log, sb_log = qb_r, qb_r, sb_r
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        cuda_lib.fp8_mx_gemm_multi([dict(A=torch.from_numpy(np.ascontiguousarray(A_dev)).cuda(), a_mn=a_mn,
                                         a_sf=to_atoms(np.ascontiguousarray(sa_log)), a_fmt=oracle.E4M3,
                                         B=torch.from_numpy(np.ascontiguousarray(B_dev)).cuda(), b_mn=b_mn,
                                         b_sf=to_atoms(np.ascontiguousarray(sb_log)), b_fmt=bf, D=D)])
        cuda_lib.fp8t_check_device_error()
        R, ab = oracle.mx_gemm(A_log, sa_log, oracle.E4M3, B_log, sb_log, bf, want_abs=True)
        ok = gemm_within_tolerance(bf16_bits(D), R, ab)
        assert ok.all(), f"{(~ok).sum()} of {ok.size} outside tolerance (b fmt {bf})"


def test_mx_step_gemms_full_size_sampled(cuda_lib):
    """The three GEMMs of the 4096 x 4096 / 8192-token Linear as an MXFP8 step issues them
    (E4M3 everywhere): fprop Xq_row x Wq_col, dgrad dYq_row x Wq_row, wgrad Xq_col x dYq_col,
    with codes and scales from the library's MX cast, in one grouped launch; 4096 sampled outputs
    each against the oracle."""
    wl = synth.LINEAR4096
    X, dY = synth.linear_inputs(wl, 0, 0, "cuda")
    W = synth.linear_weight(wl, 0, "cuda")
    T, fin, fout = 8192, 4096, 4096
    xq = mx_cast(cuda_lib, bf16_bits(X), oracle.E4M3)
    wq = mx_cast(cuda_lib, bf16_bits(W), oracle.E4M3)
    dq = mx_cast(cuda_lib, bf16_bits(dY), oracle.E4M3)
    Y = torch.empty(T, fout, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(T, fin, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(fin, fout, dtype=torch.bfloat16, device="cuda")
    E = oracle.E4M3
    cuda_lib.fp8_mx_gemm_multi([
        dict(A=xq[0], a_sf=xq[1], a_fmt=E, B=wq[2], b_sf=wq[3], b_mn=True, b_fmt=E, D=Y),
        dict(A=dq[0], a_sf=dq[1], a_fmt=E, B=wq[0], b_sf=wq[1], b_fmt=E, D=dX),
        dict(A=xq[2], a_sf=xq[3], a_mn=True, a_fmt=E, B=dq[2], b_sf=dq[3], b_mn=True, b_fmt=E, D=dW)])
    cuda_lib.fp8t_check_device_error()
    hx_r, hx_sr, hx_c, hx_sc = u8(xq[0]), from_atoms(xq[1], T, fin), u8(xq[2]), from_atoms(xq[3], fin, T)
    hw_r, hw_sr, hw_c, hw_sc = u8(wq[0]), from_atoms(wq[1], fin, fout), u8(wq[2]), from_atoms(wq[3], fout, fin)
    hd_r, hd_sr, hd_c, hd_sc = u8(dq[0]), from_atoms(dq[1], T, fout), u8(dq[2]), from_atoms(dq[3], fout, T)
    for D, A, sa, B, sb in ((Y, hx_r, hx_sr, hw_c.T, hw_sc), (dX, hd_r, hd_sr, hw_r, hw_sr),
                            (dW, hx_c.T, hx_sc, hd_c.T, hd_sc)):
        ii, jj = sample_positions(D.shape[0], D.shape[1], 4096, seed=D.shape[0] + 7)
        R, ab = oracle.mx_gemm_at(np.ascontiguousarray(A), sa, E, np.ascontiguousarray(B), sb, E, ii, jj)
        assert gemm_within_tolerance(bf16_bits(D)[ii, jj], R, ab).all()


@pytest.mark.parametrize("shapes", [[(256, 768, 512), (384, 512, 256), (256, 1152, 384)],
                                    [(256, 256, 512), (128, 384, 256)]])
def test_mx_gemm_sum_of_squares(cuda_lib, shapes):
    """fp8_mx_gemm_multi_sumsq: the first list runs the 256 x 384 kernel (every N >= 512), the
    second the 256 x 256 one. Every output against the oracle, the FP64 sum of f32(D)^2 over the
    flagged problems against numpy's, a repeat with identical bits, the workspace left at zero."""
    probs = []
    for i, (M, N, K) in enumerate(shapes):
        a_mn, b_mn = bool(i % 2), bool((i // 2) % 2) or i == 0
        (qa_r, sa_r), (qa_c, sa_c) = mx_operands(M, K, oracle.E4M3, 900 + i) if not a_mn else \
            mx_operands(K, M, oracle.E4M3, 900 + i)
        (qb_r, sb_r), (qb_c, sb_c) = mx_operands(N, K, oracle.E4M3, 950 + i) if not b_mn else \
            mx_operands(K, N, oracle.E4M3, 950 + i)
        A_dev, A_log, sa_log = (qa_c, qa_c.T, sa_c.T) if a_mn else (qa_r, qa_r, sa_r)
        B_dev, B_log, sb_log = (qb_c, qb_c.T, sb_c.T) if b_mn else (qb_r, qb_r, sb_r)
        probs.append(dict(
            desc=dict(A=torch.from_numpy(np.ascontiguousarray(A_dev)).cuda(), a_mn=a_mn,
                      a_sf=to_atoms(np.ascontiguousarray(sa_log)), a_fmt=oracle.E4M3,
                      B=torch.from_numpy(np.ascontiguousarray(B_dev)).cuda(), b_mn=b_mn,
                      b_sf=to_atoms(np.ascontiguousarray(sb_log)), b_fmt=oracle.E4M3, sumsq=i != 1,
                      D=torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")),
            ref=(A_log, sa_log, B_log, sb_log)))
    descs = [p["desc"] for p in probs]
    ws = torch.zeros(cuda_lib.fp8_mx_gemm_sumsq_workspace_bytes(descs), dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    cuda_lib.fp8_mx_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    first = out.item()
    for p in probs:
        A_log, sa_log, B_log, sb_log = p["ref"]
        R, ab = oracle.mx_gemm(A_log, sa_log, oracle.E4M3, B_log, sb_log, oracle.E4M3, want_abs=True)
        ok = gemm_within_tolerance(bf16_bits(p["desc"]["D"]), R, ab)
        assert ok.all(), f"{(~ok).sum()} of {ok.size} outside tolerance"
    squares = np.concatenate([np.square(p["desc"]["D"].float().cpu().numpy().astype(np.float64)).reshape(-1)
                              for p in probs if p["desc"]["sumsq"]])
    exact = float(np.sum(np.sort(squares)))
    assert abs(first - exact) <= 1e-13 * exact
    assert not ws[:8].any()
    cuda_lib.fp8_mx_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    assert np.float64(out.item()).view(np.uint64) == np.float64(first).view(np.uint64)


def test_mx_grouped_launch_7b_block_shapes_sampled(cuda_lib):
    """One block-scaled launch with the fprop, dgrad and wgrad of three 7B-block projections
    (q 4096 -> 4096, gate 4096 -> 11008, down 11008 -> 4096) at 256 tokens: nine problems with
    4096- and 11008-wide outputs (11008 leaves a column tile with no rows for the N = 128 MMA) and
    K of 256, 4096 and 11008, codes and scales from the library's MX cast. 1024 sampled outputs of
    each against the oracle, and the sum of squares of the three wgrad outputs against numpy's."""
    T, E = 256, oracle.E4M3
    layers = [(4096, 4096), (4096, 11008), (11008, 4096)]
    gen = torch.Generator(device="cuda").manual_seed(77)
    descs, refs = [], []
    for li, (fin, fout) in enumerate(layers):
        X = (torch.randn(T, fin, generator=gen, device="cuda") * 2).to(torch.bfloat16)
        W = (torch.randn(fin, fout, generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
        dY = (torch.randn(T, fout, generator=gen, device="cuda") * 1e-3).to(torch.bfloat16)
        xq, wq, dq = (mx_cast(cuda_lib, bf16_bits(t), E) for t in (X, W, dY))
        Y = torch.empty(T, fout, dtype=torch.bfloat16, device="cuda")
        dX = torch.empty(T, fin, dtype=torch.bfloat16, device="cuda")
        dW = torch.empty(fin, fout, dtype=torch.bfloat16, device="cuda")
        descs += [dict(A=xq[0], a_sf=xq[1], a_fmt=E, B=wq[2], b_sf=wq[3], b_mn=True, b_fmt=E, D=Y),
                  dict(A=dq[0], a_sf=dq[1], a_fmt=E, B=wq[0], b_sf=wq[1], b_fmt=E, D=dX),
                  dict(A=xq[2], a_sf=xq[3], a_mn=True, a_fmt=E, B=dq[2], b_sf=dq[3], b_mn=True,
                       b_fmt=E, D=dW, sumsq=True)]
        hx = (u8(xq[0]), from_atoms(xq[1], T, fin), u8(xq[2]), from_atoms(xq[3], fin, T))
        hw = (u8(wq[0]), from_atoms(wq[1], fin, fout), u8(wq[2]), from_atoms(wq[3], fout, fin))
        hd = (u8(dq[0]), from_atoms(dq[1], T, fout), u8(dq[2]), from_atoms(dq[3], fout, T))
        refs += [(Y, hx[0], hx[1], hw[2].T, hw[3]), (dX, hd[0], hd[1], hw[0], hw[1]),
                 (dW, hx[2].T, hx[3], hd[2].T, hd[3])]
    ws = torch.zeros(cuda_lib.fp8_mx_gemm_sumsq_workspace_bytes(descs), dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    cuda_lib.fp8_mx_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    for k, (D, A, sa, B, sb) in enumerate(refs):
        ii, jj = sample_positions(D.shape[0], D.shape[1], 1024, seed=300 + k)
        R, ab = oracle.mx_gemm_at(np.ascontiguousarray(A), sa, E, np.ascontiguousarray(B), sb, E, ii, jj)
        assert gemm_within_tolerance(bf16_bits(D)[ii, jj], R, ab).all(), f"problem {k}"
    squares = np.concatenate([np.square(d["D"].float().cpu().numpy().astype(np.float64)).reshape(-1)
                              for d in descs if d.get("sumsq")])
    exact = float(np.sum(np.sort(squares)))
    assert abs(out.item() - exact) <= 1e-13 * exact and not ws[:8].any()


@pytest.mark.parametrize("wide", [True, False], ids=["256x384-tiles", "256x256-tiles"])
def test_mx_gemm_26_problems_two_launches_with_sum_of_squares(cuda_lib, wide):
    """26 block-scaled problems are more than one launch table holds: two launches share one sum
    of squares (slots numbered over the call, the second launch reduces them). Every output
    against the oracle, the sum against numpy's, the workspace left at zero."""
    shapes = [(128, 512, 256), (256, 640, 128), (128, 1152, 128)] if wide else \
             [(128, 512, 256), (256, 256, 128), (128, 384, 128)]
    descs, refs = [], []
    for i in range(26):
        M, N, K = shapes[i % 3]
        (qa, sa), _ = mx_operands(M, K, oracle.E4M3, 1300 + i)
        (qb, sb), _ = mx_operands(N, K, oracle.E4M3, 1400 + i)
        descs.append(dict(A=torch.from_numpy(qa).cuda(), a_sf=to_atoms(sa), a_fmt=oracle.E4M3,
                          B=torch.from_numpy(qb).cuda(), b_sf=to_atoms(sb), b_fmt=oracle.E4M3,
                          sumsq=(i % 3 == 1) or i == 25,
                          D=torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")))
        refs.append((qa, sa, qb, sb))
    ws = torch.zeros(cuda_lib.fp8_mx_gemm_sumsq_workspace_bytes(descs), dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    cuda_lib.fp8_mx_gemm_multi_sumsq(descs, out, ws)
    cuda_lib.fp8t_check_device_error()
    for d, (qa, sa, qb, sb) in zip(descs, refs):
        R, ab = oracle.mx_gemm(qa, sa, oracle.E4M3, qb, sb, oracle.E4M3, want_abs=True)
        assert gemm_within_tolerance(bf16_bits(d["D"]), R, ab).all()
    squares = np.concatenate([np.square(d["D"].float().cpu().numpy().astype(np.float64)).reshape(-1)
                              for d in descs if d["sumsq"]])
    exact = float(np.sum(np.sort(squares)))
    assert abs(out.item() - exact) <= 1e-13 * exact and not ws[:8].any()
