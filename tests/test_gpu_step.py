"""Whole training steps through the C ABI, checked stage by stage against the oracle with
teacher forcing (each stage's oracle input is the GPU's actual input, so GEMM rounding never
leaks into the bit-exact checks of later casts, amax, scales and history).

Workloads: the 256 x 256 / 512-token Linear for 3 steps (every output compared in full), the
1024 x 1024 / 2048-token stress run with an x1000 batch at step 20 swept over history length,
algorithm and margin (saturation and zero counts per tensor per step), and one step of the seven
7B-block projections at 16,384 tokens (sampled GEMM outputs, full casts and AdamW samples).

[P2] "FP8 混合精度训练工程实践" §四 (precision flow of a step); [P3] "LLM FP8 微调上线生产实战"
核心原理 (delayed scaling) and 第四步 (per-tensor saturation / zero metrics)."""
import numpy as np
import pytest
import torch

import oracle
from optimizer_fp8_cast_b200 import synth
from optimizer_fp8_cast_b200.step import Fp8LinearStep
from tests._gpu import bf16_bits, f32, sample_positions, u8
from tests._pins import gemm_within_tolerance, ulp_distance_f32

pytestmark = pytest.mark.gpu
FMT = (oracle.E4M3, oracle.E4M3, oracle.E5M2)


def make_step(wl, algo=None, margin=None, H=None, counters=True, fused=True, transposes=False,
              side=False):
    """fused: scale update in the cast launch, dW sum of squares in the wgrad epilogue and (when
    no counters are kept) the next W cast inside AdamW; False: every stage its own launch.
    transposes: the casts also write q^T and the GEMMs read K-major operands only.
    side: the scale update as its own launch on a second stream, beside the GEMMs."""
    w0 = [synth.linear_weight(wl, k, "cuda") for k in range(len(wl.layers))]
    return Fp8LinearStep([(i, o) for _, i, o in wl.layers], wl.tokens,
                         H or wl.history_len, algo or wl.algo,
                         wl.margin if margin is None else margin, wl.adamw, w0, "cuda",
                         counters=counters, fused_update=fused, fused_norm=fused, fused_wcast=fused,
                         transposes=transposes, side_update=side)


def tr(q):
    return np.ascontiguousarray(q.T)


def snapshot(st):
    return dict(scale=f32(st.scale), hist=f32(st.history),
                W=[bf16_bits(l.W) for l in st.layers], master=[f32(l.master) for l in st.layers],
                Wq=[u8(l.Wq) for l in st.layers],
                WqT=[u8(l.WqT) if l.WqT is not None else tr(u8(l.Wq)) for l in st.layers],
                m=[f32(l.m) for l in st.layers], v=[f32(l.v) for l in st.layers],
                counters=st.counters.cpu().numpy().astype(np.uint64).copy() if st.counters is not None else None)


def check_step(st, pre, xs, dys, gemm_full=True, gemm_samples=2048, cast_check=True):
    """Compare everything one step produced with the oracle fed the same inputs."""
    n = 3 * len(st.layers)
    amax_ref = np.zeros(n, np.float32)
    cnt_ref = pre["counters"].copy() if pre["counters"] is not None else None
    sinv_used = np.array([np.float32(1.0) / np.float32(s) for s in pre["scale"]], np.float32)
    for k, L in enumerate(st.layers):
        srcs = (bf16_bits(xs[k]), pre["W"][k], bf16_bits(dys[k]))
        # the W codes this step's GEMMs read: cast during the previous AdamW when fused
        # (without transposed copies on the device, q^T below is the host transpose of q; the
        # GEMMs then read q MN-major)
        both = lambda q, qT: (u8(q), u8(qT) if qT is not None else tr(u8(q)))
        wq = (pre["Wq"][k], pre["WqT"][k]) if st.fused_wcast else both(L.Wq, L.WqT)
        outs = (both(L.Xq, L.XqT), wq, both(L.dYq, L.dYqT))
        for r in range(3):
            i = 3 * k + r
            if cast_check:
                q, qT, a, si, c = oracle.cast_transpose_amax(srcs[r], FMT[r], pre["scale"][i])
                assert np.array_equal(outs[r][0], q), f"layer {k} role {r} codes"
                assert np.array_equal(outs[r][1], qT), f"layer {k} role {r} transposed"
                if cnt_ref is not None:
                    cnt_ref[i] += c
            else:
                _, _, a, si, _ = oracle.cast_transpose_amax(srcs[r], FMT[r], pre["scale"][i], False, False)
            amax_ref[i] = a
        sx, sw, sdy = sinv_used[3 * k], sinv_used[3 * k + 1], sinv_used[3 * k + 2]
        (Xq, XqT), (Wq, WqT), (dYq, dYqT) = outs
        gemms = ((Xq, 0, WqT, 0, sx, sw, L.Y), (dYq, 1, Wq, 0, sdy, sw, L.dX),
                 (XqT, 0, dYqT, 1, sx, sdy, L.dW))
        for Ah, af, Bh, bf, sa, sb, D in gemms:
            Dh = bf16_bits(D)
            if gemm_full:
                R, ab = oracle.gemm(Ah, af, Bh, bf, sa, sb, want_abs=True)
                assert gemm_within_tolerance(Dh, R, ab).all()
            else:
                ii, jj = sample_positions(Dh.shape[0], Dh.shape[1], gemm_samples, seed=k)
                R, ab = oracle.gemm_at(Ah, af, Bh, bf, sa, sb, ii, jj)
                assert gemm_within_tolerance(Dh[ii, jj], R, ab).all()
    # amax (entry 0 of each history row) and the scale update; consumed amax slots are reset
    assert np.array_equal(f32(st.history)[:, 0].view(np.uint32), amax_ref.view(np.uint32))
    if not st.fused_wcast:
        assert not st.amax.any().item()
    hist, scale = pre["hist"].copy(), pre["scale"].copy()
    sinv = np.zeros_like(scale)
    oracle.scale_update(amax_ref, hist, f32(st.fp8_max), st.algo, st.margin, scale, sinv)
    assert np.array_equal(f32(st.history).view(np.uint32), hist.view(np.uint32))
    assert np.array_equal(f32(st.scale).view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(f32(st.scale_inv).view(np.uint32), sinv.view(np.uint32))
    if st.fused_wcast:                     # W's inverse scale is already the next step's
        for k in range(len(st.layers)):
            sinv_used[3 * k + 1] = np.float32(1.0) / scale[3 * k + 1]
    assert np.array_equal(f32(st.sinv_used).view(np.uint32), sinv_used.view(np.uint32))
    assert st.ticket.item() == 0 and st.adamw_ticket.item() == 0
    if cnt_ref is not None and cast_check:
        assert np.array_equal(st.counters.cpu().numpy().astype(np.uint64), cnt_ref)
    # AdamW on the GPU's own dW
    dW = [bf16_bits(l.dW) for l in st.layers]
    P, M, V = pre["master"], pre["m"], pre["v"]
    Wref = [np.zeros(p.size, np.uint16) for p in P]
    hp = dict(st.hp, step=st.t)
    rnorm, rskip = oracle.fused_adamw([p.reshape(-1) for p in P], [m.reshape(-1) for m in M],
                                      [v.reshape(-1) for v in V], [d.reshape(-1) for d in dW],
                                      Wref, hp)
    assert st.skipped.item() == rskip
    assert ulp_distance_f32(np.float32(st.grad_norm.item()), np.float32(rnorm)) <= 2
    for k, L in enumerate(st.layers):
        for got, ref in ((L.master, P[k]), (L.m, M[k]), (L.v, V[k])):
            assert ulp_distance_f32(f32(got).reshape(-1), ref.reshape(-1)).max() <= 4
        wg = bf16_bits(L.W).reshape(-1)
        assert np.abs(wg.astype(np.int32) - Wref[k].astype(np.int32)).max() <= 1
        if st.fused_wcast:
            # AdamW cast the new weight with the next step's scale: codes, amax slot
            i = 3 * k + 1
            q, qT, a, _, _ = oracle.cast_transpose_amax(bf16_bits(L.W), oracle.E4M3, scale[i],
                                                         cast_check, cast_check)
            if cast_check:
                assert np.array_equal(u8(L.Wq), q)
                assert L.WqT is None or np.array_equal(u8(L.WqT), qT)
            assert np.float32(st.amax[i].item()).view(np.uint32) == np.float32(a).view(np.uint32)
            assert st.amax[3 * k].item() == 0 and st.amax[3 * k + 2].item() == 0


def _optimizer_state(st):
    return [(f32(l.master).reshape(-1).copy(), f32(l.m).reshape(-1).copy(),
             f32(l.v).reshape(-1).copy()) for l in st.layers]


def _check_adamw_on_gpu_grad(st, pre_opt, t):
    """AdamW of step t as the oracle computes it from the optimizer state before the step and the
    GPU's own dW ("算子与编译器" Fused Optimizer 的意义: the update's order and content)."""
    P = [p.copy() for p, _, _ in pre_opt]
    M = [m.copy() for _, m, _ in pre_opt]
    V = [v.copy() for _, _, v in pre_opt]
    Wref = [np.zeros(p.size, np.uint16) for p in P]
    rnorm, rskip = oracle.fused_adamw(P, M, V, [bf16_bits(l.dW).reshape(-1) for l in st.layers],
                                      Wref, dict(st.hp, step=t))
    assert st.skipped.item() == rskip == 0
    assert ulp_distance_f32(np.float32(st.grad_norm.item()), np.float32(rnorm)) <= 2
    for k, L in enumerate(st.layers):
        for got, ref in ((L.master, P[k]), (L.m, M[k]), (L.v, V[k])):
            assert ulp_distance_f32(f32(got).reshape(-1), ref).max() <= 4
        wg = bf16_bits(L.W).reshape(-1).astype(np.int32)
        assert np.abs(wg - Wref[k].astype(np.int32)).max() <= 1


@pytest.mark.parametrize("fused,counters,transposes,side",
                         [(True, False, False, False), (True, False, False, True),
                          (True, True, False, False), (False, True, False, False),
                          (True, False, True, False), (False, True, True, False)],
                         ids=["all-fused", "side-update", "fused-with-counters", "separate-launches",
                              "all-fused-transposes", "separate-launches-transposes"])
def test_linear256_three_steps(cuda_lib, fused, counters, transposes, side):
    """Three steps in full. all-fused: scale update in the cast launch, dW sum of squares in the
    wgrad epilogue, next W cast in AdamW (three launches per step); side-update: the same with
    the scale update as its own launch on a second stream beside the GEMMs; with counters the W
    cast stays in the cast launch; separate-launches: every stage its own kernel. Without
    transposes the GEMMs read Xq, Wq, dYq MN-major where needed; with them, the K-major
    transposed copies."""
    wl = synth.LINEAR256
    st = make_step(wl, fused=fused, counters=counters, transposes=transposes, side=side)
    assert st.fused_wcast == (fused and not counters and not transposes)
    assert st.side_update == side and st.kernels_per_step() == (4 if side else 3 if fused else 5)
    for t in range(wl.steps):
        xs, dys = zip(*[synth.linear_inputs(wl, k, t, "cuda") for k in range(len(wl.layers))])
        pre = snapshot(st)
        st.step(xs, dys)
        cuda_lib.fp8t_check_device_error()
        check_step(st, pre, xs, dys)


@pytest.mark.parametrize("side", [False, True], ids=["update-in-cast", "side-update"])
def test_linear256_step_in_cuda_graph(cuda_lib, side):
    """The whole step captured once into a CUDA graph (device step counter; with side-update the
    graph forks the scale update onto a second stream and joins it before AdamW) and replayed
    three times; after every replay each stage is compared with the oracle fed the same inputs:
    casts, scales and history bit for bit, GEMMs within tolerance, AdamW within 4 ulp with the
    oracle's host bias corrections for t = 1, 2, 3 (the graph forms them on the device)."""
    wl = synth.LINEAR256
    xs, dys = zip(*[synth.linear_inputs(wl, k, 0, "cuda") for k in range(len(wl.layers))])
    graphed = Fp8LinearStep([(i, o) for _, i, o in wl.layers], wl.tokens, wl.history_len, wl.algo,
                            wl.margin, wl.adamw, [synth.linear_weight(wl, 0, "cuda")], "cuda",
                            device_step=True, side_update=side)
    assert graphed.fused_wcast
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed.step(xs, dys)
    for t in (1, 2, 3):
        pre = snapshot(graphed)
        g.replay()
        torch.cuda.synchronize()
        cuda_lib.fp8t_check_device_error()
        assert graphed.step_counter.item() == t
        graphed.t = t                      # the optimizer step the oracle applies
        check_step(graphed, pre, xs, dys)


@pytest.mark.parametrize("H,algo,margin", synth.STRESS_SWEEP)
def test_stress1024_sweep(cuda_lib, H, algo, margin):
    """50 steps with an x1000 X batch at step 20. Every step: amax, scales, history and the
    per-tensor saturation / zero / non-finite counters bit-exact (casts checked in full at the
    steps around the spike and at the ends, GEMMs sampled)."""
    wl = synth.STRESS1024
    st = make_step(wl, algo=algo, margin=margin, H=H)
    full_cast_steps = {0, 1, 19, 20, 21, 22, 49}
    sat_x = []
    for t in range(wl.steps):
        xs, dys = zip(*[synth.linear_inputs(wl, 0, t, "cuda")])
        pre = snapshot(st)
        st.counters.zero_()
        pre["counters"] = np.zeros_like(pre["counters"])
        st.step(xs, dys)
        cuda_lib.fp8t_check_device_error()
        check_step(st, pre, xs, dys, gemm_full=False, gemm_samples=256,
                   cast_check=t in full_cast_steps)
        sat_x.append(int(st.counters[0, 0].item()))
    # the spike saturates X at step 20: its scale still comes from the history before it
    assert sat_x[20] > sat_x[19]


def test_block7b_one_step(cuda_lib):
    """One step of the seven 7B-block projections (q, k, v, o, gate, up, down) at 16,384 tokens;
    casts, amax, scales and AdamW in full, GEMMs on sampled outputs."""
    wl = synth.BLOCK7B
    free, _ = torch.cuda.mem_get_info()
    if free < 40e9:
        pytest.skip("needs ~30 GB of free device memory")
    st = make_step(wl, counters=False)
    xs, dys = zip(*[synth.linear_inputs(wl, k, 0, "cuda") for k in range(len(wl.layers))])
    pre = snapshot(st)
    st.step(xs, dys)
    cuda_lib.fp8t_check_device_error()
    check_step(st, pre, xs, dys, gemm_full=False, gemm_samples=1024)


def test_host_streamed_steps_match_eager(cuda_lib):
    """Three steps fed from pinned host memory through the overlapped runner give bit for bit
    the Y, dX and weights of three eager steps on device-resident copies of the same inputs."""
    from optimizer_fp8_cast_b200.host_stream import HostStreamedStep
    wl = synth.LINEAR256
    inputs = [synth.linear_inputs(wl, 0, t, "cpu") for t in range(3)]
    eager = make_step(wl, counters=False)
    ref = []
    for X, dY in inputs:
        eager.step([X.cuda()], [dY.cuda()])
        ref.append((eager.layers[0].Y.cpu(), eager.layers[0].dX.cpu()))
    streamed = make_step(wl, counters=False)
    runner = HostStreamedStep(streamed)
    outs = []
    for X, dY in inputs:
        hy = torch.empty(wl.tokens, 256, dtype=torch.bfloat16).pin_memory()
        hdx = torch.empty(wl.tokens, 256, dtype=torch.bfloat16).pin_memory()
        runner.step([X.pin_memory()], [dY.pin_memory()], [hy], [hdx])
        outs.append((hy, hdx))
    runner.finish()
    cuda_lib.fp8t_check_device_error()
    for (ry, rdx), (gy, gdx) in zip(ref, outs):
        assert torch.equal(ry.view(torch.int16), gy.view(torch.int16))
        assert torch.equal(rdx.view(torch.int16), gdx.view(torch.int16))
    assert torch.equal(eager.layers[0].W.view(torch.int16), streamed.layers[0].W.view(torch.int16))
    assert torch.equal(eager.history, streamed.history)


def test_host_streamed_steps_against_the_oracle(cuda_lib):
    """The runner on the step the benchmark times (scale update on a side stream), one step at a
    time so that each step's codes are still on the device: every stage against the oracle fed
    the same inputs (casts, scales and history bit for bit, GEMMs within tolerance, AdamW within
    4 ulp), and the Y and dX that reached host memory equal the device's."""
    from optimizer_fp8_cast_b200.host_stream import HostStreamedStep
    wl = synth.LINEAR256
    st = make_step(wl, counters=False, side=True)
    runner = HostStreamedStep(st)
    for t in range(3):
        X, dY = synth.linear_inputs(wl, 0, t, "cpu")
        hy = torch.empty(wl.tokens, 256, dtype=torch.bfloat16).pin_memory()
        hdx = torch.empty(wl.tokens, 256, dtype=torch.bfloat16).pin_memory()
        pre = snapshot(st)
        runner.step([X.pin_memory()], [dY.pin_memory()], [hy], [hdx])
        runner.finish()
        cuda_lib.fp8t_check_device_error()
        check_step(st, pre, [X.cuda()], [dY.cuda()])
        L = st.layers[0]
        assert torch.equal(hy.view(torch.int16), L.Y.cpu().view(torch.int16))
        assert torch.equal(hdx.view(torch.int16), L.dX.cpu().view(torch.int16))


def test_checkpoint_resume_is_bit_exact(cuda_lib):
    """Six steps straight equal three steps, a save of the full training state (weights,
    master/m/v, amax history, scales, step counters) into a fresh step object, and three more.
    Restoring without the amax history (scales re-warm from 1) gives different casts."""
    wl = synth.LINEAR256
    inputs = [synth.linear_inputs(wl, 0, t, "cuda") for t in range(6)]
    straight = make_step(wl, counters=False)
    for X, dY in inputs:
        straight.step([X], [dY])
    first = make_step(wl, counters=False)
    for X, dY in inputs[:3]:
        first.step([X], [dY])
    sd = first.state_dict()
    resumed = make_step(wl, counters=False)
    resumed.load_state_dict(sd)
    for X, dY in inputs[3:]:
        resumed.step([X], [dY])
    a, b = straight.layers[0], resumed.layers[0]
    for x, y in ((a.W, b.W), (a.master, b.master), (a.m, b.m), (a.v, b.v), (a.Xq, b.Xq), (a.dW, b.dW)):
        assert torch.equal(x.view(torch.uint8) if x.dtype != torch.float32 else x,
                           y.view(torch.uint8) if y.dtype != torch.float32 else y)
    assert torch.equal(straight.history, resumed.history) and torch.equal(straight.scale, resumed.scale)
    # the incident the pages describe: weights and optimizer restored, FP8 scale state not
    broken = make_step(wl, counters=False)
    sd2 = {k: v for k, v in sd.items()}
    broken.load_state_dict(sd2)
    broken.history.zero_(); broken.scale.fill_(1.0); broken.scale_inv.fill_(1.0)
    X, dY = inputs[3]
    broken.step([X], [dY])
    ref = make_step(wl, counters=False)
    ref.load_state_dict(sd)
    ref.step([X], [dY])
    assert not torch.equal(broken.layers[0].Xq, ref.layers[0].Xq)


def test_monitor_flags_the_stress_spike(cuda_lib):
    """The x1000 X batch of the stress run at step 20 is an amax spike for the monitor."""
    from optimizer_fp8_cast_b200.monitor import HealthMonitor
    wl = synth.STRESS1024
    st = make_step(wl, counters=True)
    mon = HealthMonitor(n_tensors=3, every=1, window=9)
    flagged = []
    for t in range(22):
        X, dY = synth.linear_inputs(wl, 0, t, "cuda")
        st.step([X], [dY])
        flagged += [(s, msg) for kind, s, msg in mon.maybe_check(st) if kind == "amax_spike"]
    x_flags = [s for s, msg in flagged if msg.startswith("tensor 0:")]
    assert x_flags == [21]          # the batch of loop index 20 is the step counted t = 21


def test_current_scaling_steps(cuda_lib):
    """Three steps with current scaling: every cast uses the scale its own tensor's amax gives
    (oracle cast_current), fprop, dgrad and wgrad on every output against the oracle GEMM, and
    AdamW (the dW sum of squares from the wgrad epilogue) against oracle fused_adamw on the GPU's
    dW: norm within 2 ulp, master, m, v within 4 ulp, the BF16 weight within one step."""
    wl = synth.LINEAR256
    st = Fp8LinearStep([(256, 256)], wl.tokens, wl.history_len, wl.algo, 1, wl.adamw,
                       [synth.linear_weight(wl, 0, "cuda")], "cuda", recipe="current")
    assert not st.fused_wcast and st.kernels_per_step() == 4
    for t in range(3):
        X, dY = synth.linear_inputs(wl, 0, t, "cuda")
        W0 = bf16_bits(st.layers[0].W)
        scale0 = f32(st.scale).copy()
        pre_opt = _optimizer_state(st)
        st.step([X], [dY])
        cuda_lib.fp8t_check_device_error()
        L = st.layers[0]
        srcs = (bf16_bits(X), W0, bf16_bits(dY))
        for r, (q, src) in enumerate(zip((L.Xq, L.Wq, L.dYq), srcs)):
            rq, _, ra, rs, rsinv, _ = oracle.cast_current(src, FMT[r], 1, scale0[r], True, False)
            assert np.array_equal(u8(q), rq) and np.float32(st.scale[r].item()) == rs
            assert np.float32(st.sinv_used[r].item()) == rsinv and np.float32(st.amax[r].item()) == ra
        sx, sw, sdy = f32(st.sinv_used)
        for D, A, af, B, bf, sa, sb in ((L.Y, u8(L.Xq), 0, tr(u8(L.Wq)), 0, sx, sw),
                                        (L.dX, u8(L.dYq), 1, u8(L.Wq), 0, sdy, sw),
                                        (L.dW, tr(u8(L.Xq)), 0, tr(u8(L.dYq)), 1, sx, sdy)):
            R, ab = oracle.gemm(A, af, B, bf, sa, sb, want_abs=True)
            assert gemm_within_tolerance(bf16_bits(D), R, ab).all()
        _check_adamw_on_gpu_grad(st, pre_opt, t + 1)


@pytest.mark.parametrize("fin,fout,fused_norm", [(256, 256, True), (256, 256, False), (512, 640, True)],
                         ids=["256x256-fused-norm", "256x256-norm-pass", "512x640-fused-norm"])
def test_mxfp8_steps(cuda_lib, fin, fout, fused_norm):
    """Two steps of a Linear (512 tokens) with the MXFP8 recipe: X, W, dY quantised with E4M3
    codes and E8M0 block scales in both orientations (oracle mx_quantise, bit for bit), the three
    block-scaled GEMMs in one launch (oracle mx_gemm on every output; 512 x 640 runs the 256 x 384
    tiles, 256 x 256 the 256 x 256 ones), the sum of dW^2 from the wgrad epilogue (against numpy's)
    or AdamW's norm pass, and AdamW on the GPU's dW (oracle fused_adamw: norm within 2 ulp,
    master, m, v within 4 ulp)."""
    import dataclasses
    from tests.test_gpu_mx import from_atoms
    wl = dataclasses.replace(synth.LINEAR256, layers=[("linear", fin, fout)])
    st = Fp8LinearStep([(fin, fout)], wl.tokens, wl.history_len, wl.algo, 0, wl.adamw,
                       [synth.linear_weight(wl, 0, "cuda")], "cuda", recipe="mxfp8",
                       fused_norm=fused_norm)
    assert st.kernels_per_step() == (3 if fused_norm else 4) and st.fused_norm == fused_norm
    E = oracle.E4M3
    T = wl.tokens
    for t in range(2):
        X, dY = synth.linear_inputs(wl, 0, t, "cuda")
        L = st.layers[0]
        W0 = bf16_bits(L.W)
        pre_opt = _optimizer_state(st)
        st.step([X], [dY])
        cuda_lib.fp8t_check_device_error()
        host = {}
        for name, bits in (("X", bf16_bits(X)), ("W", W0), ("dY", bf16_bits(dY))):
            b = L.mx[name]
            r, c = bits.shape
            rq, rs = oracle.mx_quantise(bits, 0, E)
            cq, cs = oracle.mx_quantise(bits, 1, E)
            assert np.array_equal(u8(b["q_row"]), rq) and np.array_equal(from_atoms(b["sf_row"], r, c), rs)
            assert np.array_equal(u8(b["q_col"]), cq) and np.array_equal(from_atoms(b["sf_col"], c, r), cs.T)
            host[name] = (rq, rs, cq, cs)
        xr, xs_, xc, xcs = host["X"]
        wr, ws_, wc, wcs = host["W"]
        dr, ds_, dc, dcs = host["dY"]
        for D, A, sa, B, sb in ((L.Y, xr, xs_, tr(wc), tr(wcs)), (L.dX, dr, ds_, wr, ws_),
                                (L.dW, tr(xc), tr(xcs), tr(dc), tr(dcs))):
            R, ab = oracle.mx_gemm(A, sa, E, B, sb, E, want_abs=True)
            assert gemm_within_tolerance(bf16_bits(D), R, ab).all()
        if fused_norm:
            sq = np.sort(np.square(L.dW.float().cpu().numpy().astype(np.float64)).reshape(-1))
            exact = float(np.sum(sq))
            assert abs(st.sumsq.item() - exact) <= 1e-13 * exact
        _check_adamw_on_gpu_grad(st, pre_opt, t + 1)


def test_stale_error_word_leaves_a_clean_step_alone(cuda_lib):
    """An expired wait in an unrelated GEMM launch, left unread in the device error word, changes
    nothing in later fused steps: their cast launch still updates the scales, their wgrad sum of
    squares stays finite and AdamW still updates (and casts) the weights, every stage matching the
    oracle; the word still reports the old expiry afterwards."""
    from optimizer_fp8_cast_b200 import Fp8TrainError
    rng = np.random.default_rng(12)
    A = torch.from_numpy(rng.integers(0x20, 0x48, (1024, 2048)).astype(np.uint8)).cuda()
    B = torch.from_numpy(rng.integers(0x20, 0x48, (1024, 2048)).astype(np.uint8)).cuda()
    D = torch.empty(1024, 1024, dtype=torch.bfloat16, device="cuda")
    one = torch.ones(1, device="cuda")
    cuda_lib.fp8t_check_device_error()             # clean start
    try:
        cuda_lib.fp8t_set_wait_timeout_ns(1_000_000)
        cuda_lib.fp8t_debug_expire_waits(2)        # the GEMM epilogue's waits never complete
        cuda_lib.fp8_gemm(A, 0, B, 0, one, one, D)
        torch.cuda.synchronize()
    finally:
        cuda_lib.fp8t_debug_expire_waits(0)
        cuda_lib.fp8t_set_wait_timeout_ns(0)
    wl = synth.LINEAR256
    st = make_step(wl, counters=False)
    assert st.fused_update and st.fused_norm and st.fused_wcast
    for t in range(2):
        xs, dys = zip(*[synth.linear_inputs(wl, k, t, "cuda") for k in range(len(wl.layers))])
        pre = snapshot(st)
        st.step(xs, dys)
        torch.cuda.synchronize()
        assert st.skipped.item() == 0 and np.isfinite(st.sumsq.item())
        check_step(st, pre, xs, dys)
    with pytest.raises(Fp8TrainError) as e:
        cuda_lib.fp8t_check_device_error()
    assert e.value.status == 6                     # FP8T_ERR_TIMEOUT, from the unrelated GEMM
    cuda_lib.fp8t_check_device_error()
