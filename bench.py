#!/usr/bin/env python
"""Benchmark of the FP8 delayed-scaling Linear training step and fused AdamW on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of the 4096 x 4096 Linear with 8192
tokens (batch 4 x sequence 2048), four launches captured in one CUDA graph:
  1. the cast launch: X -> E4M3 and dY -> E5M2 (row-major codes, amax, inverse scales used; the
     GEMMs read the codes MN-major where they need the transpose, so no transposed copy is
     written);
  2. the amax-history roll and scale update of X, W and dY (history 1024, algo max, margin 0),
     its own small launch on a second stream, running beside
  3. one grouped GEMM launch: fprop, dgrad and wgrad (FP8 operands, FP32 accumulation, BF16
     out), the wgrad epilogue also summing dW^2 for the global norm;
  4. one fused AdamW launch over dW (unscale, clip, m, v, master, BF16 weight) that also casts
     the new weight to E4M3 codes for the next step (it waits for the scale update).
(--update-in-cast: the update runs in the cast launch's last CTA instead, three launches.)
Inputs are synthetic (seeded normals of the stated shapes), resident in HBM when timing starts.
Before every timed step L2 is flushed by writing a 256 MiB buffer (its dirty lines are written
back while the next step runs, as the previous step's AdamW writes would be in a training loop);
a second, shorter loop also reads a 256 MiB buffer after the write, so that the step starts with
clean lines, and reports each launch's time without that write-back.

Prints one JSON line (rank 0). `value` is the GEMM work of all ranks (3 x 2 x 8192 x 4096 x 4096
FLOP per step per rank) divided by the max over ranks of the summed device time of the K steps.
With N > 1 every rank runs an independent replica (the path has no data-path collective);
the barrier and the max-over-ranks reduction use NCCL. `rooflines` lists the three launches
(GEMM against the FP8 tensor peak, cast and AdamW against HBM), `roofline` is the GEMM's.

`cpu_baseline` times the CPU oracle (the correctness reference, as it stands) on this host, on
one thread and on all of them, stage by stage on samples of about two seconds each; the step
throughput it reports is the step's work over the sum of the stage times that the measured
rates give for the whole step. --impl reference times the oracle on all host threads on a
bounded sample of the workload (the GEMMs at seeded output positions, the other stages on
slices), scaled to the same TFLOP/s unit. Only rank 0 runs either.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FP8 Linear fwd+bwd TFLOP/s; cast+amax & fused AdamW GB/s vs HBM peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0        # nominal dense FP8 / BF16 tensor-core ratio (4.5 / 2.25 PFLOP/s)
DATASHEET_FP8_TFLOPS = 4500.0   # B200 dense FP8 datasheet figure (context denominator)
L2_FLUSH_BYTES = 256 << 20
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


# ----------------------------------------------------------------------------- host helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    return dict(FALLBACK_PEAKS, source="fallback")


def workload_numbers(wl):
    """Algorithmic work per step of a (multi-layer) Linear workload."""
    T = wl.tokens
    return dict(
        gemm_flop=[2 * T * fin * fout for _, fin, fout in wl.layers],   # each of fprop/dgrad/wgrad
        cast_bytes=sum(4 * (T * fin + fin * fout + T * fout) for _, fin, fout in wl.layers),
        adamw_bytes=30 * sum(fin * fout for _, fin, fout in wl.layers),   # 2 B norm + 28 B update
        params=sum(fin * fout for _, fin, fout in wl.layers),
        h2d=sum(2 * T * fin + 2 * T * fout for _, fin, fout in wl.layers),   # X and dY, BF16
        d2h=sum(2 * T * fout + 2 * T * fin for _, fin, fout in wl.layers),   # Y and dX, BF16
    )


def reduce_max(value, world_size, device=None):
    """Max of a float over all ranks (identity when not distributed)."""
    if world_size <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(flop_per_step_per_rank, steps, world_size, total_ms_max):
    """Whole-job TFLOP/s: work of all ranks over the slowest rank's device time."""
    return flop_per_step_per_rank * steps * world_size / (total_ms_max * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi sampling of one GPU's clocks and throttle reasons every 20 ms; entering waits
    (up to 15 s) until the first sample has been written, so the timed region is covered."""

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return self
        t0 = time.time()
        while time.time() - t0 < 15 and os.path.getsize(self.path) == 0 and self.proc.poll() is None:
            time.sleep(0.02)
        self.skip_lines = sum(1 for _ in open(self.path))     # samples taken before timing
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            lines = open(self.path).readlines()[getattr(self, "skip_lines", 0):]
            for line in lines:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), max=float(parts[2]),
                                     power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                     reasons={n: parts[5 + i] == "Active" for i, n in enumerate(REASON_NAMES)}))
                except ValueError:
                    continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        load = [r for r in rows if r["power"] > 250.0] or rows
        reasons = sorted({n for r in load for n, a in r["reasons"].items() if a})
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(load)}


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import optimizer_fp8_cast_b200 as fp8
    from optimizer_fp8_cast_b200 import synth
    from optimizer_fp8_cast_b200.step import Fp8LinearStep

    fp8.load()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = synth.WORKLOADS[args.workload]
    nums = workload_numbers(wl)
    peaks = load_peaks()
    nl = len(wl.layers)

    st = Fp8LinearStep([(i, o) for _, i, o in wl.layers], wl.tokens, wl.history_len, wl.algo,
                       wl.margin, wl.adamw, [synth.linear_weight(wl, k, dev) for k in range(nl)],
                       dev, device_step=True, fused_update=not args.separate_scale_update,
                       fused_norm=not args.separate_norm_pass,
                       fused_wcast=not args.separate_weight_cast, transposes=args.transposes,
                       recipe=args.recipe,
                       side_update=not (args.update_in_cast or args.separate_scale_update))
    batches = [list(zip(*[synth.linear_inputs(wl, k, t, dev) for k in range(nl)])) for t in range(2)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sweep = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    sweep_out = torch.empty((), dtype=torch.int64, device=dev)

    def flush_dirty():                    # L2 full of dirty lines of another buffer
        flush.zero_()

    def flush_clean():                    # the same write, then a read: L2 full of clean lines
        flush.zero_()
        torch.sum(sweep, dim=0, out=sweep_out)

    # one timing window per kernel launch of the step (the scale update runs in the last CTA of
    # the cast launch unless --separate-scale-update)
    stages = [("cast", None), ("gemm", None), ("adamw", None)]
    if args.separate_scale_update and args.recipe == "delayed":
        stages.insert(2, ("scale update", None))
    NEV = len(stages) + 1

    def one_step(xs, dys, ev=None):
        st.t += 1
        rec = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        rec(0)
        for i, (name, kw) in enumerate(stages):
            if name == "cast" and st.recipe == "mxfp8":
                st.mx_cast_all(xs, dys)           # X, W, dY: both orientations + block scales
            elif name == "gemm" and st.recipe == "mxfp8":
                st.mx_gemm_all(sumsq=st.fused_norm)   # grouped block-scaled fprop, dgrad, wgrad
            elif name == "cast" and st.recipe == "current":
                st.amax.zero_()
                st.cast_all_current(xs, dys)      # amax launch, then the grouped cast
            elif name == "cast":                  # grouped: X, W -> E4M3, dY -> E5M2
                st.cast_all(xs, dys, update=st.fused_update)
                if st.side_update:                # the scale update, on a side stream
                    st.side_update_begin()
            elif name == "gemm":                  # grouped: every fprop, dgrad and wgrad
                st.gemm_all(sumsq=st.fused_norm)
                if st.side_update:
                    st.side_update_end()
            elif name == "scale update":
                st.scale_update()
            elif name == "adamw":
                st.adamw(presummed=st.fused_norm)
            else:
                st.gemm(*kw)
            rec(i + 1)

    for w in range(args.warmup):
        flush_dirty()
        one_step(*batches[w % 2])
    torch.cuda.synchronize()
    fp8.fp8t_check_device_error()

    # The step as a CUDA graph (one per input batch), with timing events between its kernels:
    # a static training step is launched this way in production, and it keeps host launch
    # latency out of the kernels' event windows. AdamW counts steps on the device, so every
    # replay is a new optimizer step.
    graphs = []
    if not args.eager:
        for b in range(2):
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(NEV)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                one_step(*batches[b], ev=evs)
            graphs.append((g, evs))
        for g, _ in graphs:
            flush_dirty()
            g.replay()
        torch.cuda.synchronize()
        fp8.fp8t_check_device_error()

    def timed_loop(pre, n):
        """n steps, each after `pre` (outside the events); per-launch and per-step ms."""
        stage_ms, step_ms = [], []
        events = None if graphs else [[torch.cuda.Event(enable_timing=True) for _ in range(NEV)]
                                      for _ in range(n)]
        for t in range(n):
            pre()
            if graphs:
                g, ev = graphs[t % 2]
                g.replay()
                torch.cuda.synchronize()
                stage_ms.append([ev[i].elapsed_time(ev[i + 1]) for i in range(NEV - 1)])
                step_ms.append(ev[0].elapsed_time(ev[NEV - 1]))
            else:
                one_step(*batches[t % 2], ev=events[t])
        torch.cuda.synchronize()
        if events is not None:
            stage_ms = [[events[t][i].elapsed_time(events[t][i + 1]) for i in range(NEV - 1)]
                        for t in range(n)]
            step_ms = [events[t][0].elapsed_time(events[t][NEV - 1]) for t in range(n)]
        return stage_ms, step_ms

    gpu_id = gpu_uuid(dev, local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with ClockSampler(gpu_id) as clocks:
        stage_ms, step_ms = timed_loop(flush_dirty, args.steps)
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    fp8.fp8t_check_device_error()
    total_ms = reduce_max(sum(step_ms), world, dev)
    flop_step = 3 * sum(nums["gemm_flop"])
    value = throughput(flop_step, args.steps, world, total_ms)
    # the same steps after a clean flush: each launch without the write-back of the flush's lines
    n_clean = min(args.steps, 200)
    clean_stage_ms, clean_step_ms = timed_loop(flush_clean, n_clean)
    fp8.fp8t_check_device_error()

    # per-kernel figures (this rank), averaged over the timed steps
    avg = {name: statistics.mean(s[i] for s in stage_ms) for i, (name, _) in enumerate(stages)}
    avg_clean = {name: statistics.mean(s[i] for s in clean_stage_ms) for i, (name, _) in enumerate(stages)}
    gemm_achieved = flop_step / (avg["gemm"] * 1e-3) / 1e12
    # algorithmic bytes of the launches as configured: a cast moves 2 B in and 1 B of codes out
    # per element (+1 B with the transposed copy); the W cast moves from the cast launch into
    # AdamW as 1 B/param of codes (the new weight is already in registers there)
    per_el = (4 if st.transposes else 3) + (2 if st.recipe == "current" else 0)
    cast_bytes = nums["cast_bytes"] // 4 * per_el - (per_el * nums["params"] if st.fused_wcast else 0)
    if st.recipe == "mxfp8":                # 2 B in, 2 x 1 B of codes, 2 x 1/32 B of scales
        cast_bytes = nums["cast_bytes"] // 4 * 65 // 16
    adamw_bytes = ((28 + (1 if st.fused_wcast else 0)) * nums["params"]
                   + (0 if st.fused_norm else 2 * nums["params"]))
    cast_gbs = cast_bytes / (avg["cast"] * 1e-3) / 1e9
    adamw_gbs = adamw_bytes / (avg["adamw"] * 1e-3) / 1e9
    cast_gbs_clean = cast_bytes / (avg_clean["cast"] * 1e-3) / 1e9
    adamw_gbs_clean = adamw_bytes / (avg_clean["adamw"] * 1e-3) / 1e9
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    hbm = peaks["hbm_gbs"]
    # DRAM traffic per launch from the committed ncu counters, when they were taken on the
    # current sources of that kernel and on this configuration
    default_cfg = (args.recipe == "delayed" and not args.transposes and not args.separate_norm_pass
                   and not args.separate_weight_cast and not args.separate_scale_update)
    traffic = {k: (measured_traffic(wl.name, k) if default_cfg else None)
               for k in ("gemm", "cast", "adamw")}
    # the block-scaled launch runs 256 x 384 tiles when every GEMM output is at least 512 wide
    mx_kernel = ("k_fp8_gemm_mx_wide" if min(min(i, o) for _, i, o in wl.layers) >= 512
                 else "k_fp8_gemm<true>")
    gemm_name = (mx_kernel + " block-scaled" if st.recipe == "mxfp8" else "k_fp8_gemm") + \
        " (one grouped launch: every fprop, dgrad, wgrad)"
    cast_name = ("k_mx_cast" if st.recipe == "mxfp8" else
                 "k_current_amax + k_cast_rowmajor" if st.recipe == "current" else
                 "k_cast_transpose_amax" if st.transposes else "k_cast_rowmajor") + " (cast launch)"
    adamw_name = "k_adamw_update" + ("<cast>" if st.fused_wcast else "") + \
        ("" if st.fused_norm else " + k_adamw_sumsq")
    rooflines = [
        {"kernel": gemm_name, "bound": "tensor", "achieved": round(gemm_achieved, 1),
         "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(gemm_achieved / fp8_peak, 4),
         "traffic": traffic["gemm"], "work_per_launch": flop_step,
         "ms_per_launch": round(avg["gemm"], 5),
         "frac_of_datasheet_fp8": round(gemm_achieved / DATASHEET_FP8_TFLOPS, 4),
         "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {FP8_OVER_BF16} "
                        f"(nominal FP8/BF16 ratio); datasheet dense FP8 {DATASHEET_FP8_TFLOPS} TFLOP/s"},
        {"kernel": cast_name, "bound": "hbm", "achieved": round(cast_gbs, 1), "peak": hbm,
         "unit": "GB/s", "frac": round(cast_gbs / hbm, 4), "traffic": traffic["cast"],
         "work_per_launch": cast_bytes, "ms_per_launch": round(avg["cast"], 5),
         "achieved_clean_l2": round(cast_gbs_clean, 1), "frac_clean_l2": round(cast_gbs_clean / hbm, 4),
         "peak_source": f"{peaks['source']} HBM copy"},
        {"kernel": adamw_name, "bound": "hbm", "achieved": round(adamw_gbs, 1), "peak": hbm,
         "unit": "GB/s", "frac": round(adamw_gbs / hbm, 4), "traffic": traffic["adamw"],
         "work_per_launch": adamw_bytes, "ms_per_launch": round(avg["adamw"], 5),
         "achieved_clean_l2": round(adamw_gbs_clean, 1), "frac_clean_l2": round(adamw_gbs_clean / hbm, 4),
         "peak_source": f"{peaks['source']} HBM copy"},
    ]

    for g, _ in graphs:
        del g
    graphs.clear()
    # End to end: X and dY start in pinned host memory and Y, dX end there; every step's copies
    # are inside the timed region. The host-streamed runner overlaps step t's kernels with the
    # copy-in of step t+1 and the copy-out of step t-1 (separate streams and copy engines).
    from optimizer_fp8_cast_b200.host_stream import HostStreamedStep
    runner = HostStreamedStep(st)
    hX = [[x.cpu().pin_memory() for x in b[0]] for b in batches]
    hdY = [[d.cpu().pin_memory() for d in b[1]] for b in batches]
    hY = [[torch.empty(l.Y.shape, dtype=torch.bfloat16).pin_memory() for l in st.layers] for _ in range(2)]
    hdX = [[torch.empty(l.dX.shape, dtype=torch.bfloat16).pin_memory() for l in st.layers] for _ in range(2)]
    for t in range(2):                                   # warm the pinned paths
        runner.step(hX[t], hdY[t], hY[t], hdX[t])
    runner.finish()
    n_e2e = min(args.steps, 50)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(runner.s_in)
    for t in range(n_e2e):
        runner.step(hX[t % 2], hdY[t % 2], hY[t % 2], hdX[t % 2])
    e1.record(runner.s_out)
    runner.finish()
    fp8.fp8t_check_device_error()
    e2e_total = reduce_max(e0.elapsed_time(e1), world, dev)
    e2e_value = throughput(flop_step, n_e2e, world, e2e_total)

    shapes = {lname: [fin, fout] for lname, fin, fout in wl.layers}
    clk = clocks.summary()             # step_kcycles = ms per step x median SM MHz (clock-free)
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8 (e4m3/e5m2 operands, f32 accumulate)",
        "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.tokens,
                   "layers_in_out": shapes,
                   "recipe": "MXFP8 (E4M3, E8M0 scale per 32 values)" if args.recipe == "mxfp8"
                             else f"HYBRID, {args.recipe} per-tensor scaling",
                   "history_len": wl.history_len, "amax_algo": wl.algo, "margin": wl.margin,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": "eager" if args.eager else "CUDA graph per step (AdamW step counter on the device)",
                   "scale_update": "none (MX block scales)" if args.recipe == "mxfp8"
                                   else "none (current scaling)" if args.recipe == "current"
                                   else "separate launch" if args.separate_scale_update
                                   else "own launch on a side stream, concurrent with the GEMMs"
                                   if st.side_update
                                   else "in the last CTA of the cast launch",
                   "grad_sum_of_squares": "AdamW norm pass" if args.separate_norm_pass
                                          else "in the wgrad GEMM epilogue",
                   "weight_cast": "in AdamW (next step's codes)" if st.fused_wcast
                                  else "in the cast launch",
                   "operands": "K-major only (transposed FP8 copies written by the casts)"
                               if st.transposes else "no transposed copies (wgrad A, B and fprop B "
                                                     "read MN-major by tcgen05)",
                   "l2": "flushed before every timed step (256 MiB write; its dirty lines are "
                         "written back during the step); kernels.clean_l2: a 256 MiB read after "
                         "the write"},
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": nums["h2d"],
                "d2h_bytes_per_step": nums["d2h"], "ms_per_step": round(e2e_total / n_e2e, 4),
                "how": "pinned host X, dY in and Y, dX out every step; copies overlapped with "
                       "the previous/next step's kernels on separate streams"},
        "gpu_launches": args.steps * st.kernels_per_step(),
        "roofline": dict(rooflines[0]),
        "rooflines": rooflines,
        "kernels": {
            "stage_ms": {n: round(a, 4) for n, a in avg.items()},
            "gemm_tflops": round(gemm_achieved, 1),
            "cast_gbs": round(cast_gbs, 1), "cast_frac_of_hbm": round(cast_gbs / hbm, 4),
            "cast_bytes_per_step": cast_bytes, "adamw_bytes_per_step": adamw_bytes,
            "adamw_gbs": round(adamw_gbs, 1), "adamw_frac_of_hbm": round(adamw_gbs / hbm, 4),
            "hbm_peak_gbs": hbm, "peak_source": peaks["source"],
            "clean_l2": {"steps": n_clean,
                         "stage_ms": {n: round(a, 4) for n, a in avg_clean.items()},
                         "ms_per_step": round(statistics.mean(clean_step_ms), 4),
                         "cast_gbs": round(cast_gbs_clean, 1),
                         "cast_frac_of_hbm": round(cast_gbs_clean / hbm, 4),
                         "adamw_gbs": round(adamw_gbs_clean, 1),
                         "adamw_frac_of_hbm": round(adamw_gbs_clean / hbm, 4),
                         "gemm_tflops": round(flop_step / (avg_clean["gemm"] * 1e-3) / 1e12, 1),
                         "how": "256 MiB write then 256 MiB read before each step (outside the "
                                "events): L2 holds clean lines, nothing is written back during the step"},
        },
        "clocks": clk,
        "step_kcycles": (round(total_ms / args.steps * clk["sm_mhz"], 1) if clk.get("sm_mhz") else None),
        "wall_s_timed_region": round(wall, 3),
    }
    if world == 1 and nl == 1 and not args.no_comparator:
        _, fin, fout = wl.layers[0]
        result["comparator"] = {
            "what": "torch._scaled_mm (cuBLAS FP8) vs this library's fp8_gemm, the step's three GEMM "
                    "shapes with K-major E4M3 operands, back-to-back launches, L2 warm; not the step",
            "shapes": gemm_comparator(fp8, dev, [(wl.tokens, fout, fin), (wl.tokens, fin, fout),
                                                 (fin, fout, wl.tokens)])}
    if rank == 0 and world == 1 and nl == 1 and not args.no_cpu_baseline:
        b0 = (batches[0][0][0], batches[0][1][0])
        result["cpu_baseline"] = cpu_baseline(st, wl, nums, b0)
    return result


def run_adamw_only(args):
    """The standalone multi-tensor AdamW workload: 4.0e9 FP32 parameters in 512 tensors."""
    import torch

    import optimizer_fp8_cast_b200 as fp8
    from optimizer_fp8_cast_b200 import synth
    fp8.load()
    dev = torch.device("cuda", 0)
    cfg = synth.ADAMW4E9
    sizes = [int(n) for n in synth.adamw_sizes(cfg["n_tensors"], cfg["total"], cfg["seed"],
                                               cfg["min_bytes"] // 4, cfg["max_bytes"] // 4)]
    free, _ = torch.cuda.mem_get_info()
    need = 16 * sum(sizes) + (1 << 30)
    if free < need:
        return {"metric": METRIC, "workload": cfg["name"], "unavailable":
                f"needs {need / 1e9:.0f} GB of free device memory, {free / 1e9:.0f} GB free"}
    P = [synth.adamw_tensor("master", n, i, cfg, dev) for i, n in enumerate(sizes)]
    M = [synth.adamw_tensor("m", n, i, cfg, dev) for i, n in enumerate(sizes)]
    V = [synth.adamw_tensor("v", n, i, cfg, dev) for i, n in enumerate(sizes)]
    G = [synth.adamw_tensor("grad", n, i, cfg, dev) for i, n in enumerate(sizes)]
    W = [torch.empty(n, dtype=torch.bfloat16, device=dev) for n in sizes]
    ws = torch.empty(fp8.fused_adamw_workspace_bytes(sizes), dtype=torch.uint8, device=dev)
    counter = torch.tensor([cfg["hp"]["step"] - 1], dtype=torch.int64, device=dev)
    hp = {k: v for k, v in cfg["hp"].items() if k != "step"}

    def step():
        fp8.fused_adamw_multi_tensor(P, M, V, G, W, step=0, step_counter=counter, workspace=ws, **hp)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    fp8.fp8t_check_device_error()
    steps = min(args.steps, 20)
    e = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with ClockSampler(gpu_uuid(dev, 0)) as clocks:
        e[0].record()
        for t in range(steps):
            step()
            e[t + 1].record()
        torch.cuda.synchronize()
    fp8.fp8t_check_device_error()
    ms = [e[t].elapsed_time(e[t + 1]) for t in range(steps)]
    total = sum(sizes)
    gbs = 30 * total * steps / (sum(ms) * 1e-3) / 1e9
    hbm = load_peaks()["hbm_gbs"]
    return {"metric": METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": steps,
            "warmup": args.warmup, "ms_per_step": round(statistics.mean(ms), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": cfg["name"], "params": total, "tensors": len(sizes),
                       "bytes_per_param": "30 (2 norm pass + 28 update)",
                       "l2": "inputs (64 GB) far larger than L2"},
            "roofline": {"kernel": "k_adamw_sumsq + k_adamw_update", "bound": "hbm",
                         "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "traffic": None},
            "gpu_launches": steps * 4, "clocks": clocks.summary()}


def run_stress_sweep(args):
    """The 1024 x 1024 / 2048-token stress run, 50 steps with the x1000 X batch at step 20, swept
    over history length, algorithm and margin: per-tensor saturation and zero fractions every
    step, and the cast launch's share of the step time."""
    import torch

    import optimizer_fp8_cast_b200 as fp8
    from optimizer_fp8_cast_b200 import synth
    from optimizer_fp8_cast_b200.step import Fp8LinearStep
    fp8.load()
    dev = torch.device("cuda", 0)
    wl = synth.STRESS1024
    _, fin, fout = wl.layers[0]
    n_el = [wl.tokens * fin, fin * fout, wl.tokens * fout]
    table, summary = [], []
    for H, algo, margin in synth.STRESS_SWEEP:
        st = Fp8LinearStep([(fin, fout)], wl.tokens, H, algo, margin, wl.adamw,
                           [synth.linear_weight(wl, 0, dev)], dev, counters=True)
        cast_ms, step_ms = [], []
        for t in range(wl.steps):
            X, dY = synth.linear_inputs(wl, 0, t, dev)
            st.counters.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            st.t += 1
            e[0].record()
            st.cast_all([X], [dY])
            e[1].record()
            for which in (0, 1, 2):
                st.gemm(0, which)
            st.update()
            e[2].record()
            torch.cuda.synchronize()
            cast_ms.append(e[0].elapsed_time(e[1]))
            step_ms.append(e[0].elapsed_time(e[2]))
            c = st.counters.cpu().numpy()
            row = {"H": H, "algo": algo, "margin": margin, "step": t}
            for r, name in enumerate(("X", "W", "dY")):
                row[f"sat_{name}"] = float(c[r, 0]) / n_el[r]
                row[f"zero_{name}"] = float(c[r, 1]) / n_el[r]
            row["scale_X"] = float(st.scale[0].item())
            table.append(row)
        fp8.fp8t_check_device_error()
        rows = table[-wl.steps:]
        summary.append({"H": H, "algo": algo, "margin": margin,
                        "sat_X_step19": rows[19]["sat_X"], "sat_X_step20": rows[20]["sat_X"],
                        "sat_X_step21": rows[21]["sat_X"],
                        "zero_X_step21": rows[21]["zero_X"], "zero_X_step49": rows[49]["zero_X"],
                        "zero_W_step1": rows[1]["zero_W"], "zero_W_step49": rows[49]["zero_W"],
                        "sat_dY_mean": statistics.mean(r["sat_dY"] for r in rows),
                        "cast_overhead_frac": round(sum(cast_ms[5:]) / sum(step_ms[5:]), 4)})
    if args.out:
        with open(args.out, "w") as f:
            json.dump(table, f)
    return {"metric": METRIC, "workload": wl.name, "unit": "fractions",
            "config": {"workload": wl.name, "tokens": wl.tokens, "in_features": fin,
                       "out_features": fout, "steps": wl.steps, "spike_step": wl.x_spike_step,
                       "launch": "eager, counters on, one synchronisation per step (not a throughput run)"},
            "sweep": summary, "per_step_table": args.out}


def gpu_uuid(dev, fallback):
    """nvidia-smi identifier of a torch device (its UUID), independent of device renumbering."""
    import torch
    props = torch.cuda.get_device_properties(dev)
    u = getattr(props, "uuid", None)
    if u is None:
        return fallback
    s = str(u)
    return s if s.startswith("GPU-") else "GPU-" + s


def gemm_comparator(fp8, dev, shapes, seconds=0.3):
    """cuBLAS FP8 (torch._scaled_mm, E4M3 x E4M3 -> BF16, unit scales) beside this library's GEMM
    on the same shapes and K-major operands, back-to-back launches (L2 warm), each timed for about
    `seconds`. A comparator only: nothing on the measured path calls a library GEMM."""
    import torch
    out = []
    one_t = torch.ones((), device=dev)
    one = torch.ones(1, device=dev)
    for M, N, K in shapes:
        A = torch.randint(0, 120, (M, K), dtype=torch.uint8, device=dev)
        B = torch.randint(0, 120, (N, K), dtype=torch.uint8, device=dev)
        D = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        a8, b8 = A.view(torch.float8_e4m3fn), B.view(torch.float8_e4m3fn)
        row = {"M": M, "N": N, "K": K}
        for name, fn in (("ours", lambda: fp8.fp8_gemm_multi([dict(A=A, a_fmt=0, B=B, b_fmt=0, a_scale_inv=one,
                                                                     b_scale_inv=one, D=D)])),
                         ("cublas", lambda: torch._scaled_mm(a8, b8.t(), scale_a=one_t, scale_b=one_t,
                                                             out_dtype=torch.bfloat16))):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            n = max(10, int(seconds / (2.0 * M * N * K / 3.0e15)))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(n):
                fn()
            e1.record()
            torch.cuda.synchronize()
            row[name + "_tflops"] = round(2.0 * M * N * K * n / (e0.elapsed_time(e1) * 1e-3) / 1e12, 1)
        out.append(row)
    return out


# source files whose change invalidates a kernel's committed DRAM counters
KERNEL_SOURCES = {
    "gemm": ("gemm_tcgen05.cuh", "ptx.cuh", "fp8train.cu"),
    "cast": ("cast_transpose_amax.cuh", "scale_update.cuh", "ptx.cuh", "fp8train.cu"),
    "adamw": ("fused_adamw.cuh", "ptx.cuh", "fp8train.cu"),
}


def kernel_source_sha(kernel):
    """Hash of the sources a kernel's launches are built from."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "optimizer_fp8_cast_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload, kernel):
    """DRAM bytes (read + write) per launch of a kernel of the default step, from the ncu counters
    committed in profiles/traffic_<workload>.json, or None when there are none or they were taken
    on other sources of that kernel."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entry = json.load(f).get("kernels", {}).get(kernel)
    if not entry or entry.get("source_sha") != kernel_source_sha(kernel):
        return None
    return int(entry["dram_bytes_per_launch"])


# ----------------------------------------------------------------------------- CPU oracle
def cpu_host():
    """The host the CPU figures were taken on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


CPU_STAGE_S = 1.5      # oracle seconds per stage and thread setting, about


def _calibrated(run, unit_max, budget_s, probe_units):
    """Run `run(units)` once on a probe, then on as many units as fill about budget_s (at most
    unit_max); returns (seconds, units) of the second run."""
    t0 = time.perf_counter()
    run(probe_units)
    dt = max(time.perf_counter() - t0, 1e-6)
    units = int(min(unit_max, max(probe_units, probe_units * budget_s / dt)))
    t0 = time.perf_counter()
    run(units)
    return time.perf_counter() - t0, units


def oracle_stage_rates(oracle, host, wl, threads, budget_s=CPU_STAGE_S):
    """The CPU oracle, stage by stage, on samples of the workload sized to about budget_s each:
    casts of X (E4M3) and dY (E5M2) rows, the three GEMMs at seeded output positions, the scale
    update of X, W and dY (history H), AdamW (norm pass and update) on a slice of the parameters.
    Returns the rates and what each sample was."""
    import numpy as np
    oracle.set_threads(threads)
    _, fin, fout = wl.layers[0]
    T = wl.tokens
    out = {}
    # casts: 3 B per element (2 read, 1 code written), as the GPU cast's algorithmic bytes
    def cast(rows):
        oracle.cast_transpose_amax(host["X"][:rows], oracle.E4M3, 1.0, True, False)
        oracle.cast_transpose_amax(host["dY"][:rows], oracle.E5M2, 1.0, True, False)
    dt, rows = _calibrated(cast, T, budget_s, 4)
    out["cast"] = {"gbs": 3 * rows * (fin + fout) / dt / 1e9, "sample": f"{rows} rows of X and dY"}
    # GEMMs: n outputs of each (fprop K = in, dgrad K = out, wgrad K = tokens)
    rng = np.random.default_rng(7)
    gemms = ((host["Xq"], 0, host["WqT"], 0, fin), (host["dYq"], 1, host["Wq"], 0, fout),
             (host["XqT"], 0, host["dYqT"], 1, T))
    def gemm(n):
        for A, af, B, bf, _ in gemms:
            oracle.gemm_at(A, af, B, bf, 1.0, 1.0, rng.integers(0, A.shape[0], n),
                           rng.integers(0, B.shape[0], n))
    dt, n = _calibrated(gemm, 1 << 22, budget_s, 8 * max(1, threads))
    out["gemm"] = {"tflops": 2 * n * (fin + fout + T) / dt / 1e12,
                   "sample": f"{n} outputs of each of the three GEMMs"}
    # scale update of the three tensors (median of 9)
    times = []
    for _ in range(9):
        hist = np.zeros((3, wl.history_len), np.float32)
        sc, si = np.ones(3, np.float32), np.ones(3, np.float32)
        t0 = time.perf_counter()
        oracle.scale_update(np.ones(3, np.float32), hist, [448.0, 448.0, 57344.0], 0, 0, sc, si)
        times.append(time.perf_counter() - t0)
    out["scale_update"] = {"us": statistics.median(times) * 1e6, "sample": f"3 tensors, H = {wl.history_len}"}
    # AdamW: norm pass (2 B/param) + update (28 B/param)
    def adamw(n):
        oracle.fused_adamw([host["master"][:n].copy()], [np.zeros(n, np.float32)],
                           [np.zeros(n, np.float32)], [host["dW"][:n]], [np.zeros(n, np.uint16)],
                           dict(wl.adamw, step=1))
    dt, n = _calibrated(adamw, host["master"].size, budget_s, 1 << 16)
    out["adamw"] = {"gbs": 30 * n / dt / 1e9, "sample": f"{n} parameters"}
    return out


def oracle_step_value(rates, nums, flop_step):
    """Step throughput (TFLOP/s) the measured stage rates give for one whole step."""
    t = (nums["cast_bytes"] // 4 * 3 / (rates["cast"]["gbs"] * 1e9)
         + flop_step / (rates["gemm"]["tflops"] * 1e12)
         + rates["scale_update"]["us"] * 1e-6
         + 30 * nums["params"] / (rates["adamw"]["gbs"] * 1e9))
    return flop_step / t / 1e12, t


def oracle_output_sample_step(oracle, host, wl, n_out, rng):
    """One step of the path with every stage on a small sample: casts of one row of X, W and dY,
    the three GEMMs at n_out seeded output positions each (oracle.gemm_at), the scale update
    and AdamW on 16 * n_out parameters. Returns (seconds, GEMM FLOP of the sample)."""
    import numpy as np
    _, fin, fout = wl.layers[0]
    T = wl.tokens
    t0 = time.perf_counter()
    oracle.cast_transpose_amax(host["X"][:1], oracle.E4M3, 1.0)
    oracle.cast_transpose_amax(host["W"][:1], oracle.E4M3, 1.0)
    oracle.cast_transpose_amax(host["dY"][:1], oracle.E5M2, 1.0)
    flop = 0
    for A, af, B, bf, K in ((host["Xq"], 0, host["WqT"], 0, fin), (host["dYq"], 1, host["Wq"], 0, fout),
                            (host["XqT"], 0, host["dYqT"], 1, T)):
        ii = rng.integers(0, A.shape[0], n_out)
        jj = rng.integers(0, B.shape[0], n_out)
        oracle.gemm_at(A, af, B, bf, 1.0, 1.0, ii, jj)
        flop += 2 * n_out * K
    hist = np.zeros((3, wl.history_len), np.float32)
    sc = np.ones(3, np.float32)
    si = np.ones(3, np.float32)
    oracle.scale_update(np.ones(3, np.float32), hist, [448.0, 448.0, 57344.0], 0, 0, sc, si)
    n = min(16 * n_out, host["master"].size)
    oracle.fused_adamw([host["master"][:n].copy()], [np.zeros(n, np.float32)], [np.zeros(n, np.float32)],
                       [host["dW"][:n]], [np.zeros(n, np.uint16)], dict(wl.adamw, step=1))
    return time.perf_counter() - t0, flop


def host_copies(st, batch):
    from optimizer_fp8_cast_b200.synth import bf16_bits, u8
    import numpy as np
    L = st.layers[0]
    t = lambda q, qT: u8(qT) if qT is not None else np.ascontiguousarray(u8(q).T)
    return dict(X=bf16_bits(batch[0]), dY=bf16_bits(batch[1]), W=bf16_bits(L.W), Xq=u8(L.Xq),
                XqT=t(L.Xq, L.XqT), Wq=u8(L.Wq), WqT=t(L.Wq, L.WqT), dYq=u8(L.dYq),
                dYqT=t(L.dYq, L.dYqT),
                master=L.master.detach().cpu().numpy().reshape(-1),
                dW=bf16_bits(L.dW).reshape(-1))


def cpu_baseline(st, wl, nums, batch):
    import oracle
    host = host_copies(st, batch)
    flop_step = 3 * sum(nums["gemm_flop"])
    t0 = time.perf_counter()
    one = oracle_stage_rates(oracle, host, wl, 1)
    n_all = oracle.set_threads(0)
    every = oracle_stage_rates(oracle, host, wl, n_all)
    spent = time.perf_counter() - t0
    v1, t1 = oracle_step_value(one, nums, flop_step)
    va, ta = oracle_step_value(every, nums, flop_step)
    stages = {k: {"one_thread": {m: (round(x, 6) if isinstance(x, float) else x) for m, x in one[k].items()},
                  "all_threads": {m: (round(x, 6) if isinstance(x, float) else x) for m, x in every[k].items()}}
              for k in one}
    return {"value": round(va, 9), "unit": UNIT, "cores": n_all, "kind": "oracle",
            "sample": f"each stage on a sample of about {CPU_STAGE_S} s per thread setting "
                      f"({spent:.0f} s in all); value = the step's GEMM FLOP over the whole-step "
                      f"time the {n_all}-thread stage rates give ({ta:.1f} s)",
            "host": cpu_host(), "one_thread": {"value": round(v1, 9), "step_s": round(t1, 2)},
            "all_threads_step_s": round(ta, 2), "stages": stages}


REFERENCE_BUDGET_S = 90.0       # the reference arm's warm-up plus timed steps, about


def run_reference(args):
    """The CPU oracle as the reference arm: bounded samples, same metric and unit."""
    import torch

    import oracle
    from optimizer_fp8_cast_b200 import synth
    import numpy as np
    wl = synth.WORKLOADS[args.workload]
    _, fin, fout = wl.layers[0]
    # inputs: seeded CPU draws of the workload's shapes, quantised by the oracle itself
    X, dY = synth.linear_inputs(wl, 0, 0, "cpu")
    W = synth.linear_weight(wl, 0, "cpu")
    host = dict(X=synth.bf16_bits(X), dY=synth.bf16_bits(dY), W=synth.bf16_bits(W))
    q, qT, _, _, _ = oracle.cast_transpose_amax(host["X"], oracle.E4M3, 1.0)
    host["Xq"], host["XqT"] = q, qT
    q, qT, _, _, _ = oracle.cast_transpose_amax(host["W"], oracle.E4M3, 1.0)
    host["Wq"], host["WqT"] = q, qT
    q, qT, _, _, _ = oracle.cast_transpose_amax(host["dY"], oracle.E5M2, 1.0)
    host["dYq"], host["dYqT"] = q, qT
    host["master"] = W.float().numpy().reshape(-1)
    host["dW"] = synth.bf16_bits(torch.randn(fin * fout, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16))
    host = {k: np.ascontiguousarray(v) for k, v in host.items()}
    threads = oracle.set_threads(0)          # every host core
    # size each step's sample so that warm-up plus timed steps take about REFERENCE_BUDGET_S
    rng = np.random.default_rng(0)
    probe_n = 64 * threads
    probe, _ = oracle_output_sample_step(oracle, host, wl, probe_n, rng)
    per_step = REFERENCE_BUDGET_S / max(1, args.steps + args.warmup)
    n_out = int(min(1 << 20, max(8, probe_n * per_step / max(probe, 1e-6))))
    for _ in range(args.warmup):
        oracle_output_sample_step(oracle, host, wl, n_out, rng)
    times, flops = [], []
    for _ in range(args.steps):
        dt, fl = oracle_output_sample_step(oracle, host, wl, n_out, rng)
        times.append(dt)
        flops.append(fl)
    total = sum(times)
    value = sum(flops) / total / 1e12
    sample = (f"every stage on a sample per step: casts of one row of X, W, dY; each GEMM at {n_out} "
              f"seeded outputs ({flops[0] / 1e9:.3f} GFLOP); scale update; AdamW on {16 * n_out} "
              f"parameters; C oracle on {threads} host threads")
    return {
        "metric": METRIC, "value": round(value, 9), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8 codes, exact integer accumulation (CPU oracle)", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.tokens, "in_features": fin,
                   "out_features": fout, "history_len": wl.history_len},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 9), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample, "host": cpu_host()},
        "e2e": {"value": round(value, 9), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="linear4096_t8192",
                    help="linear4096_t8192 (default), linear256_t512, block7b_t16384, "
                         "adamw4e9_512t, stress1024_t2048")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-comparator", action="store_true",
                    help="skip the cuBLAS FP8 comparator timing of the step's GEMM shapes")
    ap.add_argument("--eager", action="store_true", help="time eager launches, not CUDA graphs")
    ap.add_argument("--recipe", choices=("delayed", "current", "mxfp8"), default="delayed",
                    help="current: each scale from its own tensor's amax (an extra read); "
                         "mxfp8: E4M3 with one E8M0 scale per 32 values, block-scaled GEMMs")
    ap.add_argument("--transposes", action="store_true",
                    help="casts also write q^T and every GEMM reads K-major operands")
    ap.add_argument("--separate-weight-cast", action="store_true",
                    help="cast W in the cast launch instead of inside AdamW")
    ap.add_argument("--separate-norm-pass", action="store_true",
                    help="run AdamW's own norm pass instead of summing dW^2 in the wgrad epilogue")
    ap.add_argument("--separate-scale-update", action="store_true",
                    help="run the scale update as its own launch instead of in the cast launch")
    ap.add_argument("--update-in-cast", action="store_true",
                    help="run the scale update in the cast launch's last CTA instead of as its own "
                         "launch on a second stream, concurrently with the GEMM launch (default)")
    ap.add_argument("--out", default=None, help="stress sweep: write the per-step table here")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload == "adamw4e9_512t":
            result = run_adamw_only(args)
        elif args.workload == "stress1024_t2048":
            result = run_stress_sweep(args)
        else:
            result = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
