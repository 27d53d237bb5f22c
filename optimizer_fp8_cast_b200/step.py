"""Device state and call sequence of one FP8 delayed-scaling training step of Linear layers.

One step for each layer (W stored in x out, Y = X.W), following the precision flow of
"FP8 混合精度训练工程实践" §四 and the HYBRID recipe of "LLM FP8 微调上线生产实战":

  cast X, W -> E4M3 and dY -> E5M2 with the scales of the previous step (delayed scaling)
  Y  = Xq . Wq      (fprop,  A = Xq K-major,  B = Wq MN-major)
  dX = dYq . Wq^T   (dgrad,  A = dYq K-major, B = Wq K-major)
  dW = Xq^T . dYq   (wgrad,  A = Xq MN-major, B = dYq MN-major)
The tensor cores read 8-bit operands MN-major, so by default no transposed FP8 copy is made;
with transposes=True the casts also write Xq^T, Wq^T, dYq^T and every GEMM reads K-major
operands (the layout a K-major-only tensor core needs).
then, for all layers at once, the amax-history roll and next scales, and one fused AdamW over
every dW (loss-scale unscale, global-norm clip, FP32 master/m/v, BF16 weight for the next step).
With fused_update (the default) the roll and next scales run in the last CTA of the cast launch,
which is possible because the GEMMs read the inverse scales the casts used (sinv_used), not the
next ones (scale_inv). With side_update the same update runs as its own small kernel on a second
stream, concurrently with the GEMM launch (whose one CTA per SM leaves room for it), and AdamW
waits for it: the cast launch then ends without the update's tail. With fused_norm (the default) the wgrad epilogues also form the gradient
sum of squares, and AdamW runs without its norm pass, so each dW is read once. With fused_wcast
(the default when both are on and no counters are kept) AdamW also casts each new BF16 weight
for the next step with that step's scale, which the cast launch's update has already formed;
the cast launch then carries only the scale update of W (its amax came from AdamW), and W is
never read by a cast. The first step's W cast happens once, at construction (prime). All
scalars stay on the device; nothing in a step synchronises with the host.
"""
import torch

from . import (AMAX_MAX, AMAX_MOST_RECENT, CURRENT_WORKSPACE_BYTES, E4M3, E5M2, FP8_MAX,
               fp8_cast_transpose_amax, fp8_cast_transpose_amax_current_multi,
               fp8_cast_transpose_amax_multi, fp8_cast_transpose_amax_update_multi,
               fp8_gemm_multi, fp8_gemm_multi_sumsq, fp8_gemm_sumsq_workspace_bytes,
               fp8_mx_cast_multi, fp8_mx_gemm_multi, fp8_mx_gemm_multi_sumsq,
               fp8_mx_gemm_sumsq_workspace_bytes, mx_scale_bytes,
               fp8_scale_update, fused_adamw_multi_tensor, fused_adamw_multi_tensor_presummed,
               fused_adamw_workspace_bytes)

ROLE_X, ROLE_W, ROLE_DY = 0, 1, 2
ROLE_FMT = (E4M3, E4M3, E5M2)


class LinearLayerBuffers:
    def __init__(self, fin, fout, tokens, w_init, device, transposes=False):
        u8 = dict(dtype=torch.uint8, device=device)
        bf = dict(dtype=torch.bfloat16, device=device)
        self.fin, self.fout, self.tokens = fin, fout, tokens
        self.W = w_init.to(device=device, dtype=torch.bfloat16).contiguous().clone()
        self.master = self.W.float()
        self.m = torch.zeros_like(self.master)
        self.v = torch.zeros_like(self.master)
        self.Xq = torch.empty(tokens, fin, **u8)
        self.Wq = torch.empty(fin, fout, **u8)
        self.dYq = torch.empty(tokens, fout, **u8)
        self.XqT = torch.empty(fin, tokens, **u8) if transposes else None
        self.WqT = torch.empty(fout, fin, **u8) if transposes else None
        self.dYqT = torch.empty(fout, tokens, **u8) if transposes else None
        self.Y = torch.empty(tokens, fout, **bf)
        self.dX = torch.empty(tokens, fin, **bf)
        self.dW = torch.empty(fin, fout, **bf)


class Fp8LinearStep:
    """A group of Linear layers sharing one scale update and one fused AdamW per step.

    Scale state is indexed 3*layer + role (role 0 = X, 1 = W, 2 = dY)."""

    def __init__(self, layer_shapes, tokens, history_len, algo="max", margin=0, adamw=None,
                 w_init=None, device="cuda", counters=False, device_step=False, fused_update=True,
                 fused_norm=True, fused_wcast=True, transposes=False, recipe="delayed",
                 side_update=False):
        self.device = torch.device(device)
        self.tokens = tokens
        self.algo = AMAX_MAX if algo == "max" else AMAX_MOST_RECENT
        self.margin = int(margin)
        self.hp = dict(adamw)
        n = 3 * len(layer_shapes)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.amax = torch.zeros(n, **f32)
        self.history = torch.zeros(n, history_len, **f32)
        self.scale = torch.ones(n, **f32)
        self.scale_inv = torch.ones(n, **f32)          # 1 / next scale (scale update output)
        self.sinv_used = torch.ones(n, **f32)          # 1 / scale the casts used (GEMM input)
        # side_update: the scale update on a second stream, concurrent with the GEMMs
        self.side_update = bool(side_update) and recipe == "delayed"
        self.fused_update = fused_update and not self.side_update
        self.ticket = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.fp8_max = torch.tensor([FP8_MAX[ROLE_FMT[i % 3]] for i in range(n)], **f32)
        self.counters = torch.zeros(n, 3, dtype=torch.int64, device=self.device) if counters else None
        self.transposes = transposes
        self.layers = [LinearLayerBuffers(fi, fo, tokens, w_init[k], self.device, transposes)
                       for k, (fi, fo) in enumerate(layer_shapes)]
        self.grad_norm = torch.zeros(1, **f32)
        self.skipped = torch.zeros(1, dtype=torch.int32, device=self.device)
        ws = fused_adamw_workspace_bytes([l.master.numel() for l in self.layers])
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.device)
        self.t = 0
        # device_step: AdamW counts steps in device memory, so a captured graph can be replayed
        self.step_counter = (torch.zeros(1, dtype=torch.int64, device=self.device)
                             if device_step else None)
        # gradient sum of squares from the wgrad epilogues (fused_norm)
        self.fused_norm = fused_norm
        self.sumsq = torch.zeros(1, dtype=torch.float64, device=self.device)
        gws = fp8_gemm_sumsq_workspace_bytes(self._gemm_descs(sumsq=True))
        self.gemm_workspace = torch.zeros(gws, dtype=torch.uint8, device=self.device)
        self.adamw_ticket = torch.zeros(1, dtype=torch.int32, device=self.device)
        # current scaling: every scale from the tensor's own amax (no history, no delayed update)
        # mxfp8: E4M3 codes with a scale per 32 values, both orientations, block-scaled GEMMs
        assert recipe in ("delayed", "current", "mxfp8")
        self.recipe = recipe
        self.current_ws = torch.zeros(CURRENT_WORKSPACE_BYTES, dtype=torch.uint8, device=self.device)
        if recipe != "delayed":
            fused_update = fused_wcast = False
            self.fused_update = False
        if recipe == "mxfp8":
            u8 = dict(dtype=torch.uint8, device=self.device)
            for L in self.layers:
                shapes = dict(X=(tokens, L.fin), W=(L.fin, L.fout), dY=(tokens, L.fout))
                L.mx = {}
                for name, (r, c) in shapes.items():
                    L.mx[name] = dict(q_row=torch.empty(r, c, **u8), q_col=torch.empty(r, c, **u8),
                                      sf_row=torch.empty(mx_scale_bytes(r, c), **u8),
                                      sf_col=torch.empty(mx_scale_bytes(c, r), **u8))
            if self.fused_norm:            # the wgrad epilogues of the block-scaled launch sum dW^2
                mws = fp8_mx_gemm_sumsq_workspace_bytes(self.mx_gemm_descs(sumsq=True))
                self.mx_gemm_workspace = torch.zeros(mws, **u8)
        # the W cast inside AdamW needs the in-launch scale update and the presummed AdamW, and
        # writes row-major codes only; the saturation / zero counters of W are only kept by the
        # separate cast
        self.fused_wcast = (fused_wcast and (self.fused_update or self.side_update) and fused_norm
                            and not counters and not transposes)
        if self.side_update and self.device.type == "cuda":
            self._side = torch.cuda.Stream(device=self.device)
            self._cast_done = torch.cuda.Event()
            self._update_done = torch.cuda.Event()
        if self.fused_wcast and self.device.type == "cuda":
            self.prime()

    def prime(self):
        """Cast every W with its current scale (codes, transposed codes, amax, scale inverse), as
        the AdamW of a previous step would have: needed before the first step, and after the
        weights or the scale state were loaded."""
        fp8_cast_transpose_amax_multi(
            [self.cast_desc(k, ROLE_W, L.W, L.Wq, L.WqT) for k, L in enumerate(self.layers)])

    def _slot(self, t, i):
        return t[i:i + 1]

    def cast(self, k, role, src, q, qT, stream=None):
        i = 3 * k + role
        fp8_cast_transpose_amax(src, ROLE_FMT[role], self._slot(self.scale, i), q, qT,
                                self._slot(self.amax, i), self._slot(self.sinv_used, i),
                                self.counters[i] if self.counters is not None else None,
                                stream=stream)

    def cast_desc(self, k, role, src, q, qT):
        i = 3 * k + role
        return dict(x=src, fmt=ROLE_FMT[role], scale=self._slot(self.scale, i), q=q, qT=qT,
                    amax=self._slot(self.amax, i),
                    scale_inv=self._slot(self.sinv_used, i) if src is not None else None,
                    counters=self.counters[i] if self.counters is not None and src is not None
                    else None)

    def cast_all(self, xs, dys, stream=None, update=False):
        """Every layer's X, W and dY casts, grouped into launches of up to 8 tensors; with
        update, each launch's last CTA also performs those tensors' scale update."""
        descs = []
        for k, L in enumerate(self.layers):
            # with the W cast inside AdamW, W has no cast here: an update-only entry when the
            # launch updates the scales, nothing otherwise
            w = ([self.cast_desc(k, ROLE_W, None, None, None)] if update else []) if self.fused_wcast \
                else [self.cast_desc(k, ROLE_W, L.W, L.Wq, L.WqT)]
            descs += [self.cast_desc(k, ROLE_X, xs[k], L.Xq, L.XqT)] + w + \
                     [self.cast_desc(k, ROLE_DY, dys[k], L.dYq, L.dYqT)]
        if update:
            ups = [dict(history=self.history[i], scale_inv_next=self._slot(self.scale_inv, i))
                   for i in range(len(descs))]
            assert len(descs) == 3 * len(self.layers)
            fp8_cast_transpose_amax_update_multi(descs, ups, self.algo, self.margin, self.ticket,
                                                 stream=stream)
        else:
            fp8_cast_transpose_amax_multi(descs, stream=stream)

    def mx_cast_all(self, xs, dys, stream=None):
        """MXFP8: X, W and dY quantised with E4M3 codes and one E8M0 scale per 32 values, in
        both orientations (row-wise for K-major use, column-wise for MN-major use)."""
        casts = []
        for k, L in enumerate(self.layers):
            for name, src in (("X", xs[k]), ("W", L.W), ("dY", dys[k])):
                casts.append(dict(x=src, fmt=E4M3, **L.mx[name]))
        fp8_mx_cast_multi(casts, stream=stream)

    def mx_gemm_descs(self, sumsq=False):
        out = []
        for L in self.layers:
            X, W, dY = L.mx["X"], L.mx["W"], L.mx["dY"]
            out += [dict(A=X["q_row"], a_sf=X["sf_row"], a_fmt=E4M3, B=W["q_col"], b_sf=W["sf_col"],
                         b_mn=True, b_fmt=E4M3, D=L.Y),
                    dict(A=dY["q_row"], a_sf=dY["sf_row"], a_fmt=E4M3, B=W["q_row"], b_sf=W["sf_row"],
                         b_fmt=E4M3, D=L.dX),
                    dict(A=X["q_col"], a_sf=X["sf_col"], a_mn=True, a_fmt=E4M3, B=dY["q_col"],
                         b_sf=dY["sf_col"], b_mn=True, b_fmt=E4M3, D=L.dW, sumsq=sumsq)]
        return out

    def mx_gemm_all(self, stream=None, sumsq=False):
        """The block-scaled fprop, dgrad and wgrad of every layer in one grouped launch; with sumsq
        the wgrad epilogues also leave the FP64 sum of dW^2 in self.sumsq."""
        if sumsq:
            fp8_mx_gemm_multi_sumsq(self.mx_gemm_descs(sumsq=True), self.sumsq, self.mx_gemm_workspace,
                                    stream=stream)
        else:
            fp8_mx_gemm_multi(self.mx_gemm_descs(), stream=stream)

    def cast_all_current(self, xs, dys, stream=None):
        """Current scaling: the X, W and dY scales from their own amax, then the casts."""
        descs = []
        for k, L in enumerate(self.layers):
            descs += [self.cast_desc(k, ROLE_X, xs[k], L.Xq, L.XqT),
                      self.cast_desc(k, ROLE_W, L.W, L.Wq, L.WqT),
                      self.cast_desc(k, ROLE_DY, dys[k], L.dYq, L.dYqT)]
        fp8_cast_transpose_amax_current_multi(descs, self.margin, self.current_ws, stream=stream)

    def gemm(self, k, which, stream=None):
        """which: 0 = fprop Y = X.W, 1 = dgrad dX = dY.W^T, 2 = wgrad dW = X^T.dY."""
        fp8_gemm_multi([self.gemm_desc(k, which)], stream=stream)

    def gemm_desc(self, k, which):
        L = self.layers[k]
        sx, sw, sdy = (self._slot(self.sinv_used, 3 * k + r) for r in (ROLE_X, ROLE_W, ROLE_DY))
        t = self.transposes
        if which == 0:
            return dict(A=L.Xq, a_fmt=E4M3, B=L.WqT if t else L.Wq, b_mn=not t, b_fmt=E4M3,
                        a_scale_inv=sx, b_scale_inv=sw, D=L.Y)
        if which == 1:
            return dict(A=L.dYq, a_fmt=E5M2, B=L.Wq, b_fmt=E4M3, a_scale_inv=sdy, b_scale_inv=sw, D=L.dX)
        return dict(A=L.XqT if t else L.Xq, a_mn=not t, a_fmt=E4M3, B=L.dYqT if t else L.dYq,
                    b_mn=not t, b_fmt=E5M2, a_scale_inv=sx, b_scale_inv=sdy, D=L.dW)

    def _gemm_descs(self, sumsq=False):
        descs = [self.gemm_desc(k, w) for k in range(len(self.layers)) for w in (0, 1, 2)]
        if sumsq:
            for i in range(2, len(descs), 3):
                descs[i]["sumsq"] = True                     # the wgrad outputs are the gradients
        return descs

    def gemm_all(self, stream=None, sumsq=False):
        """Every layer's fprop, dgrad and wgrad in one grouped launch (24 GEMMs per launch); with
        sumsq the wgrad epilogues also leave the FP64 sum of dW^2 in self.sumsq."""
        if sumsq:
            fp8_gemm_multi_sumsq(self._gemm_descs(sumsq=True), self.sumsq, self.gemm_workspace,
                                 stream=stream)
        else:
            fp8_gemm_multi(self._gemm_descs(), stream=stream)

    def layer_forward_backward(self, k, X, dY, stream=None):
        L = self.layers[k]
        self.cast(k, ROLE_X, X, L.Xq, L.XqT, stream)
        self.cast(k, ROLE_W, L.W, L.Wq, L.WqT, stream)
        self.cast(k, ROLE_DY, dY, L.dYq, L.dYqT, stream)
        for which in (0, 1, 2):
            self.gemm(k, which, stream)

    def scale_update(self, stream=None):
        fp8_scale_update(self.amax, self.history, self.fp8_max, self.algo, self.margin,
                         self.scale, self.scale_inv, stream=stream)

    def update(self, stream=None):
        self.scale_update(stream)
        self.adamw(stream)

    def adamw(self, stream=None, presummed=False):
        """One fused AdamW over every layer's dW; presummed: take the sum of squares the wgrad
        epilogues left in self.sumsq instead of running the norm pass."""
        hp = self.hp
        if presummed:
            fused_adamw_multi_tensor_presummed(
                [l.master for l in self.layers], [l.m for l in self.layers],
                [l.v for l in self.layers], [l.dW for l in self.layers], [l.W for l in self.layers],
                lr=hp["lr"], beta1=hp["beta1"], beta2=hp["beta2"], eps=hp["eps"],
                weight_decay=hp["weight_decay"], step=self.t, loss_scale=hp["loss_scale"],
                max_grad_norm=hp["max_grad_norm"], grad_sumsq=self.sumsq, grad_norm=self.grad_norm,
                skipped=self.skipped, step_counter=self.step_counter, ticket=self.adamw_ticket,
                casts=self._weight_casts() if self.fused_wcast else None, stream=stream)
            return
        fused_adamw_multi_tensor([l.master for l in self.layers], [l.m for l in self.layers],
                                 [l.v for l in self.layers], [l.dW for l in self.layers],
                                 [l.W for l in self.layers], lr=hp["lr"], beta1=hp["beta1"],
                                 beta2=hp["beta2"], eps=hp["eps"], weight_decay=hp["weight_decay"],
                                 step=self.t, loss_scale=hp["loss_scale"],
                                 max_grad_norm=hp["max_grad_norm"], grad_norm=self.grad_norm,
                                 skipped=self.skipped, workspace=self.workspace,
                                 step_counter=self.step_counter, stream=stream)

    def _weight_casts(self):
        out = []
        for k, L in enumerate(self.layers):
            i = 3 * k + ROLE_W
            out.append(dict(rows=L.fin, cols=L.fout, fmt=E4M3, scale=self._slot(self.scale, i),
                            q=L.Wq, amax=self._slot(self.amax, i),
                            scale_inv=self._slot(self.sinv_used, i)))
        return out

    def step(self, xs, dys, stream=None):
        """One training step; xs[k] = X [tokens, in_k], dys[k] = dY [tokens, out_k] (BF16, device)."""
        self.t += 1
        if self.recipe == "mxfp8":
            self.mx_cast_all(xs, dys, stream)
            self.mx_gemm_all(stream, sumsq=self.fused_norm)
            self.adamw(stream, presummed=self.fused_norm)
            return
        if self.recipe == "current":
            self.amax.zero_()                  # amax slots report this step's tensors only
            self.cast_all_current(xs, dys, stream)
        else:
            self.cast_all(xs, dys, stream, update=self.fused_update)
        if self.side_update:
            self.side_update_begin(stream)
        self.gemm_all(stream, sumsq=self.fused_norm)
        if self.side_update:
            self.side_update_end(stream)
        elif not self.fused_update and self.recipe == "delayed":
            self.scale_update(stream)
        self.adamw(stream, presummed=self.fused_norm)

    def side_update_begin(self, stream=None):
        """After the cast launch: the scale update of every tensor on the side stream."""
        main = torch.cuda.current_stream(self.device) if stream is None else stream
        self._cast_done.record(main)
        self._side.wait_event(self._cast_done)
        self.scale_update(self._side)
        self._update_done.record(self._side)

    def side_update_end(self, stream=None):
        """Before AdamW (which reads the next W scale and accumulates W's amax): join."""
        main = torch.cuda.current_stream(self.device) if stream is None else stream
        main.wait_event(self._update_done)

    # ------------------------------------------------------------------ training state
    def state_dict(self):
        """Everything a resumed run needs to continue bit for bit: per layer the BF16 weight,
        FP32 master, m and v; the FP8 scale state (amax slots, amax history, scales, scale
        inverses); the step count (host and, when used, device counter). The pages' checkpoint
        incident (a restore without the amax history re-warms the scales and drifts) is why the
        scale state is part of it."""
        out = {"t": self.t, "amax": self.amax.clone(), "history": self.history.clone(),
               "scale": self.scale.clone(), "scale_inv": self.scale_inv.clone(),
               "layers": [{"W": l.W.clone(), "master": l.master.clone(), "m": l.m.clone(),
                           "v": l.v.clone()} for l in self.layers]}
        if self.step_counter is not None:
            out["step_counter"] = self.step_counter.clone()
        return out

    def load_state_dict(self, sd):
        """Restore a state_dict into this step's buffers (shapes must match)."""
        self.t = int(sd["t"])
        for name in ("amax", "history", "scale", "scale_inv"):
            getattr(self, name).copy_(sd[name])
        for l, s in zip(self.layers, sd["layers"]):
            for name in ("W", "master", "m", "v"):
                getattr(l, name).copy_(s[name])
        if self.step_counter is not None:
            self.step_counter.copy_(sd.get("step_counter", torch.tensor([self.t])))
        if self.fused_wcast and self.device.type == "cuda":
            self.prime()

    # launches of the library's kernels per step (for the benchmark's launch count)
    def kernels_per_step(self):
        n_adamw_batches = (len(self.layers) + 255) // 256
        # a cast launch carries up to 8 entries: X and dY of every layer, and W unless AdamW casts
        # it and no update in the cast launch needs its (update-only) entry
        per_layer = 2 if self.fused_wcast and not self.fused_update else 3
        n_cast_launches = (per_layer * len(self.layers) + 7) // 8
        n_gemm_launches = (3 * len(self.layers) + 23) // 24
        if self.recipe == "mxfp8":
            return ((3 * len(self.layers) + 7) // 8 + (3 * len(self.layers) + 23) // 24 +
                    (1 if self.fused_norm else 2) * n_adamw_batches)
        n_scale_launches = 0 if (self.fused_update and not self.side_update) or self.recipe == "current" else 1
        if self.recipe == "current":
            n_cast_launches *= 2                   # an amax launch before each cast launch
        n_adamw_launches = (1 if self.fused_norm else 2) * n_adamw_batches
        return n_cast_launches + n_gemm_launches + n_scale_launches + n_adamw_launches
