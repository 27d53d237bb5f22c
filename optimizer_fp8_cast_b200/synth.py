"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and rounds them once to BF16 (or keeps FP32 state); it
holds none of the method's arithmetic and imports neither the CUDA library nor the oracle, so
both sides of every parity check can take their inputs from it.

Recipe (the same on CPU and GPU; values differ between the two generators, which is fine because
a parity check always gives both sides the same bytes):
  * each tensor has its own seed crc32("<config seed>/<tensor name>/<step>");
  * draw in FP32 from a torch generator on the target device, apply outliers in FP32, then round
    once to BF16 (round to nearest even).

Workloads (the Linear weight W is stored in x out so that Y = X.W):
  linear256_t512     in = out = 256, 512 tokens, 3 steps, history 16, algo max, margin 0
  linear4096_t8192   4096 x 4096, 8192 tokens (batch 4 x sequence 2048), history 1024, 10 steps
  block7b_t16384     q, k, v, o 4096->4096; gate, up 4096->11008; down 11008->4096; 16384 tokens;
                     X has 6 outlier input columns x100; history 16
  adamw4e9_512t      standalone AdamW over 4.0e9 FP32 parameters in 512 tensors, sizes
                     log-uniform over [4 KB, 256 MB] of FP32 then rescaled to the total
  stress1024_t2048   1024 x 1024, 2048 tokens, 50 steps, X of step 20 multiplied by 1000; swept
                     over history {1, 16, 1024} x algo {max, most_recent} x margin {0, 1}
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field

import numpy as np
import torch

ADAMW_DEFAULT = dict(lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01,
                     loss_scale=1024.0, max_grad_norm=1.0)


@dataclass
class LinearWorkload:
    name: str
    layers: list            # [(name, in_features, out_features)]
    tokens: int
    steps: int
    history_len: int
    algo: str = "max"       # "max" | "most_recent"
    margin: int = 0
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    dy_std: float = 1e-3
    dy_outlier_frac: float = 0.0   # Bernoulli fraction of dY entries multiplied by dy_outlier_mul
    dy_outlier_mul: float = 1000.0
    x_outlier_cols: int = 0        # number of input columns of X multiplied by x_outlier_mul
    x_outlier_mul: float = 100.0
    x_spike_step: int = -1         # step whose whole X batch is multiplied by x_spike_mul
    x_spike_mul: float = 1000.0
    adamw: dict = field(default_factory=lambda: dict(ADAMW_DEFAULT))

    def gemm_flops_per_step(self) -> int:
        return sum(3 * 2 * self.tokens * i * o for _, i, o in self.layers)

    def cast_bytes_per_step(self) -> int:
        """Algorithmic bytes of the three casts per layer: 2 B read + 1 B + 1 B written per element."""
        return sum(4 * (self.tokens * i + i * o + self.tokens * o) for _, i, o in self.layers)

    def params(self) -> int:
        return sum(i * o for _, i, o in self.layers)


LINEAR256 = LinearWorkload("linear256_t512", [("linear", 256, 256)], tokens=512, steps=3,
                           history_len=16, dy_outlier_frac=1e-3)
LINEAR4096 = LinearWorkload("linear4096_t8192", [("linear", 4096, 4096)], tokens=8192, steps=10,
                            history_len=1024)
BLOCK7B = LinearWorkload("block7b_t16384",
                         [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096),
                          ("o", 4096, 4096), ("gate", 4096, 11008), ("up", 4096, 11008),
                          ("down", 11008, 4096)],
                         tokens=16384, steps=1, history_len=16, dy_outlier_frac=1e-3,
                         x_outlier_cols=6)
STRESS1024 = LinearWorkload("stress1024_t2048", [("linear", 1024, 1024)], tokens=2048, steps=50,
                            history_len=16, x_spike_step=20)
STRESS_SWEEP = [(h, a, mg) for h in (1, 16, 1024) for a in ("max", "most_recent") for mg in (0, 1)]

WORKLOADS = {w.name: w for w in (LINEAR256, LINEAR4096, BLOCK7B, STRESS1024)}


def tensor_seed(config_seed: int, name: str, step: int) -> int:
    return zlib.crc32(f"{config_seed}/{name}/{step}".encode()) & 0x7FFFFFFF


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_f32(shape, std, seed, device="cpu"):
    g = _gen(device, seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def linear_inputs(wl: LinearWorkload, layer: int, step: int, device="cpu"):
    """X [tokens, in] and dY [tokens, out] as BF16 tensors for one layer and step."""
    lname, fin, fout = wl.layers[layer]
    x = normal_f32((wl.tokens, fin), wl.x_std, tensor_seed(wl.seed, f"{lname}.X", step), device)
    if wl.x_outlier_cols:
        g = _gen(device, tensor_seed(wl.seed, f"{lname}.Xcols", 0))
        cols = torch.randperm(fin, generator=g, device=device)[: wl.x_outlier_cols]
        x[:, cols] *= wl.x_outlier_mul
    if step == wl.x_spike_step:
        x *= wl.x_spike_mul
    dy = normal_f32((wl.tokens, fout), wl.dy_std, tensor_seed(wl.seed, f"{lname}.dY", step), device)
    if wl.dy_outlier_frac:
        g = _gen(device, tensor_seed(wl.seed, f"{lname}.dYmask", step))
        mask = torch.rand((wl.tokens, fout), generator=g, device=device) < wl.dy_outlier_frac
        dy = torch.where(mask, dy * wl.dy_outlier_mul, dy)
    return x.to(torch.bfloat16), dy.to(torch.bfloat16)


def linear_weight(wl: LinearWorkload, layer: int, device="cpu"):
    """Initial W [in, out] in BF16."""
    lname, fin, fout = wl.layers[layer]
    return normal_f32((fin, fout), wl.w_std, tensor_seed(wl.seed, f"{lname}.W", 0),
                      device).to(torch.bfloat16)


# ----------------------------------------------------------------------------- standalone AdamW
ADAMW4E9 = dict(name="adamw4e9_512t", n_tensors=512, total=4_000_000_000, seed=3,
                min_bytes=4096, max_bytes=256 << 20, grad_std=1e-3, loss_scale=1024.0,
                master_std=0.02, m_std=1e-4, v_std=1e-6,
                hp=dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1,
                        loss_scale=1024.0, max_grad_norm=1.0, step=1000))


def adamw_sizes(n_tensors: int, total: int, seed: int, min_el: int, max_el: int):
    """Element counts: log-uniform over [min_el, max_el], rescaled by one common factor so they sum
    to `total`, clamped to the range, rounded, nudged off multiples of 8 (to exercise vector
    tails), the remainder absorbed by the tensors with room."""
    rng = np.random.default_rng(seed)
    u = rng.random(n_tensors)
    raw = np.exp(math.log(min_el) + u * (math.log(max_el) - math.log(min_el)))
    lo, hi = 1e-3, 1e3
    for _ in range(200):                 # bisection on the common factor
        f = math.sqrt(lo * hi)
        s = np.clip(raw * f, min_el, max_el).sum()
        if s > total:
            hi = f
        else:
            lo = f
    sizes = np.clip(np.rint(raw * lo), min_el, max_el).astype(np.int64)
    sizes[sizes % 8 == 0] += 1
    sizes = np.minimum(sizes, max_el)
    diff = int(total - sizes.sum())
    order = np.argsort(sizes)
    for i in order if diff > 0 else order[::-1]:
        if diff == 0:
            break
        room = (max_el - sizes[i]) if diff > 0 else (sizes[i] - min_el)
        d = min(abs(diff), int(room))
        sizes[i] += d if diff > 0 else -d
        diff += -d if diff > 0 else d
    assert sizes.sum() == total, "size budget not met"
    return sizes


def adamw_tensor(kind: str, numel: int, index: int, cfg: dict, device="cpu"):
    """One tensor of the standalone AdamW workload: kind in {grad, master, m, v}."""
    seed = tensor_seed(cfg["seed"], f"{kind}{index}", 0)
    if kind == "grad":
        g = normal_f32((numel,), cfg["grad_std"], seed, device) * cfg["loss_scale"]
        return g.to(torch.bfloat16)
    if kind == "master":
        return normal_f32((numel,), cfg["master_std"], seed, device)
    if kind == "m":
        return normal_f32((numel,), cfg["m_std"], seed, device)
    if kind == "v":
        return normal_f32((numel,), cfg["v_std"], seed, device).abs_()
    raise ValueError(kind)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a BF16 tensor's bit patterns (uint16)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint8)
