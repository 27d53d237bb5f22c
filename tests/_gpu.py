"""Helpers for the GPU parity tests: host copies in the oracle's representation."""
import numpy as np
import torch

from optimizer_fp8_cast_b200.synth import bf16_bits, u8  # noqa: F401  (re-exported)


def f32(t):
    return t.detach().float().contiguous().cpu().numpy()


def bf16_from_bits(bits, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


def dev_scalar(v, device="cuda"):
    return torch.tensor([v], dtype=torch.float32, device=device)


def sample_positions(M, N, n, seed, tile_m=128, tile_n=256):
    """n seeded random (i, j) plus the first and last row and column of the last tile edges."""
    rng = np.random.default_rng(seed)
    ii = list(rng.integers(0, M, n))
    jj = list(rng.integers(0, N, n))
    edges_i = sorted({0, M - 1, min(M - 1, tile_m), min(M - 1, tile_m - 1), (M - 1) // tile_m * tile_m})
    edges_j = sorted({0, N - 1, min(N - 1, tile_n), min(N - 1, tile_n - 1), (N - 1) // tile_n * tile_n})
    for i in edges_i:
        for j in rng.integers(0, N, 64):
            ii.append(i); jj.append(int(j))
    for j in edges_j:
        for i in rng.integers(0, M, 64):
            ii.append(int(i)); jj.append(j)
    return np.array(ii, np.int64), np.array(jj, np.int64)
