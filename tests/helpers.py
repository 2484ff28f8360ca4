"""Shared helpers of the GPU tests: seeded cases on the device and their float64 copies."""
from __future__ import annotations

import numpy as np
import torch

from diffusion_transformer_sparse_b200 import synth

# Tolerances on max_i |gpu_i - oracle_i| / max_i |oracle_i| per output tensor.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), "non-finite GPU output"
    return float(np.max(np.abs(got - want)) / max(1e-30, np.max(np.abs(want))))


class Case:
    """Seeded latents and weights of one workload, on the GPU and as float64."""

    def __init__(self, B, grid, D, heads, dtype, seed_offset=0):
        self.B, self.grid, self.D, self.heads, self.dtype = B, tuple(grid), D, heads, dtype
        self.N = grid[0] * grid[1] * grid[2]
        z = synth.latents(B, self.N, D, dtype)
        if seed_offset:
            z = torch.stack([synth.latent(self.N, D, b + seed_offset, dtype) for b in range(B)])
        self.z_cpu = z
        self.z = z.cuda()
        w = synth.weights(D, dtype)
        self.w_cpu = w
        self.w = {m: tuple(x.cuda() for x in ws) for m, ws in w.items()}
        self.z64 = synth.as_f64(z)
        self.w64 = {m: tuple(synth.as_f64(x) for x in ws) for m, ws in w.items()}

    def out64(self, t) -> np.ndarray:
        torch.cuda.synchronize()
        return t.detach().to("cpu", torch.float64).numpy()


def sample_rows(grid, k=6, seed=0):
    """Corner tokens of the grid (every wrapped-window edge) plus k random ones."""
    f, h, w = grid
    rows = set()
    for t in (0, f - 1):
        for y in (0, h - 1):
            for x in (0, w - 1):
                rows.add((t * h + y) * w + x)
    rng = np.random.default_rng(seed)
    rows.update(int(r) for r in rng.integers(0, f * h * w, k))
    return np.array(sorted(rows))
