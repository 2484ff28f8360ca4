"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

Holds no arithmetic of the method: it only draws numbers.  Latents z ~ N(0, 1)
(seed 1234 + batch index); the 16 projection matrices are Xavier-uniform
U(-a, a), a = sqrt(6 / (D + D)), seeds 1..16 in the order
psa(q,k,v,o), cross(q,k,v,o), wsa(q,k,v,o), swsa(q,k,v,o).  Values are drawn
in float64 and rounded once to the run dtype; both sides read the rounded
values.
"""
from __future__ import annotations

import math

import numpy as np
import torch

MODULES = ("psa", "cross", "wsa", "swsa")
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def round_to(x: np.ndarray, dtype: str) -> torch.Tensor:
    """float64 array -> CPU tensor of the run dtype (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(TORCH_DTYPE[dtype])


def latent(N: int, D: int, b: int, dtype: str) -> torch.Tensor:
    rng = np.random.default_rng(1234 + b)
    return round_to(rng.standard_normal((N, D)), dtype)


def latents(B: int, N: int, D: int, dtype: str) -> torch.Tensor:
    """[B, N, D] on the CPU in the run dtype."""
    return torch.stack([latent(N, D, b, dtype) for b in range(B)])


def weights(D: int, dtype: str) -> dict:
    """{module: (Wq, Wk, Wv, Wo)}, each [D][D] (PyTorch Linear layout, y = x W^T)."""
    a = math.sqrt(6.0 / (D + D))
    out, seed = {}, 1
    for m in MODULES:
        ws = []
        for _ in range(4):
            rng = np.random.default_rng(seed)
            ws.append(round_to(rng.uniform(-a, a, (D, D)), dtype))
            seed += 1
        out[m] = tuple(ws)
    return out


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 view of a run-dtype tensor (for the oracle)."""
    return t.detach().to("cpu", torch.float64).numpy()
