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


def proxy_slots(B: int, M: int, P: int, seed: int = 4321) -> torch.Tensor:
    """Random window members for the 'random' proxy extraction: int32 [B, M],
    uniform over [0, P), seeded."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.integers(0, P, size=(B, M)).astype(np.int32))


NORMS = ("proxy", "cross", "wsa", "swsa", "text", "mlp")


def block_params(D: int, Dh: int, dtype: str) -> dict:
    """The complete block's parameters beyond the four attention modules:
    {"text": (Wq, Wk, Wv, Wo) Xavier-uniform [D][D] (seeds 17-20),
     "norms": {name: (gamma, beta)}: gamma ~ U(0.9, 1.1), beta ~ U(-0.1, 0.1)
              (seeds 21-32, in NORMS order),
     "mlp": (W1 [Dh][D], b1 [Dh], W2 [D][Dh], b2 [D]): Xavier-uniform weights,
            biases U(-0.05, 0.05) (seeds 33-36)}."""
    a = math.sqrt(6.0 / (D + D))
    text = tuple(round_to(np.random.default_rng(17 + i).uniform(-a, a, (D, D)), dtype)
                 for i in range(4))
    norms, seed = {}, 21
    for k in NORMS:
        g = round_to(np.random.default_rng(seed).uniform(0.9, 1.1, D), dtype)
        b = round_to(np.random.default_rng(seed + 1).uniform(-0.1, 0.1, D), dtype)
        norms[k] = (g, b)
        seed += 2
    a1 = math.sqrt(6.0 / (D + Dh))
    mlp = (round_to(np.random.default_rng(33).uniform(-a1, a1, (Dh, D)), dtype),
           round_to(np.random.default_rng(34).uniform(-0.05, 0.05, Dh), dtype),
           round_to(np.random.default_rng(35).uniform(-a1, a1, (D, Dh)), dtype),
           round_to(np.random.default_rng(36).uniform(-0.05, 0.05, D), dtype))
    return {"text": text, "norms": norms, "mlp": mlp}


def text_tokens(B: int, L: int, D: int, dtype: str) -> torch.Tensor:
    """[B, L, D] stand-ins for the text encoder's tokens projected to width D:
    N(0, 1), seed 777 + batch index."""
    return torch.stack([round_to(np.random.default_rng(777 + b).standard_normal((L, D)), dtype)
                        for b in range(B)])
