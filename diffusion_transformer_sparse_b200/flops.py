"""Algorithmic FLOP and byte counts of the PT-DiT attention path.

A multiply-add is 2 FLOP.  Attention cores count every score of every window
(the shift mask removes no work).  Per batch item, with N tokens, M proxies,
n tokens per TCM window and width D:

  proxy SA     projections 8 M D^2        core 4 M^2 D
  cross-attn   projections 4 N D^2 + 4 M D^2   core 4 N M D
  WSA, SWSA    projections 8 N D^2 each   core 4 N n D each

Full global self-attention over the same tokens costs 8 N D^2 + 4 N^2 D.  The
core ratio M^2/N^2 + M/N + 2n/N is the complexity paragraph of the Qihoo-T2X
reading note (§3 Method, "2.3% of full attention at 2048^2").
"""
from __future__ import annotations


def block_flops(N: int, M: int, n: int, D: int) -> dict:
    f = {
        "psa_proj": 8 * M * D * D,
        "psa_core": 4 * M * M * D,
        "cross_proj": 4 * N * D * D + 4 * M * D * D,
        "cross_core": 4 * N * M * D,
        "wsa_proj": 8 * N * D * D,
        "wsa_core": 4 * N * n * D,
        "swsa_proj": 8 * N * D * D,
        "swsa_core": 4 * N * n * D,
    }
    f["proj"] = f["psa_proj"] + f["cross_proj"] + f["wsa_proj"] + f["swsa_proj"]
    f["core"] = f["psa_core"] + f["cross_core"] + f["wsa_core"] + f["swsa_core"]
    f["total"] = f["proj"] + f["core"]
    return f


def dense_flops(N: int, D: int) -> dict:
    return {"proj": 8 * N * D * D, "core": 4 * N * N * D, "total": 8 * N * D * D + 4 * N * N * D}


def core_ratio(N: int, M: int, n: int) -> float:
    """Cost of the GIIM + TCM attention cores relative to global attention (2 N^2 D)."""
    return (M / N) ** 2 + M / N + 2 * n / N


def average_bytes(N: int, M: int, D: int, elem: int) -> int:
    """Window averaging: read every token once, write every proxy once."""
    return (N + M) * D * elem


def pt_block_flops(N: int, M: int, n: int, D: int, L: int, Dh: int) -> dict:
    """The complete PT-Block: the attention path plus the text cross-attention
    (projections 4 N D^2 + 4 L D^2, core 4 N L D) and the MLP (4 N D Dh).
    Norms, bias adds and the GELU are not counted."""
    f = block_flops(N, M, n, D)
    f["text_proj"] = 4 * N * D * D + 4 * L * D * D
    f["text_core"] = 4 * N * L * D
    f["mlp"] = 4 * N * D * Dh
    f["proj"] += f["text_proj"] + f["mlp"]
    f["core"] += f["text_core"]
    f["total"] = f["proj"] + f["core"]
    return f


def window_bwd_flops(N: int, n: int, D: int) -> dict:
    """Backward of one TCM branch as ptdit_window_attn_bwd runs it, per batch item:
    the recomputed forward (Q/K/V projections 6 N D^2, attention 4 N n D), dA = dout Wo
    (2 N D^2), the attention backward (S, dP, dV, dK, dQ: 10 N n D), the input gradient
    [dQ dK dV][Wq; Wk; Wv] (6 N D^2) and the weight gradients (8 N D^2)."""
    f = {
        "recompute_proj": 6 * N * D * D,
        "recompute_core": 4 * N * n * D,
        "dA": 2 * N * D * D,
        "core_bwd": 10 * N * n * D,
        "dx": 6 * N * D * D,
        "wgrad": 8 * N * D * D,
    }
    f["gemm"] = f["recompute_proj"] + f["dA"] + f["dx"]
    f["total"] = sum(v for k, v in f.items() if k != "gemm")
    return f


def giim_bwd_flops(N: int, M: int, D: int) -> dict:
    """Backward of GIIM as ptdit_giim_bwd runs it, per batch item: the forward
    recomputed without the output projection, dA = dout Wo (2 N D^2), the cross
    core's backward (S, dP, dV, dK, dQ: 10 N M D), dP' = [dK dV][Wk; Wv] (4 M D^2),
    dA_p = dP' Wo (2 M D^2), the proxy core's backward (10 M^2 D), dP_a =
    [dQ dK dV][Wq; Wk; Wv] (6 M D^2), dz = dQ Wq (2 N D^2) and the weight gradients
    (cross 4 N D^2 + 4 M D^2, proxy 8 M D^2)."""
    fwd = block_flops(N, M, 0, D)
    f = {
        "recompute": fwd["psa_proj"] + fwd["psa_core"] + fwd["cross_proj"] - 2 * N * D * D
        + fwd["cross_core"],
        "rows_core_bwd": 10 * N * M * D + 10 * M * M * D,
        "dx": 2 * N * D * D + 4 * M * D * D + 2 * M * D * D + 6 * M * D * D + 2 * N * D * D,
        "wgrad": 4 * N * D * D + 4 * M * D * D + 8 * M * D * D,
    }
    f["total"] = sum(f.values())
    return f


def block_bwd_flops(N: int, M: int, n: int, D: int) -> dict:
    """Backward of the block-attention path as ptdit_block_attn_bwd runs it, per batch
    item: GIIM's forward for z1, TCM's backward (the WSA forward for z^, then both
    branches' backward, WSA's on the forward kept from z^) and GIIM's backward."""
    fwd = block_flops(N, M, n, D)
    w = window_bwd_flops(N, n, D)
    g = giim_bwd_flops(N, M, D)
    f = {
        "giim_forward": fwd["psa_proj"] + fwd["psa_core"] + fwd["cross_proj"] + fwd["cross_core"],
        "tcm_recompute": fwd["wsa_proj"] + fwd["wsa_core"],
        "tcm_bwd": 2 * w["total"] - w["recompute_proj"] - w["recompute_core"],
        "giim_bwd": g["total"],
    }
    f["total"] = sum(f.values())
    f["window_core_bwd"] = 2 * w["core_bwd"]
    f["rows_core_bwd"] = g["rows_core_bwd"]
    return f


def train_step_flops(N: int, M: int, n: int, D: int) -> dict:
    """A training step of the block-attention path as ptdit_block_attn_fwd_train plus
    ptdit_block_attn_bwd_saved run it, per batch item: the forward (block_flops) and the
    backward without any recomputation (both window branches' and GIIM's backward
    proper)."""
    fwd = block_flops(N, M, n, D)
    w = window_bwd_flops(N, n, D)
    g = giim_bwd_flops(N, M, D)
    f = {
        "forward": fwd["total"],
        "tcm_bwd": 2 * (w["total"] - w["recompute_proj"] - w["recompute_core"]),
        "giim_bwd": g["total"] - g["recompute"],
    }
    f["total"] = sum(f.values())
    f["window_core_bwd"] = 2 * w["core_bwd"]
    f["rows_core_bwd"] = g["rows_core_bwd"]
    return f
