"""GPU parity of the complete PT-Block (ptdit_pt_block) against the float64 oracle.

The block adds to the attention path the pre-norms of every sub-layer, the
text cross-attention and the MLP (fc1 -> tanh-GELU -> fc2).  Small grids span
several tiles and ragged tails (text lengths that fill part of a key tile,
head widths on both the tensor-core and the CUDA-core attention paths); the
1024 px and 2048 px text-to-image grids run at full size.  Whole outputs are
compared with max|gpu - oracle| / max|oracle| <= 1e-4 (fp32) or 2e-2 (bf16).
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_sparse_b200 as pt
import oracle as O
from diffusion_transformer_sparse_b200 import build, synth
from diffusion_transformer_sparse_b200.configs import WORKLOADS
from tests.helpers import TOL, Case, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pt.lib()


def _run_block(c, ratio, window, shift, L, Dh, mode="mean", slots=None):
    bp = synth.block_params(c.D, Dh, c.dtype)
    text = synth.text_tokens(c.B, L, c.D, c.dtype)
    attn = dict(c.w)
    attn["text"] = tuple(x.cuda() for x in bp["text"])
    norms = {k: tuple(x.cuda() for x in v) for k, v in bp["norms"].items()}
    mlp = tuple(x.cuda() for x in bp["mlp"])
    out = c.out64(pt.ptdit_pt_block(c.z, c.grid, ratio, window, shift, attn, norms, mlp,
                                    text.cuda(), c.heads, mode=mode,
                                    slots=None if slots is None else slots.cuda()))
    W64 = dict(c.w64)
    W64["text"] = tuple(synth.as_f64(x) for x in bp["text"])
    n64 = {k: tuple(synth.as_f64(x) for x in v) for k, v in bp["norms"].items()}
    m64 = tuple(synth.as_f64(x) for x in bp["mlp"])
    for b in range(c.B):
        want = O.pt_block(c.z64[b], c.grid, ratio, window, shift, W64, n64, m64,
                          synth.as_f64(text[b]), c.heads, proxy_mode=mode,
                          slots=None if slots is None else slots[b].numpy())
        err = rel_err(out[b], want)
        assert err <= TOL[c.dtype], (b, err)


@pytest.mark.parametrize("dtype,B,grid,D,heads,ratio,window,shift,L,Dh", [
    ("f32", 1, (1, 16, 16), 64, 2, (1, 2, 2), (1, 4, 4), (0, 2, 2), 7, 256),
    ("bf16", 1, (1, 16, 16), 64, 2, (1, 2, 2), (1, 4, 4), (0, 2, 2), 7, 256),
    ("bf16", 2, (2, 16, 16), 1152, 16, (1, 4, 4), (2, 8, 8), (1, 4, 4), 120, 4608),
    ("bf16", 1, (1, 20, 40), 144, 2, (1, 2, 2), (1, 4, 8), (0, 2, 4), 200, 576),
    ("bf16", 1, (1, 24, 40), 1152, 16, (1, 4, 4), (1, 8, 8), (0, 4, 4), 300, 4608),
])
def test_pt_block_small(dtype, B, grid, D, heads, ratio, window, shift, L, Dh):
    _run_block(Case(B, grid, D, heads, dtype), ratio, window, shift, L, Dh)


def test_pt_block_random_proxies():
    c = Case(2, (2, 16, 16), 1152, 16, "bf16")
    slots = synth.proxy_slots(2, 32, 16, seed=5)
    _run_block(c, (1, 4, 4), (2, 8, 8), (1, 4, 4), 120, 4608, mode="random", slots=slots)


@pytest.mark.parametrize("name", ["t2i_1024px_64x64_b4", "t2i_2048px_128x128"])
def test_pt_block_workload(name):
    w = WORKLOADS[name]
    _run_block(Case(w.B, w.grid, w.D, w.heads, w.dtype), w.ratio, w.window, w.shift, 120,
               4 * w.D)
