"""The fused window Q/K/V projection + window attention (ptdit_window_fused(1)) and
the two-kernel form (ptdit_window_fused(0), the default)
against the float64 oracle, whole tensors: 3D windows with and without the roll's
wrap masks (the rolled windows load as sub-boxes at their original coordinates),
head widths 72 (two swizzle atoms), 64 and 32, several batch items, a grid whose
windows leave one CTA with more units than another, and the T2V workload in full.
Both forms must also agree with each other closely (same operands, different
rounding order in the softmax)."""
import ctypes

import numpy as np
import pytest
import torch

import diffusion_transformer_sparse_b200 as pt
import oracle as O
from diffusion_transformer_sparse_b200 import build
from tests.helpers import TOL, Case, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pt.lib()
    yield
    pt.lib().ptdit_window_fused(0)


def _run(c, window, shift, m, flags, fused):
    prev = pt.lib().ptdit_window_fused(1 if fused else 0)
    try:
        out = pt.ptdit_window_attn(c.z, c.grid, window, shift, c.w[m], c.heads, flags)
        torch.cuda.synchronize()
    finally:
        pt.lib().ptdit_window_fused(prev)
    return c.out64(out)


CASES = [  # B, grid, D, heads, window, shift
    (1, (2, 16, 16), 1152, 16, (2, 8, 8), (0, 0, 0)),
    (1, (2, 16, 16), 1152, 16, (2, 8, 8), (1, 4, 4)),
    (2, (4, 16, 24), 1152, 16, (2, 8, 8), (1, 4, 4)),   # 2 x 24 windows, wraps in t, y and x
    (1, (4, 16, 16), 1024, 16, (2, 8, 8), (1, 4, 4)),   # d = 64
    (1, (2, 16, 16), 256, 8, (2, 8, 8), (1, 4, 4)),     # d = 32
    (1, (2, 16, 32), 1152, 16, (2, 8, 8), (0, 4, 0)),   # wraps in y only: two sub-boxes
]


@pytest.mark.parametrize("B,grid,D,heads,window,shift", CASES)
def test_fused_window_matches_oracle(B, grid, D, heads, window, shift):
    c = Case(B, grid, D, heads, "bf16")
    m = "swsa" if any(shift) else "wsa"
    got = _run(c, window, shift, m, 0, True)
    two = _run(c, window, shift, m, 0, False)
    for b in range(B):
        want = O.window_self_attention(c.z64[b], grid, window, shift, c.w64[m], heads)
        assert rel_err(got[b], want) <= TOL["bf16"], ("fused", b)
        assert rel_err(two[b], want) <= TOL["bf16"], ("two kernels", b)
    assert rel_err(got, two) <= 1e-2


def test_fused_window_without_residual():
    c = Case(1, (2, 16, 16), 1152, 16, "bf16")
    got = _run(c, (2, 8, 8), (1, 4, 4), "swsa", pt.PTDIT_NO_RESIDUAL, True)
    want = O.window_self_attention(c.z64[0], c.grid, (2, 8, 8), (1, 4, 4), c.w64["swsa"], c.heads,
                                   residual=False)
    assert rel_err(got[0], want) <= TOL["bf16"]


def test_fused_tcm_full_size_t2v():
    """Both TCM branches on the T2V grid (16 x 32 x 48, D = 1152), fused."""
    c = Case(1, (16, 32, 48), 1152, 16, "bf16")
    window, shift = (2, 8, 8), (1, 4, 4)
    prev = pt.lib().ptdit_window_fused(1)
    try:
        out = c.out64(pt.ptdit_tcm(c.z, c.grid, window, shift, c.w["wsa"], c.w["swsa"], c.heads))
    finally:
        pt.lib().ptdit_window_fused(prev)
    want = O.tcm(c.z64[0], c.grid, window, shift, c.w64["wsa"], c.w64["swsa"], c.heads)
    assert rel_err(out[0], want) <= TOL["bf16"]


def test_fused_setting_reads_and_restores():
    L = pt.lib()
    prev = L.ptdit_window_fused(0)
    assert L.ptdit_window_fused(-1) == 0
    assert L.ptdit_window_fused(prev) == 0
    assert L.ptdit_window_fused(7) == prev  # any other value only reads


def test_fused_in_the_complete_block():
    """The complete PT-Block with the fused window kernel: its window branches read the
    LayerNorm output and add the residual stream."""
    from tests.test_gpu_block import _run_block
    c = Case(2, (2, 16, 16), 1152, 16, "bf16")
    prev = pt.lib().ptdit_window_fused(1)
    try:
        _run_block(c, (1, 4, 4), (2, 8, 8), (1, 4, 4), 120, 4608)
    finally:
        pt.lib().ptdit_window_fused(prev)


def test_fused_needs_its_workspace():
    """A workspace that holds everything but the repacked weight rows runs the two-kernel
    form: same result as a full workspace with the fused kernel off."""
    c = Case(1, (2, 16, 16), 1152, 16, "bf16")
    window, shift = (2, 8, 8), (1, 4, 4)
    shape = pt.make_shape(c.z, c.grid, c.heads)
    full = pt.lib().ptdit_workspace_bytes(ctypes.byref(shape), None, pt._i3(window))
    small = full - 16 * 224 * 1152 * 2  # less the repacked weight rows
    ws = torch.empty(small, dtype=torch.uint8, device="cuda")
    prev = pt.lib().ptdit_window_fused(1)
    try:
        got = pt.ptdit_window_attn(c.z, c.grid, window, shift, c.w["swsa"], c.heads, ws=ws)
    finally:
        pt.lib().ptdit_window_fused(prev)
    pt.lib().ptdit_window_fused(0)
    want = pt.ptdit_window_attn(c.z, c.grid, window, shift, c.w["swsa"], c.heads)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
