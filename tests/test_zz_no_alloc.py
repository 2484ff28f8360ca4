"""ptdit_window_attn_static: window attention for callers that cannot allocate.

Some callers cannot call cudaMalloc (it may synchronise the device, it may be
forbidden where they run, or they only receive input and output buffers from a
framework whose allocator they cannot reach).  For them the library offers one
entry point whose scratch is a static device array inside the library.  This
test calls it through the C ABI twice in a row, with different inputs, weights
and shifts, and checks each result against ptdit_window_attn given a
caller-allocated workspace.  It also checks that a shape needing more scratch
than the static maximum is refused before anything is launched.

This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import diffusion_transformer_sparse_b200 as pt
from diffusion_transformer_sparse_b200 import build
from tests.helpers import TOL, Case, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pt.lib()


def _call_static(z, grid, window, shift, w, heads, flags=0):
    out = torch.empty_like(z)
    shape = pt.make_shape(z, grid, heads)
    ww = pt.attn_w(w)
    rc = pt.lib().ptdit_window_attn_static(
        ctypes.byref(shape), pt._i3(window), pt._i3(shift), ctypes.byref(ww), flags,
        z.data_ptr(), out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return rc, out


@pytest.mark.parametrize("dtype,grid,D,heads,window,shift", [
    ("bf16", (1, 64, 64), 1152, 16, (1, 8, 8), (0, 4, 4)),
    ("f32", (1, 16, 16), 64, 2, (1, 4, 4), (0, 2, 2)),
])
def test_static_scratch_matches_workspace_entry_point(dtype, grid, D, heads, window, shift):
    first = Case(1, grid, D, heads, dtype)
    second = Case(1, grid, D, heads, dtype, seed_offset=7)
    calls = [(first.z, (0, 0, 0), first.w["wsa"], 0),
             (second.z, shift, second.w["swsa"], 0),
             (first.z, shift, first.w["swsa"], pt.PTDIT_NO_RESIDUAL)]
    for z, sh, w, flags in calls:
        rc, got = _call_static(z, grid, window, sh, w, heads, flags)
        assert rc == 0, pt.lib().ptdit_last_error()
        want = pt.ptdit_window_attn(z, grid, window, sh, w, heads, flags)
        torch.cuda.synchronize()
        assert rel_err(got.double().cpu().numpy(), want.double().cpu().numpy()) <= TOL[dtype]


def test_static_scratch_refuses_oversize_shapes():
    z = torch.empty(1, 128 * 128, 1152, dtype=torch.bfloat16, device="cuda")
    w = tuple(torch.empty(1152, 1152, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    launches = pt.ptdit_launch_count()
    rc, _ = _call_static(z, (1, 128, 128), (1, 8, 8), (0, 4, 4), w, 16)
    assert rc == 4
    assert b"static scratch" in pt.lib().ptdit_last_error()
    assert pt.ptdit_launch_count() == launches
