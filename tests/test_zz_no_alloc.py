"""ptdit_window_attn_static: window attention for callers that cannot allocate.

Some callers cannot call cudaMalloc (it may synchronise the device, it may be
forbidden where they run, or they only receive input and output buffers from a
framework whose allocator they cannot reach).  For them the library offers one
entry point whose scratch is a static device array inside the library.  This
test calls it through the C ABI several times in a row, with different inputs,
weights, shifts and grid sizes, and checks each result bit for bit against
ptdit_window_attn given a caller-allocated workspace and, within the parity
tolerance, against the float64 oracle.  It also checks that a shape needing more scratch
than the static maximum is refused before anything is launched.

This file is collected last on purpose.
"""
import ctypes

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
    """Calls in a row with different inputs, weights and shifts: each result is bit
    for bit the result of ptdit_window_attn with a caller-allocated workspace (the
    same kernels on the same inputs), and within the tolerance of the oracle."""
    first = Case(1, grid, D, heads, dtype)
    second = Case(1, grid, D, heads, dtype, seed_offset=7)
    calls = [(first, (0, 0, 0), "wsa", 0),
             (second, shift, "swsa", 0),
             (first, shift, "swsa", pt.PTDIT_NO_RESIDUAL)]
    for c, sh, m, flags in calls:
        rc, got = _call_static(c.z, grid, window, sh, c.w[m], heads, flags)
        assert rc == 0, pt.lib().ptdit_last_error()
        want = pt.ptdit_window_attn(c.z, grid, window, sh, c.w[m], heads, flags)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
        ref = O.window_self_attention(c.z64[0], grid, window, sh, c.w64[m], heads,
                                      residual=not flags & pt.PTDIT_NO_RESIDUAL)
        assert rel_err(c.out64(got)[0], ref) <= TOL[dtype]


def test_static_scratch_after_a_larger_call():
    """A large bf16 call leaves the shared scratch full of its data; a following call
    on a small grid with an odd number of 64-token windows (3 windows: the second
    128-row tile half empty, rows that must read as zeros) is still bit for bit the
    workspace entry point's result and matches the oracle."""
    big = Case(1, (1, 64, 64), 1152, 16, "bf16", seed_offset=3)
    rc, _ = _call_static(big.z, big.grid, (1, 8, 8), (0, 4, 4), big.w["swsa"], 16)
    assert rc == 0, pt.lib().ptdit_last_error()
    small = Case(1, (1, 8, 24), 1152, 16, "bf16")
    for sh in [(0, 0, 0), (0, 4, 4)]:
        rc, got = _call_static(small.z, small.grid, (1, 8, 8), sh, small.w["wsa"], 16)
        assert rc == 0, pt.lib().ptdit_last_error()
        want = pt.ptdit_window_attn(small.z, small.grid, (1, 8, 8), sh, small.w["wsa"], 16)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
        ref = O.window_self_attention(small.z64[0], small.grid, (1, 8, 8), sh, small.w64["wsa"],
                                      16)
        assert rel_err(small.out64(got)[0], ref) <= TOL["bf16"]


def test_static_scratch_refuses_oversize_shapes():
    z = torch.empty(1, 128 * 128, 1152, dtype=torch.bfloat16, device="cuda")
    w = tuple(torch.empty(1152, 1152, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    launches = pt.ptdit_launch_count()
    rc, _ = _call_static(z, (1, 128, 128), (1, 8, 8), (0, 4, 4), w, 16)
    assert rc == 4
    assert b"static scratch" in pt.lib().ptdit_last_error()
    assert pt.ptdit_launch_count() == launches
