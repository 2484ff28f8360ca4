"""Failure detection without a GPU fault.

Host side (CPU): PTDIT_FAULT=workspace makes every workspace-taking call
report PTDIT_ERR_WORKSPACE before anything is launched.  GPU side: a bounded
device wait on a barrier that nothing releases gives up after its limit,
records PTDIT_ERR_TIMEOUT in the library's status word, and the context stays
usable for the next call; PTDIT_FAULT=launch refuses launches on the host.
Nothing here traps, faults or hangs a GPU.
"""
import ctypes
import os
import subprocess
import sys
import textwrap

import pytest

import diffusion_transformer_sparse_b200 as pt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 20  # aligned, never dereferenced: the call fails before any launch


def _run(code, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, "-c", textwrap.dedent(code)], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=300)


def test_injected_workspace_fault_is_reported_on_the_host():
    code = """
        import ctypes
        import diffusion_transformer_sparse_b200 as pt
        from diffusion_transformer_sparse_b200 import build
        build.build()
        L = pt.lib()
        F = 1 << 20
        s = pt.Shape(B=1, F=1, H=16, W=16, D=64, heads=2, dtype=pt.PTDIT_F32)
        w = pt.AttnW(F, F + 4096, F + 8192, F + 12288)
        n = L.ptdit_workspace_bytes(ctypes.byref(s), pt._i3((1, 2, 2)), pt._i3((1, 4, 4)))
        before = L.ptdit_launch_count()
        rc = L.ptdit_window_attn(ctypes.byref(s), pt._i3((1, 4, 4)), pt._i3((0, 2, 2)),
                                 ctypes.byref(w), 0, F + (1 << 20), F + (2 << 20), F + (4 << 20),
                                 n, None)
        print(rc, L.ptdit_launch_count() - before, L.ptdit_last_error().decode())
    """
    out = _run(code, {"PTDIT_FAULT": "workspace"})
    assert out.returncode == 0, out.stderr
    rc, launched, msg = out.stdout.strip().split(" ", 2)
    assert int(rc) == pt.PTDIT_ERR_WORKSPACE and int(launched) == 0
    assert "PTDIT_FAULT" in msg


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_reports_timeout():
    import torch
    pt.lib()
    assert pt.ptdit_device_status(reset=True) in (pt.PTDIT_OK, pt.PTDIT_ERR_TIMEOUT)
    assert pt.ptdit_device_status() == pt.PTDIT_OK
    pt.ptdit_debug_timeout(2_000_000)  # 2 ms
    torch.cuda.synchronize()
    assert pt.ptdit_device_status(reset=True) == pt.PTDIT_ERR_TIMEOUT
    assert pt.ptdit_device_status() == pt.PTDIT_OK
    # the context is still usable: a regular call runs and leaves the word clear
    from tests.helpers import Case, rel_err, TOL
    import oracle as O
    c = Case(1, (1, 16, 16), 64, 2, "f32")
    out = c.out64(pt.ptdit_window_attn(c.z, (1, 16, 16), (1, 4, 4), (0, 2, 2), c.w["wsa"], 2))
    want = O.window_self_attention(c.z64[0], (1, 16, 16), (1, 4, 4), (0, 2, 2), c.w64["wsa"], 2)
    assert rel_err(out[0], want) <= TOL["f32"]
    assert pt.ptdit_device_status() == pt.PTDIT_OK


@pytest.mark.gpu
def test_window_kernel_gives_up_as_whole_warps():
    """The window-attention kernel with a 1 ns limit on its waits for work: the
    waits give up (the loader and softmax warps decide per warp, so no lane is
    left behind at a warp-collective TMEM access), the kernel records
    PTDIT_ERR_TIMEOUT and returns, and the next regular call matches the oracle."""
    import torch
    import oracle as O
    from tests.helpers import Case, rel_err, TOL
    pt.lib()
    grid, window, shift = (1, 64, 64), (1, 8, 8), (0, 4, 4)
    c = Case(1, grid, 1152, 16, "bf16")
    pt.ptdit_device_status(reset=True)
    pt.ptdit_debug_wait_limit(1)
    try:
        pt.ptdit_window_attn(c.z, grid, window, shift, c.w["swsa"], 16)
        torch.cuda.synchronize()
    finally:
        pt.ptdit_debug_wait_limit(0)
    assert pt.ptdit_device_status(reset=True) == pt.PTDIT_ERR_TIMEOUT
    assert pt.ptdit_device_status() == pt.PTDIT_OK
    out = c.out64(pt.ptdit_window_attn(c.z, grid, window, shift, c.w["swsa"], 16))
    want = O.window_self_attention(c.z64[0], grid, window, shift, c.w64["swsa"], 16)
    assert rel_err(out[0], want) <= TOL["bf16"]
    assert pt.ptdit_device_status() == pt.PTDIT_OK


@pytest.mark.gpu
def test_injected_launch_fault_launches_nothing():
    code = """
        import torch
        import diffusion_transformer_sparse_b200 as pt
        from tests.helpers import Case
        c = Case(1, (1, 16, 16), 64, 2, "f32")
        before = pt.ptdit_launch_count()
        try:
            pt.ptdit_window_attn(c.z, (1, 16, 16), (1, 4, 4), (0, 2, 2), c.w["wsa"], 2)
            print("no error")
        except pt.PtditError as e:
            print(e.code, pt.ptdit_launch_count() - before)
    """
    out = _run(code, {"PTDIT_FAULT": "launch"})
    assert out.returncode == 0, out.stderr
    rc, launched = out.stdout.split()
    assert int(rc) == pt.PTDIT_ERR_CUDA and int(launched) == 0


def test_timeout_limit_is_validated():
    pt.lib()
    assert pt.lib().ptdit_debug_timeout(0, None) == pt.PTDIT_ERR_SHAPE
    assert pt.lib().ptdit_debug_timeout(20_000_000_000, None) == pt.PTDIT_ERR_SHAPE
    assert pt.lib().ptdit_debug_wait_limit(-1) == pt.PTDIT_ERR_SHAPE
    assert pt.lib().ptdit_debug_wait_limit(20_000_000_000) == pt.PTDIT_ERR_SHAPE
    assert pt.lib().ptdit_debug_wait_limit(0) == pt.PTDIT_OK
