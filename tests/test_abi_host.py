"""Host-side tests of the C ABI: runs without a GPU.

The library must load, export every function include/ptdit.h declares, size
its workspace, and reject invalid arguments with a status code before it
touches CUDA.
"""
import ctypes
import os
import re

import pytest

import diffusion_transformer_sparse_b200 as pt
from diffusion_transformer_sparse_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return pt.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "ptdit.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ptdit_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 14
    assert set(names) == set(pt.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
    # nm agrees: the symbols are real dynamic exports with C linkage
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", pt.LIB_PATH], capture_output=True,
                         text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}$", out, re.M), n


def test_strerror(L):
    for code in range(9):
        assert L.ptdit_strerror(code)
    assert L.ptdit_strerror(0) == b"ok"


def _shape(**kw):
    d = dict(B=1, F=1, H=16, W=16, D=64, heads=2, dtype=pt.PTDIT_F32)
    d.update(kw)
    return pt.Shape(**d)


def _bytes(L, shape, ratio, window):
    return L.ptdit_workspace_bytes(ctypes.byref(shape), pt._i3(ratio), pt._i3(window))


def test_workspace_bytes(L):
    s = _shape(B=4, H=64, W=64, D=1152, heads=16, dtype=pt.PTDIT_BF16)
    N, M, D, e = 4096, 256, 1152, 2

    def a(x):
        return (x + 255) // 256 * 256

    # bf16 with heads of 72: Q, K and V are stored as (128-row tile, head) blocks of
    # 20 KB (columns padded to 80), V of the row kernel as 32 KB blocks (padded to 128)
    def tiled(rows, blk):
        return 4 * -(-rows // 128) * 16 * blk

    pm, tn = 4 * M * D * e, 4 * N * D * e
    proxy = 3 * a(pm) + 3 * a(max(pm, tiled(M, 20480))) + 2 * a(max(pm, tiled(M, 32768)))
    token = 2 * a(max(tn, tiled(N, 20480))) + a(max(tn, tiled(N, 32768))) + a(tn)
    assert _bytes(L, s, (1, 4, 4), (1, 8, 8)) == proxy + token
    assert _bytes(L, s, None, (1, 8, 8)) == token
    # fp32 keeps every operand row-major
    f = _shape(B=4, H=64, W=64, D=1152, heads=16, dtype=pt.PTDIT_F32)
    assert _bytes(L, f, (1, 4, 4), (1, 8, 8)) == 8 * a(4 * M * D * 4) + 4 * a(4 * N * D * 4)
    assert _bytes(L, s, (1, 3, 4), (1, 8, 8)) == 0      # 64 not divisible by 3
    assert _bytes(L, s, (1, 4, 4), (1, 8, 7)) == 0
    assert _bytes(L, _shape(D=63, heads=2), None, None) == 0


def test_workspace_bytes_with_128_token_windows(L):
    """Windows of 128 tokens in bf16: the size adds the fused kernel's repacked weight
    rows, 16 heads x 224 rows (3 x 72 rounded up to 16) x 1152 columns."""
    s = _shape(B=1, F=2, H=16, W=16, D=1152, heads=16, dtype=pt.PTDIT_BF16)
    plain = _bytes(L, s, None, (1, 8, 8))
    assert _bytes(L, s, None, (2, 8, 8)) == plain + 16 * 224 * 1152 * 2
    f = _shape(B=1, F=2, H=16, W=16, D=1152, heads=16, dtype=pt.PTDIT_F32)
    assert _bytes(L, f, None, (2, 8, 8)) == _bytes(L, f, None, (1, 8, 8))


FAKE = 1 << 20  # an aligned non-null address that is never dereferenced: validation fails first


def _w(p=FAKE):
    return pt.AttnW(p, p + 4096, p + 8192, p + 12288)


def _block(L, shape, ratio=(1, 2, 2), window=(1, 4, 4), shift=(0, 2, 2), w=None, flags=0,
           z_in=FAKE, z_out=FAKE * 64, ws=FAKE * 128, ws_bytes=1 << 40):
    w = w or _w()
    return L.ptdit_block_attn(ctypes.byref(shape) if shape is not None else None,
                              pt._i3(ratio), pt._i3(window), pt._i3(shift), ctypes.byref(w),
                              ctypes.byref(w), ctypes.byref(w), ctypes.byref(w), flags, z_in,
                              z_out, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(shape=None), 1),
    (dict(ratio=None), 1),
    (dict(shift=None), 1),
    (dict(ratio=(1, 3, 2)), 2),
    (dict(window=(1, 5, 4)), 2),
    (dict(shift=(0, 4, 2)), 2),
    (dict(shift=(0, -1, 2)), 2),
    (dict(z_in=0), 1),
    (dict(z_out=FAKE + 8), 7),
    (dict(ws_bytes=1024), 4),
    (dict(z_out=FAKE + 4096), 8),
    (dict(ws=FAKE * 64 + 256), 8),
    (dict(w=pt.AttnW(FAKE, 0, FAKE, FAKE)), 1),
])
def test_block_attn_rejects(L, kw, code):
    shape = kw.pop("shape", _shape())
    assert _block(L, shape, **kw) == code
    assert L.ptdit_last_error()


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), 3),
    (dict(D=65, heads=2), 2),
    (dict(D=1024, heads=4), 2),   # head dim 256
    (dict(B=0), 2),
    (dict(H=0), 2),
])
def test_shape_rejects(L, kw, code):
    assert _block(L, _shape(**kw)) == code


def test_debug_maps_reject(L):
    out = FAKE
    assert L.ptdit_debug_window_map(pt._i3((1, 4, 4)), pt._i3((1, 3, 2)), pt._i3((0, 0, 0)),
                                    out, None, None) == 2
    assert L.ptdit_debug_proxy_map(pt._i3((1, 4, 4)), pt._i3((1, 2, 2)), None, None) == 1


def test_python_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(pt, "_lib", None)
    monkeypatch.setattr(pt, "LIB_PATH", "/nonexistent/libptdit.so")
    with pytest.raises(RuntimeError, match="missing"):
        pt.lib()


# ---------------------------------------------------------------- bf16 tensor-core shapes

@pytest.mark.parametrize("kw,window,msg", [
    (dict(D=176, heads=2, dtype=pt.PTDIT_BF16), (1, 4, 4), b"head width 88"),
    (dict(D=120, heads=2, dtype=pt.PTDIT_BF16), (1, 4, 4), b"multiples of 16"),
    (dict(F=4, H=8, W=12, D=96, heads=4, dtype=pt.PTDIT_BF16), (2, 4, 3), b"24 tokens"),
    (dict(F=2, H=16, W=16, D=64, heads=2, dtype=pt.PTDIT_BF16), (2, 16, 16), b"512 tokens"),
])
def test_bf16_shapes_without_tensor_core_kernel_are_refused(L, kw, window, msg):
    s = _shape(**kw)
    assert _block(L, s, ratio=(1, 2, 2), window=window, shift=(0, 0, 0)) == 2
    assert msg in L.ptdit_last_error()


def test_fp32_takes_the_shapes_bf16_refuses(L):
    # same shape in fp32 passes validation and only fails on the (fake) workspace size
    s = _shape(F=4, H=8, W=12, D=96, heads=4, dtype=pt.PTDIT_F32)
    assert _block(L, s, ratio=(1, 2, 2), window=(2, 4, 3), shift=(0, 0, 0), ws_bytes=16) == 4


# ---------------------------------------------------------------- proxy modes and the complete block

def test_proxy_extract_rejects(L):
    s = _shape()
    r = pt._i3((1, 2, 2))
    assert L.ptdit_proxy_extract(ctypes.byref(s), r, 3, None, FAKE, FAKE * 64, None) == 2
    assert L.ptdit_proxy_extract(ctypes.byref(s), r, pt.PTDIT_PROXY_RANDOM, None, FAKE,
                                 FAKE * 64, None) == 1
    assert L.ptdit_proxy_extract(ctypes.byref(s), r, pt.PTDIT_PROXY_RANDOM, FAKE + 2, FAKE,
                                 FAKE * 64, None) == 7
    assert L.ptdit_proxy_extract(ctypes.byref(s), pt._i3((1, 3, 2)), 1, None, FAKE, FAKE * 64,
                                 None) == 2


def _bw(**kw):
    bw = pt.BlockW()
    for i, m in enumerate(("psa", "cross", "wsa", "swsa", "text")):
        setattr(bw, m, _w(FAKE * (2 + i)))
    for i, k in enumerate(("proxy", "cross", "wsa", "swsa", "text", "mlp")):
        setattr(bw, "norm_" + k, pt.NormW(FAKE * 8 + i * 4096, FAKE * 9 + i * 4096))
    bw.w1, bw.b1, bw.w2, bw.b2 = FAKE * 10, FAKE * 11, FAKE * 12, FAKE * 13
    bw.mlp_hidden, bw.eps = 256, 1e-6
    for k, v in kw.items():
        setattr(bw, k, v)
    return bw


def _pt_block(L, shape, bw, text=FAKE * 14, text_len=7, mode=0, slots=None, ws_bytes=1 << 40):
    return L.ptdit_pt_block(ctypes.byref(shape), pt._i3((1, 2, 2)), pt._i3((1, 4, 4)),
                            pt._i3((0, 2, 2)), ctypes.byref(bw), text, text_len, mode, slots,
                            FAKE * 32, FAKE * 64, FAKE * 128, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(text_len=0), 2),
    (dict(text=0), 1),
    (dict(bw=dict(mlp_hidden=0)), 2),
    (dict(bw=dict(eps=0.0)), 2),
    (dict(bw=dict(eps=2.0)), 2),
    (dict(bw=dict(w1=0)), 1),
    (dict(bw=dict(b2=FAKE * 13 + 4)), 7),
    (dict(mode=2), 1),
    (dict(ws_bytes=4096), 4),
])
def test_pt_block_rejects(L, kw, code):
    bw = _bw(**kw.pop("bw", {}))
    assert _pt_block(L, _shape(), bw, **kw) == code
    assert L.ptdit_last_error()


def test_pt_block_rejects_bf16_mlp_width_not_multiple_of_16(L):
    s = _shape(D=64, heads=2, dtype=pt.PTDIT_BF16)
    assert _pt_block(L, s, _bw(mlp_hidden=200)) == 2
    assert b"multiples of 16" in L.ptdit_last_error()


def test_pt_block_workspace_covers_the_attention_path(L):
    s = _shape(B=2, F=2, H=16, W=16, D=1152, heads=16, dtype=pt.PTDIT_BF16)
    attn = _bytes(L, s, (1, 4, 4), (2, 8, 8))
    n = L.ptdit_pt_block_workspace_bytes(ctypes.byref(s), pt._i3((1, 4, 4)), 120, 4608)
    # plus the norm output, the MLP hidden layer and the text K / V blocks
    assert n >= attn + 2 * 512 * 4608 * 2 + 2 * 512 * 1152 * 2
    assert L.ptdit_pt_block_workspace_bytes(ctypes.byref(s), pt._i3((1, 4, 4)), 0, 4608) == 0


# ---------------------------------------------------------------- backward entry points (host checks)

def _bshape(**kw):
    d = dict(B=1, F=1, H=16, W=16, D=128, heads=2, dtype=pt.PTDIT_BF16)
    d.update(kw)
    return pt.Shape(**d)


def _wg(base):
    return pt.AttnWgrad(base, base + 0x100000, base + 0x200000, base + 0x300000)


def _bwd(L, shape, dw, window=(1, 8, 8), z_in=FAKE * 20, dz_out=FAKE * 21, dz_in=FAKE * 22,
         ws_bytes=1 << 40):
    g = None if dw is None else ctypes.byref(dw)
    return L.ptdit_window_attn_bwd(ctypes.byref(shape), pt._i3(window), pt._i3((0, 4, 4)),
                                   ctypes.byref(_w(FAKE * 2)), 0, z_in, dz_out, dz_in, g,
                                   FAKE * 128, ws_bytes, None)


def test_window_bwd_workspace_bytes(L):
    s = _bshape(B=4, H=64, W=64, D=1152, heads=16)
    n = L.ptdit_window_attn_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 8, 8)))
    tq = 4 * 32 * 16 * 20480          # Q, K, V, dA window tiles (32 tiles per item)
    tn = 4 * 4096 * 1152 * 2
    assert n == 4 * tq + tn + 3 * tn + 1152 * 1152 * 2 + 3 * 1152 * 1152 * 2
    t = L.ptdit_tcm_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 8, 8)))
    assert t == n + 2 * tn + 3 * tq + tn  # plus z^, dL/dz^ and WSA's kept Q, K, V and A
    assert L.ptdit_window_attn_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 3, 8))) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(shape=dict(dtype=pt.PTDIT_F32)), 3),          # bf16 only
    (dict(shape=dict(D=64, heads=1)), 2),                # D a multiple of 128
    (dict(shape=dict(D=128, heads=1)), 2),               # head width 128: no bf16 kernel
    (dict(window=(1, 4, 2)), 2),                         # a window of 8 tokens
    (dict(dw=None), 1),
    (dict(dw="null_dwk"), 1),
    (dict(dw="misaligned_dwv"), 7),
    (dict(dw="dwq_on_dz_in"), 8),
    (dict(dz_in=FAKE * 21), 8),                          # dz_in is dz_out
    (dict(dz_out=0), 1),
    (dict(ws_bytes=4096), 4),
])
def test_window_bwd_rejects(L, kw, code):
    """Every case fails validation on the host: nothing is launched."""
    s = _bshape(**kw.pop("shape", {}))
    dw = _wg(FAKE * 40)
    special = kw.pop("dw", dw)
    if special == "null_dwk":
        dw.dwk = 0
    elif special == "misaligned_dwv":
        dw.dwv = FAKE * 40 + 0x200004
    elif special == "dwq_on_dz_in":
        dw.dwq = FAKE * 22
    elif special is None:
        dw = None
    assert _bwd(L, s, dw, **kw) == code
    assert L.ptdit_last_error()


def test_tcm_bwd_rejects_overlapping_gradients(L):
    s = _bshape()
    a, b = _wg(FAKE * 40), _wg(FAKE * 40 + 0x300000)  # b.dwq is a.dwo
    rc = L.ptdit_tcm_bwd(ctypes.byref(s), pt._i3((1, 8, 8)), pt._i3((0, 4, 4)),
                         ctypes.byref(_w(FAKE * 2)), ctypes.byref(_w(FAKE * 3)), 0, FAKE * 20,
                         FAKE * 21, FAKE * 22, ctypes.byref(a), ctypes.byref(b), FAKE * 128,
                         1 << 40, None)
    assert rc == 8
    assert b"overlap" in L.ptdit_last_error()


def _giim_bwd(L, shape, dwp, dwc, ratio=(1, 2, 2), z_in=FAKE * 20, dz_out=FAKE * 21,
              dz_in=FAKE * 22, ws_bytes=1 << 40):
    gp = None if dwp is None else ctypes.byref(dwp)
    return L.ptdit_giim_bwd(ctypes.byref(shape), pt._i3(ratio), ctypes.byref(_w(FAKE * 2)),
                            ctypes.byref(_w(FAKE * 3)), 0, z_in, dz_out, dz_in, gp,
                            ctypes.byref(dwc), FAKE * 128, ws_bytes, None)


def test_giim_and_block_bwd_workspace_bytes(L):
    s = _bshape(B=4, H=64, W=64, D=1152, heads=16)
    g = L.ptdit_giim_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 4, 4)))
    t = L.ptdit_tcm_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 8, 8)))
    f = _bytes(L, s, (1, 4, 4), (1, 8, 8))
    tn = 4 * 4096 * 1152 * 2
    # at least the proxies' Q/K/V blocks, the latents' Q and dA blocks and the
    # stacked dQ blocks (two key tiles of 128 proxies: 256 proxies per item)
    assert g >= 2 * 4 * 32 * 16 * 20480 + 4 * 4096 * 2 * 1152 * 2
    n = L.ptdit_block_attn_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 4, 4)),
                                               pt._i3((1, 8, 8)))
    assert n == 2 * tn + g + t  # z1, dL/dz1, GIIM's backward area, TCM's backward area
    assert f > 0
    assert L.ptdit_giim_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 3, 4))) == 0
    assert L.ptdit_block_attn_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 4, 4)),
                                                  pt._i3((1, 3, 8))) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(shape=dict(dtype=pt.PTDIT_F32)), 3),          # bf16 only
    (dict(shape=dict(D=64, heads=1)), 2),                # D a multiple of 128
    (dict(ratio=(1, 3, 2)), 2),                          # ratio does not divide the grid
    (dict(shape=dict(H=512, W=512), ratio=(1, 1, 2)), 2),  # 131072 proxies: above 8192
    (dict(dwp=None), 1),
    (dict(dwp="on_dw_cross"), 8),
    (dict(dz_in=FAKE * 21), 8),                          # dz_in is dz_out
    (dict(z_in=0), 1),
    (dict(ws_bytes=4096), 4),
])
def test_giim_bwd_rejects(L, kw, code):
    """Every case fails validation on the host: nothing is launched."""
    s = _bshape(**kw.pop("shape", {}))
    dwp, dwc = _wg(FAKE * 40), _wg(FAKE * 80)
    special = kw.pop("dwp", dwp)
    if special == "on_dw_cross":
        dwp = _wg(FAKE * 80 + 0x100000)  # dwp.dwq is dwc.dwk
    elif special is None:
        dwp = None
    assert _giim_bwd(L, s, dwp, dwc, **kw) == code
    assert L.ptdit_last_error()


def test_block_attn_bwd_rejects(L):
    s = _bshape()
    g = [_wg(FAKE * (40 + 8 * i)) for i in range(4)]

    def call(shape=s, grads=g, window=(1, 8, 8), ws_bytes=1 << 40):
        return L.ptdit_block_attn_bwd(
            ctypes.byref(shape), pt._i3((1, 2, 2)), pt._i3(window), pt._i3((0, 4, 4)),
            *[ctypes.byref(_w(FAKE * (2 + i))) for i in range(4)], 0, FAKE * 20, FAKE * 21,
            FAKE * 22, *[ctypes.byref(x) for x in grads], FAKE * 128, ws_bytes, None)

    assert call(shape=_bshape(dtype=pt.PTDIT_F32)) == 3
    assert call(window=(1, 4, 2)) == 2                   # a window of 8 tokens
    assert call(ws_bytes=4096) == 4
    clash = [g[0], g[1], g[2], _wg(FAKE * 40 + 0x200000)]  # dw_swsa.dwq is dw_psa.dwv
    assert call(grads=clash) == 8
    assert b"dw_swsa and dw_psa overlap" in L.ptdit_last_error()


def test_training_pair_workspace_and_refusals(L):
    """The training pair's workspace adds SWSA's kept Q, K, V tiles and attention output to
    the whole-path backward's; both calls validate on the host first."""
    s = _bshape(B=4, H=64, W=64, D=1152, heads=16)
    b = L.ptdit_block_attn_bwd_workspace_bytes(ctypes.byref(s), pt._i3((1, 4, 4)), pt._i3((1, 8, 8)))
    t = L.ptdit_block_attn_train_workspace_bytes(ctypes.byref(s), pt._i3((1, 4, 4)), pt._i3((1, 8, 8)))
    tq = 4 * 32 * 16 * 20480  # window tiles of 72 columns padded to 80, 32 tiles per item
    assert t == b + 3 * tq + 4 * 4096 * 1152 * 2
    small = _bshape()
    args = (ctypes.byref(small), pt._i3((1, 2, 2)), pt._i3((1, 8, 8)), pt._i3((0, 4, 4)),
            *[ctypes.byref(_w(FAKE * (2 + i))) for i in range(4)], 0)
    assert L.ptdit_block_attn_fwd_train(*args, FAKE * 20, FAKE * 21, FAKE * 128, 4096, None) == 4
    assert L.ptdit_block_attn_fwd_train(*args, FAKE * 20, FAKE * 20, FAKE * 128, 1 << 40, None) == 8
    g = [_wg(FAKE * (40 + 8 * i)) for i in range(4)]
    assert L.ptdit_block_attn_bwd_saved(*args, FAKE * 20, FAKE * 21, FAKE * 22,
                                        *[ctypes.byref(x) for x in g], FAKE * 128, 4096, None) == 4
    f32 = _bshape(dtype=pt.PTDIT_F32)
    assert L.ptdit_block_attn_fwd_train(ctypes.byref(f32), *args[1:], FAKE * 20, FAKE * 21,
                                        FAKE * 128, 1 << 40, None) == 3


def test_window_fused_setting_is_per_thread(L):
    """ptdit_window_fused: off by default, 0/1 set it, anything else only reads it, and
    the setting belongs to the calling host thread."""
    import threading
    assert L.ptdit_window_fused(-1) == 0
    assert L.ptdit_window_fused(1) == 0
    assert L.ptdit_window_fused(2) == 1  # reads only
    seen = []
    t = threading.Thread(target=lambda: seen.append(L.ptdit_window_fused(-1)))
    t.start()
    t.join()
    assert seen == [0]  # another thread still has the default
    assert L.ptdit_window_fused(0) == 1
    assert L.ptdit_window_fused(-1) == 0
