"""Backward of one TCM branch (ptdit_window_attn_bwd) on the GPU against the
float64 oracle's hand-derived gradients (pinned on the CPU by finite
differences and autograd): dL/dz and the four weight gradients, whole tensors,
at shapes that reach every window size, head width, the roll's wrap masks and a
ragged last tile, and at a full-size workload in the bench's launch
configuration (persistent kernels with many units per CTA, split-K weight
gradients over all tokens)."""
import numpy as np
import pytest
import torch

import diffusion_transformer_sparse_b200 as pt
import oracle as O
from diffusion_transformer_sparse_b200 import build, synth
from tests.helpers import TOL, Case, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pt.lib()


def _dout(B, N, D, seed=500):
    return torch.stack([synth.latent(N, D, seed + b, "bf16") for b in range(B)])


def _check(c, window, shift, flags=0):
    dout_cpu = _dout(c.B, c.N, c.D)
    dz, dw = pt.ptdit_window_attn_bwd(c.z, dout_cpu.cuda(), c.grid, window, shift, c.w["wsa"],
                                      c.heads, flags)
    dz = c.out64(dz)
    dw = [c.out64(x) for x in dw]
    g64 = synth.as_f64(dout_cpu)
    want_w = [np.zeros((c.D, c.D)) for _ in range(4)]
    for b in range(c.B):
        wdz, wdw = O.window_self_attention_bwd(c.z64[b], c.grid, window, shift, c.w64["wsa"],
                                               c.heads, g64[b], residual=not flags)
        assert rel_err(dz[b], wdz) <= TOL["bf16"], ("dz", b)
        for i in range(4):
            want_w[i] += wdw[i]
    for i, name in enumerate(("dWq", "dWk", "dWv", "dWo")):
        assert rel_err(dw[i], want_w[i]) <= TOL["bf16"], name


CASES = [  # grid, D, heads, window, shift
    ((1, 16, 16), 128, 2, (1, 8, 8), (0, 0, 0)),    # 2D windows of 64, two per tile, d = 64
    ((1, 16, 16), 128, 2, (1, 8, 8), (0, 4, 4)),    # the same shifted: wrap masks
    ((2, 16, 16), 256, 4, (2, 8, 8), (1, 4, 4)),    # 3D windows of 128 tokens
    ((2, 8, 16), 1152, 16, (2, 8, 8), (1, 4, 4)),   # d = 72: V's ones column
    ((1, 24, 8), 1152, 16, (1, 8, 8), (0, 4, 4)),   # 3 windows: the last tile half empty
    ((1, 16, 16), 128, 4, (1, 4, 4), (0, 2, 2)),    # windows of 16 (eight per tile), d = 32
    ((1, 16, 32), 128, 2, (1, 4, 8), (0, 2, 4)),    # windows of 32 (four per tile)
    ((2, 16, 16), 640, 8, (2, 8, 8), (1, 4, 4)),    # d = 80
]


@pytest.mark.parametrize("grid,D,heads,window,shift", CASES)
def test_window_bwd_small(grid, D, heads, window, shift):
    c = Case(1, grid, D, heads, "bf16")
    _check(c, window, shift)


def test_window_bwd_without_residual():
    c = Case(1, (2, 16, 16), 256, 4, "bf16")
    _check(c, (2, 8, 8), (1, 4, 4), pt.PTDIT_NO_RESIDUAL)


def test_window_bwd_full_size_1024px():
    """t2i 1024 px: B = 4 items of 64 x 64 tokens, D = 1152, 16 heads, windows of 8 x 8,
    shifted by half a window; 2048 units over 148 CTAs, weight gradients over 16384 tokens."""
    c = Case(4, (1, 64, 64), 1152, 16, "bf16")
    _check(c, (1, 8, 8), (0, 4, 4))


def test_window_bwd_full_size_t2v():
    """t2v: 16 x 32 x 48 tokens, 3D windows of 2 x 8 x 8 = 128 tokens, shifted."""
    c = Case(1, (16, 32, 48), 1152, 16, "bf16")
    _check(c, (2, 8, 8), (1, 4, 4))


def test_window_bwd_refuses_what_it_does_not_run():
    z = torch.zeros(1, 256, 64, dtype=torch.bfloat16, device="cuda")
    w = tuple(torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    with pytest.raises(pt.PtditError) as e:  # D not a multiple of 128
        pt.ptdit_window_attn_bwd(z, z.clone(), (1, 16, 16), (1, 8, 8), (0, 0, 0), w, 1)
    assert e.value.code == pt.PTDIT_ERR_SHAPE
    z32 = torch.zeros(1, 256, 128, dtype=torch.float32, device="cuda")
    w32 = tuple(torch.zeros(128, 128, dtype=torch.float32, device="cuda") for _ in range(4))
    with pytest.raises(pt.PtditError) as e:  # fp32
        pt.ptdit_window_attn_bwd(z32, z32.clone(), (1, 16, 16), (1, 8, 8), (0, 0, 0), w32, 2)
    assert e.value.code == pt.PTDIT_ERR_DTYPE


@pytest.mark.parametrize("grid,D,heads,window,shift,B", [
    ((2, 16, 16), 256, 4, (2, 8, 8), (1, 4, 4), 1),
    ((1, 64, 64), 1152, 16, (1, 8, 8), (0, 4, 4), 2),
])
def test_tcm_bwd(grid, D, heads, window, shift, B):
    """Both TCM branches: dL/dz and each module's weight gradients."""
    c = Case(B, grid, D, heads, "bf16")
    dout_cpu = _dout(c.B, c.N, c.D)
    dz, dwa, dwb = pt.ptdit_tcm_bwd(c.z, dout_cpu.cuda(), c.grid, window, shift, c.w["wsa"],
                                    c.w["swsa"], c.heads)
    dz = c.out64(dz)
    g64 = synth.as_f64(dout_cpu)
    want_a = [np.zeros((c.D, c.D)) for _ in range(4)]
    want_b = [np.zeros((c.D, c.D)) for _ in range(4)]
    for b in range(c.B):
        wdz, wa, wb = O.tcm_bwd(c.z64[b], c.grid, window, shift, c.w64["wsa"], c.w64["swsa"],
                                c.heads, g64[b])
        assert rel_err(dz[b], wdz) <= TOL["bf16"], ("dz", b)
        for i in range(4):
            want_a[i] += wa[i]
            want_b[i] += wb[i]
    for i in range(4):
        assert rel_err(c.out64(dwa[i]), want_a[i]) <= TOL["bf16"], ("wsa", i)
        assert rel_err(c.out64(dwb[i]), want_b[i]) <= TOL["bf16"], ("swsa", i)



# ---------------------------------------------------------------- GIIM

def _proxy_kappa(z64, grid, ratio, Wp, heads, proxy_residual):
    """max |column mean| / max |deviation| of the PSA output P' (the cross keys' source).

    P' stores in bf16 within 2^-8 of each element, i.e. within 2^-8 |mean| absolute,
    while dWq and dWk of the cross-attention depend only on the proxies' deviations
    from their mean (the softmax ignores a shift common to all keys): their error
    relative to their size is of order 2^-8 kappa."""
    Pa = O.averaging(z64, grid, ratio)
    Pp = O.attention_heads(Pa @ Wp[0].T, Pa @ Wp[1].T, Pa @ Wp[2].T, heads) @ Wp[3].T
    if proxy_residual:
        Pp = Pp + Pa
    m = Pp.mean(axis=0)
    return float(np.abs(m).max() / np.abs(Pp - m).max())


def _check_giim(c, ratio, flags=0):
    dout_cpu = _dout(c.B, c.N, c.D)
    dz, dwp, dwc = pt.ptdit_giim_bwd(c.z, dout_cpu.cuda(), c.grid, ratio, c.w["psa"], c.w["cross"],
                                     c.heads, flags)
    dz = c.out64(dz)
    g64 = synth.as_f64(dout_cpu)
    want_p = [np.zeros((c.D, c.D)) for _ in range(4)]
    want_c = [np.zeros((c.D, c.D)) for _ in range(4)]
    kappa = 0.0
    for b in range(c.B):
        kappa = max(kappa, _proxy_kappa(c.z64[b], c.grid, ratio, c.w64["psa"], c.heads,
                                        bool(flags & pt.PTDIT_PROXY_RESIDUAL)))
        wdz, wp, wc = O.giim_bwd(c.z64[b], c.grid, ratio, c.w64["psa"], c.w64["cross"], c.heads,
                                 g64[b], proxy_residual=bool(flags & pt.PTDIT_PROXY_RESIDUAL),
                                 residual=not flags & pt.PTDIT_NO_RESIDUAL)
        assert rel_err(dz[b], wdz) <= TOL["bf16"], ("dz", b)
        for i in range(4):
            want_p[i] += wp[i]
            want_c[i] += wc[i]
    # the cross dWq, dWk: the bf16 tolerance plus twice the storage bound 2^-8 kappa
    tol_qk = TOL["bf16"] + 2 * 2.0 ** -8 * kappa
    for i, name in enumerate(("dWq", "dWk", "dWv", "dWo")):
        assert rel_err(c.out64(dwp[i]), want_p[i]) <= TOL["bf16"], ("psa", name)
        tol = tol_qk if i < 2 else TOL["bf16"]
        assert rel_err(c.out64(dwc[i]), want_c[i]) <= tol, ("cross", name, kappa)


GIIM_CASES = [  # grid, D, heads, ratio
    ((1, 16, 16), 128, 2, (1, 4, 4)),     # 16 proxies: one ragged key tile, d = 64
    ((2, 16, 16), 256, 4, (1, 2, 2)),     # 128 proxies: one full key tile
    ((2, 16, 32), 1152, 16, (1, 2, 2)),   # 256 proxies: two key tiles, d = 72
    ((1, 24, 40), 640, 8, (1, 2, 2)),     # 240 proxies, 960 latents: ragged tiles, d = 80
    ((1, 16, 16), 128, 4, (1, 1, 1)),     # every token a proxy (256 x 256), d = 32
]


@pytest.mark.parametrize("grid,D,heads,ratio", GIIM_CASES)
def test_giim_bwd_small(grid, D, heads, ratio):
    _check_giim(Case(1, grid, D, heads, "bf16"), ratio)


@pytest.mark.parametrize("flags", ["proxy_residual", "no_residual"])
def test_giim_bwd_flags(flags):
    f = pt.PTDIT_PROXY_RESIDUAL if flags == "proxy_residual" else pt.PTDIT_NO_RESIDUAL
    _check_giim(Case(1, (2, 16, 32), 1152, 16, "bf16"), (1, 2, 2), f)


def test_giim_bwd_full_size_1024px():
    """t2i 1024 px: B = 4 items of 64 x 64 latents, 256 proxies each, D = 1152."""
    _check_giim(Case(4, (1, 64, 64), 1152, 16, "bf16"), (1, 4, 4))


# ---------------------------------------------------------------- the whole path

def _check_path(c, ratio, window, shift, dout_cpu, dz, dw, flags=0):
    """dz and the four modules' weight gradients of the whole path against the oracle."""
    dz = c.out64(dz)
    g64 = synth.as_f64(dout_cpu)
    mods = ("psa", "cross", "wsa", "swsa")
    want = [[np.zeros((c.D, c.D)) for _ in range(4)] for _ in mods]
    kappa = 0.0
    pres = bool(flags & pt.PTDIT_PROXY_RESIDUAL)
    for b in range(c.B):
        wdz, *ww = O.block_attn_bwd(c.z64[b], c.grid, ratio, window, shift,
                                    *[c.w64[m] for m in mods], c.heads, g64[b],
                                    proxy_residual=pres,
                                    residual=not flags & pt.PTDIT_NO_RESIDUAL)
        assert rel_err(dz[b], wdz) <= TOL["bf16"], ("dz", b)
        for m in range(4):
            for i in range(4):
                want[m][i] += ww[m][i]
        kappa = max(kappa, _proxy_kappa(c.z64[b], c.grid, ratio, c.w64["psa"], c.heads, pres))
    tol_qk = TOL["bf16"] + 2 * 2.0 ** -8 * kappa
    for m, name in enumerate(mods):
        # without the residual stream z1 is the cross-attention output alone, nearly the
        # same row for every token, so the window modules' scores are nearly equal across
        # keys and their dWq, dWk nearly vanish: there each gradient's error is measured
        # against its module's gradient scale (the largest entry of its four matrices)
        scale = max(np.abs(x).max() for x in want[m]) if flags & pt.PTDIT_NO_RESIDUAL else None
        for i in range(4):
            tol = tol_qk if (name == "cross" and i < 2) else TOL["bf16"]
            got = c.out64(dw[m][i])
            err = (rel_err(got, want[m][i]) if scale is None
                   else float(np.abs(got - want[m][i]).max() / scale))
            assert err <= tol, (name, i, kappa, err)


@pytest.mark.parametrize("grid,D,heads,ratio,window,shift,B", [
    ((2, 16, 32), 1152, 16, (1, 2, 2), (2, 8, 8), (1, 4, 4), 1),
    # t2i 1024 px (two of its four items): 64 x 64 latents, 256 proxies, 8 x 8 windows
    ((1, 64, 64), 1152, 16, (1, 4, 4), (1, 8, 8), (0, 4, 4), 2),
    # t2v in full: 16 x 32 x 48 latents, 1536 proxies (12 key tiles summed), 3D windows
    ((16, 32, 48), 1152, 16, (1, 4, 4), (2, 8, 8), (1, 4, 4), 1),
])
def test_block_attn_bwd(grid, D, heads, ratio, window, shift, B):
    """GIIM then TCM: dL/dz and the four modules' weight gradients."""
    c = Case(B, grid, D, heads, "bf16")
    dout_cpu = _dout(c.B, c.N, c.D)
    dz, *dw = pt.ptdit_block_attn_bwd(c.z, dout_cpu.cuda(), c.grid, ratio, window, shift,
                                      c.w["psa"], c.w["cross"], c.w["wsa"], c.w["swsa"], c.heads)
    _check_path(c, ratio, window, shift, dout_cpu, dz, dw)


@pytest.mark.parametrize("grid,D,heads,ratio,window,shift,B", [
    ((2, 16, 32), 1152, 16, (1, 2, 2), (2, 8, 8), (1, 4, 4), 1),
    ((1, 64, 64), 1152, 16, (1, 4, 4), (1, 8, 8), (0, 4, 4), 2),
])
def test_block_attn_train_pair(grid, D, heads, ratio, window, shift, B):
    """The forward that keeps its activations, then the backward from them: the forward's
    output and every gradient against the oracle, and the gradients against the backward
    that recomputes the forward (same kernels; only the order of the fp32 reductions of
    dK, dV and the weight gradients differs)."""
    c = Case(B, grid, D, heads, "bf16")
    mods = ("psa", "cross", "wsa", "swsa")
    W = [c.w[m] for m in mods]
    ws = pt.train_workspace(c.z, grid, ratio, window, heads)
    out = c.out64(pt.ptdit_block_attn_fwd_train(c.z, grid, ratio, window, shift, *W, heads, ws))
    for b in range(B):
        want = O.block_attn(c.z64[b], grid, ratio, window, shift, *[c.w64[m] for m in mods], heads)
        assert rel_err(out[b], want) <= TOL["bf16"], ("forward", b)
    dout_cpu = _dout(c.B, c.N, c.D)
    dz, *dw = pt.ptdit_block_attn_bwd_saved(c.z, dout_cpu.cuda(), grid, ratio, window, shift, *W,
                                            heads, ws)
    _check_path(c, ratio, window, shift, dout_cpu, dz, dw)
    dz2, *dw2 = pt.ptdit_block_attn_bwd(c.z, dout_cpu.cuda(), grid, ratio, window, shift, *W, heads)
    assert rel_err(c.out64(dz), c.out64(dz2)) <= 1e-2
    for m in range(4):
        for i in range(4):
            assert rel_err(c.out64(dw[m][i]), c.out64(dw2[m][i])) <= 1e-2, (mods[m], i)


@pytest.mark.parametrize("flags", ["proxy_residual", "no_residual"])
def test_block_attn_bwd_flags(flags):
    """The whole path with the proxy residual and without the latent residuals, through
    both the recomputing backward and the training pair."""
    f = pt.PTDIT_PROXY_RESIDUAL if flags == "proxy_residual" else pt.PTDIT_NO_RESIDUAL
    grid, ratio, window, shift = (2, 16, 32), (1, 2, 2), (2, 8, 8), (1, 4, 4)
    c = Case(1, grid, 1152, 16, "bf16")
    W = [c.w[m] for m in ("psa", "cross", "wsa", "swsa")]
    dout_cpu = _dout(c.B, c.N, c.D)
    dz, *dw = pt.ptdit_block_attn_bwd(c.z, dout_cpu.cuda(), grid, ratio, window, shift, *W,
                                      c.heads, f)
    _check_path(c, ratio, window, shift, dout_cpu, dz, dw, f)
    ws = pt.train_workspace(c.z, grid, ratio, window, c.heads)
    out = c.out64(pt.ptdit_block_attn_fwd_train(c.z, grid, ratio, window, shift, *W, c.heads, ws, f))
    want = O.block_attn(c.z64[0], grid, ratio, window, shift,
                        *[c.w64[m] for m in ("psa", "cross", "wsa", "swsa")], c.heads,
                        proxy_residual=bool(f & pt.PTDIT_PROXY_RESIDUAL),
                        residual=not f & pt.PTDIT_NO_RESIDUAL)
    assert rel_err(out[0], want) <= TOL["bf16"]
    dz, *dw = pt.ptdit_block_attn_bwd_saved(c.z, dout_cpu.cuda(), grid, ratio, window, shift, *W,
                                            c.heads, ws, f)
    _check_path(c, ratio, window, shift, dout_cpu, dz, dw, f)
