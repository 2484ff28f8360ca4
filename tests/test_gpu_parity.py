"""GPU parity: the CUDA library against the float64 oracle, element by element.

Small cases span several tiles and ragged tails and are compared in full; so
are the five workloads at full size (in the launch configuration the bench
times), each branch without its residual, the long-video ratio sweep on its
4 x 64 x 64 subgrid and the dense comparator at 4096 tokens.  The sweep's
32768-proxy point on the whole video grid and the dense comparator at 16384
tokens are compared on sampled rows.
Index maps are compared bit-exact.  Tolerance: max|gpu - oracle| / max|oracle|
<= 1e-4 (fp32) or 2e-2 (bf16) per output tensor, with the residual on and off.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_sparse_b200 as pt
import oracle as O
from diffusion_transformer_sparse_b200 import build, synth
from diffusion_transformer_sparse_b200.configs import RATIO_SWEEP, WORKLOADS
from tests.helpers import TOL, Case, rel_err, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pt.lib()


# ---------------------------------------------------------------- index maps (bit-exact)

@pytest.mark.parametrize("grid,ratio", [((1, 16, 16), (1, 2, 2)), ((1, 64, 64), (1, 4, 4)),
                                        ((16, 32, 48), (1, 4, 4)), ((4, 8, 12), (2, 4, 3)),
                                        ((32, 64, 64), (1, 16, 16)), ((3, 5, 7), (1, 1, 1)),
                                        ((2, 4, 6), (2, 4, 6))])
def test_proxy_map_bit_exact(grid, ratio):
    got = pt.ptdit_debug_proxy_map(grid, ratio).cpu().numpy()
    np.testing.assert_array_equal(got, O.proxy_index(grid, ratio))


@pytest.mark.parametrize("grid,window,shift", [
    ((1, 16, 16), (1, 4, 4), (0, 2, 2)), ((1, 64, 64), (1, 8, 8), (0, 4, 4)),
    ((16, 32, 48), (2, 8, 8), (1, 4, 4)), ((4, 8, 12), (2, 4, 3), (1, 3, 1)),
    ((2, 6, 10), (2, 3, 5), (1, 1, 4)), ((1, 16, 16), (1, 16, 16), (0, 0, 0)),
    ((1, 4, 4), (1, 2, 2), (0, 1, 1)),
])
def test_window_map_bit_exact(grid, window, shift):
    tok, allowed = pt.ptdit_debug_window_map(grid, window, shift)
    tmap = O.window_token_map(grid, window, shift)
    np.testing.assert_array_equal(tok.cpu().numpy().reshape(tmap.shape), tmap)
    lab = O.window_region_labels(grid, window, shift)
    want = lab[:, :, None] == lab[:, None, :]
    np.testing.assert_array_equal(allowed.cpu().numpy().reshape(want.shape).astype(bool), want)


# ---------------------------------------------------------------- averaging

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,grid,D,ratio", [
    (1, (1, 16, 16), 64, (1, 2, 2)), (2, (4, 8, 12), 40, (2, 4, 3)), (1, (2, 6, 10), 1152, (1, 3, 5)),
    (4, (1, 64, 64), 1152, (1, 4, 4)), (1, (3, 8, 8), 24, (3, 8, 8)), (1, (2, 4, 4), 36, (1, 1, 1)),
    (1, (1, 8, 8), 2100, (1, 2, 2)),
])
def test_proxy_average(dtype, B, grid, D, ratio):
    c = Case(B, grid, D, 1, dtype)
    got = c.out64(pt.ptdit_proxy_average(c.z, grid, ratio))
    # fp32: P summands of unit size lose at most ~P * 2^-24 of the largest mean
    # (1e-5 covers P = 192); bf16 adds one output rounding of 2^-9 relative.
    for b in range(B):
        err = rel_err(got[b], O.averaging(c.z64[b], grid, ratio))
        assert err <= (1e-5 if dtype == "f32" else 4e-3), err


def test_proxy_average_is_deterministic():
    c = Case(1, (1, 128, 128), 1152, 1, "bf16")
    a = pt.ptdit_proxy_average(c.z, c.grid, (1, 8, 8))
    b = pt.ptdit_proxy_average(c.z, c.grid, (1, 8, 8))
    assert torch.equal(a, b)


# ---------------------------------------------------------------- modules on small grids

SMALL = [
    # B, grid, D, heads, ratio, window, shift
    (1, (1, 16, 16), 64, 2, (1, 2, 2), (1, 4, 4), (0, 2, 2)),
    (2, (2, 8, 8), 48, 3, (1, 4, 2), (2, 4, 4), (1, 2, 2)),
    (1, (4, 8, 12), 96, 4, (2, 2, 3), (2, 4, 3), (1, 1, 2)),
    (1, (1, 24, 24), 144, 2, (1, 3, 3), (1, 8, 8), (0, 4, 4)),
    (1, (2, 16, 16), 1152, 16, (1, 4, 4), (2, 8, 8), (1, 4, 4)),
    # head width 64 (no columns past the first 128-byte swizzle atom)
    (1, (1, 16, 16), 128, 2, (1, 2, 2), (1, 8, 8), (0, 4, 4)),
    # 2 x 4 x 16 windows (rows of 16 tokens) with a shift that is not half the window
    (1, (2, 16, 32), 144, 2, (1, 4, 4), (2, 4, 16), (1, 1, 4)),
    # 200 and 100 proxies: key tiles whose second 64-key half is partly filled
    (1, (1, 20, 40), 144, 2, (1, 2, 2), (1, 4, 8), (0, 2, 4)),
    (1, (1, 20, 20), 144, 2, (1, 2, 2), (1, 4, 4), (0, 2, 2)),
]


def _bf16_window_ok(dtype, window):
    """bf16 window attention runs on the tensor cores for windows of 16..128 tokens."""
    return dtype != "bf16" or window[0] * window[1] * window[2] in (16, 32, 64, 128)


def _expect_refusal(call):
    launches = pt.ptdit_launch_count()
    with pytest.raises(pt.PtditError) as e:
        call()
    assert e.value.code == pt.PTDIT_ERR_SHAPE
    assert pt.ptdit_launch_count() == launches  # refused before any launch


def _oracle_branch(c, b, which, window, shift, ratio, flags):
    z = c.z64[b]
    if which == "giim":
        return O.giim(z, c.grid, ratio, c.w64["psa"], c.w64["cross"], c.heads,
                      proxy_residual=bool(flags & pt.PTDIT_PROXY_RESIDUAL),
                      residual=not flags & pt.PTDIT_NO_RESIDUAL)
    return O.window_self_attention(z, c.grid, window, shift, c.w64["wsa"], c.heads,
                                   residual=not flags & pt.PTDIT_NO_RESIDUAL)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("flags", [0, pt.PTDIT_NO_RESIDUAL,
                                   pt.PTDIT_NO_RESIDUAL | pt.PTDIT_PROXY_RESIDUAL])
def test_giim_small(dtype, case, flags):
    B, grid, D, heads, ratio, window, shift = case
    c = Case(B, grid, D, heads, dtype)
    out = c.out64(pt.ptdit_giim(c.z, grid, ratio, c.w["psa"], c.w["cross"], heads, flags))
    for b in range(B):
        assert rel_err(out[b], _oracle_branch(c, b, "giim", None, None, ratio, flags)) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("shifted", [False, True])
@pytest.mark.parametrize("flags", [0, pt.PTDIT_NO_RESIDUAL])
def test_window_attn_small(dtype, case, shifted, flags):
    B, grid, D, heads, ratio, window, shift = case
    shift = shift if shifted else (0, 0, 0)
    c = Case(B, grid, D, heads, dtype)
    if not _bf16_window_ok(dtype, window):
        _expect_refusal(lambda: pt.ptdit_window_attn(c.z, grid, window, shift, c.w["wsa"], heads,
                                                     flags))
        return
    out = c.out64(pt.ptdit_window_attn(c.z, grid, window, shift, c.w["wsa"], heads, flags))
    for b in range(B):
        want = _oracle_branch(c, b, "win", window, shift, None, flags)
        assert rel_err(out[b], want) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", SMALL[:4])
def test_block_attn_small(dtype, case):
    B, grid, D, heads, ratio, window, shift = case
    c = Case(B, grid, D, heads, dtype)
    if not _bf16_window_ok(dtype, window):
        _expect_refusal(lambda: pt.ptdit_block_attn(c.z, grid, ratio, window, shift, c.w["psa"],
                                                    c.w["cross"], c.w["wsa"], c.w["swsa"], heads))
        return
    out = c.out64(pt.ptdit_block_attn(c.z, grid, ratio, window, shift, c.w["psa"], c.w["cross"],
                                      c.w["wsa"], c.w["swsa"], heads))
    for b in range(B):
        want = O.block_attn(c.z64[b], grid, ratio, window, shift, c.w64["psa"], c.w64["cross"],
                            c.w64["wsa"], c.w64["swsa"], heads)
        assert rel_err(out[b], want) <= TOL[dtype]
    tcm = c.out64(pt.ptdit_tcm(c.z, grid, window, shift, c.w["wsa"], c.w["swsa"], heads,
                               pt.PTDIT_NO_RESIDUAL))
    for b in range(B):
        want = O.tcm(c.z64[b], grid, window, shift, c.w64["wsa"], c.w64["swsa"], heads,
                     residual=False)
        assert rel_err(tcm[b], want) <= TOL[dtype]


@pytest.mark.parametrize("D,heads", [(1152, 9), (60, 2), (176, 2)])
def test_bf16_head_width_without_tensor_core_kernel_is_refused(D, heads):
    """Head widths 128, 30 and 88: bf16 has no CUDA-core fallback, the call is refused."""
    c = Case(1, (1, 16, 16), D, heads, "bf16")
    _expect_refusal(lambda: pt.ptdit_giim(c.z, c.grid, (1, 4, 4), c.w["psa"], c.w["cross"], heads))
    _expect_refusal(lambda: pt.ptdit_full_attn(c.z, c.grid, c.w["wsa"], heads))


@pytest.mark.parametrize("dtype,grid,D,heads,window,shift", [
    ("bf16", (2, 8, 16), 128, 8, (2, 4, 2), (1, 2, 1)),    # head width 16, windows of 16
    ("bf16", (2, 16, 16), 96, 2, (2, 4, 4), (1, 2, 2)),    # head width 48, windows of 32
    ("bf16", (1, 24, 24), 192, 3, (1, 4, 8), (0, 2, 4)),   # head width 64, windows of 32
    ("bf16", (1, 32, 32), 80, 2, (1, 8, 8), (0, 4, 4)),    # head width 40, windows of 64
    ("bf16", (4, 8, 8), 64, 8, (2, 8, 8), (1, 4, 4)),      # head width 8, windows of 128
])
def test_window_attn_tensor_core_shapes(dtype, grid, D, heads, window, shift):
    """The packings of 8, 4, 2 and 1 windows per 128-row tile and head widths below 64."""
    c = Case(1, grid, D, heads, dtype)
    for sh in ((0, 0, 0), shift):
        for flags in (0, pt.PTDIT_NO_RESIDUAL):
            out = c.out64(pt.ptdit_window_attn(c.z, grid, window, sh, c.w["swsa"], heads, flags))
            want = O.window_self_attention(c.z64[0], grid, window, sh, c.w64["swsa"], heads,
                                           residual=not flags)
            assert rel_err(out[0], want) <= TOL[dtype], (sh, flags)


# ---------------------------------------------------------------- degenerate cases of the method

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_window_broadcasts(dtype):
    """ratio = grid: one proxy, so every latent receives the same cross-attention vector."""
    grid = (2, 8, 8)
    c = Case(1, grid, 64, 2, dtype)
    out = pt.ptdit_giim(c.z, grid, grid, c.w["psa"], c.w["cross"], 2, pt.PTDIT_NO_RESIDUAL)
    o = c.out64(out)[0]
    assert np.all(o == o[0:1])  # bit-identical rows
    want = O.giim(c.z64[0], grid, grid, c.w64["psa"], c.w64["cross"], 2, residual=False)
    assert rel_err(o, want) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ratio_111_and_full_window(dtype):
    grid = (1, 8, 16)
    c = Case(1, grid, 64, 2, dtype)
    out = c.out64(pt.ptdit_giim(c.z, grid, (1, 1, 1), c.w["psa"], c.w["cross"], 2))
    want = O.giim(c.z64[0], grid, (1, 1, 1), c.w64["psa"], c.w64["cross"], 2)
    assert rel_err(out[0], want) <= TOL[dtype]
    # window = grid is full self-attention, and so is the dense comparator
    a = c.out64(pt.ptdit_window_attn(c.z, grid, grid, (0, 0, 0), c.w["wsa"], 2))
    f = c.out64(pt.ptdit_full_attn(c.z, grid, c.w["wsa"], 2))
    want = O.masked_self_attention(c.z64[0], c.w64["wsa"], 2, np.ones((128, 128), bool))
    assert rel_err(a[0], want) <= TOL[dtype]
    assert rel_err(f[0], want) <= TOL[dtype]


def test_rescale_on_part_of_a_warp():
    """Dense attention over two 128-key tiles where, inside every 32-row warp of the
    first query tile, rows 0-15 score about 17 (in log2 units) against the second key
    tile and about 0 against the first, and rows 16-31 score about 0 everywhere: half
    of each warp raises its softmax reference (rescaling O) at the second tile and
    half does not.  Both halves must match the oracle."""
    grid, D, heads, a = (1, 16, 16), 144, 2, 10.0
    N, d = 256, D // heads
    rng = np.random.default_rng(77)
    z = rng.normal(0.0, 0.1, (N, D))
    rows = np.arange(N)
    for h in range(heads):
        e1, e2 = h * d, h * d + 1
        z[(rows < 128) & (rows % 32 < 16), e1] += a   # queries that jump at key tile 1
        z[rows >= 128, e2] += a                        # key tile 1
    eye = np.eye(D)
    wk = eye.copy()
    for h in range(heads):  # K swaps each head's first two columns
        e1, e2 = h * d, h * d + 1
        wk[[e1, e2]] = wk[[e2, e1]]
    zt = torch.tensor(z, dtype=torch.bfloat16)
    W = tuple(torch.tensor(m, dtype=torch.bfloat16) for m in (eye, wk, eye, eye))
    out = pt.ptdit_full_attn(zt[None].cuda(), grid, tuple(x.cuda() for x in W), heads)
    torch.cuda.synchronize()
    got = out[0].to("cpu", torch.float64).numpy()
    z64 = zt.to(torch.float64).numpy()
    W64 = tuple(x.to(torch.float64).numpy() for x in W)
    want = O.masked_self_attention(z64, W64, heads, np.ones((N, N), bool))
    # the jumping rows do attend to key tile 1 (the set-up does what it says)
    assert np.allclose(want[0, 1] - z64[0, 1], a, atol=0.5)
    assert rel_err(got, want) <= TOL["bf16"]


def test_block_attn_is_deterministic():
    w = WORKLOADS["tiny_16x16_f32"].with_(dtype="bf16", D=144, heads=2)
    c = Case(2, w.grid, w.D, w.heads, "bf16")
    args = (w.grid, w.ratio, w.window, w.shift, c.w["psa"], c.w["cross"], c.w["wsa"],
            c.w["swsa"], w.heads)
    a = pt.ptdit_block_attn(c.z, *args)
    b = pt.ptdit_block_attn(c.z, *args)
    assert torch.equal(a, b)


def test_rejects_invalid_on_device_tensors():
    c = Case(1, (1, 16, 16), 64, 2, "f32")
    with pytest.raises(pt.PtditError) as e:
        pt.ptdit_window_attn(c.z, (1, 16, 16), (1, 5, 4), (0, 0, 0), c.w["wsa"], 2)
    assert e.value.code == 2
    with pytest.raises(pt.PtditError) as e:
        pt.ptdit_window_attn(c.z, (1, 16, 16), (1, 4, 4), (0, 0, 0), c.w["wsa"], 2, z_out=c.z)
    assert e.value.code == 8


# ---------------------------------------------------------------- the five workloads, full size

@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_block_attn(name):
    """Whole [B, N, D] outputs of every workload against the oracle, in the launch
    configuration the bench times (persistent kernels run many units per CTA)."""
    w = WORKLOADS[name]
    c = Case(w.B, w.grid, w.D, w.heads, w.dtype)
    out = c.out64(pt.ptdit_block_attn(c.z, w.grid, w.ratio, w.window, w.shift, c.w["psa"],
                                      c.w["cross"], c.w["wsa"], c.w["swsa"], w.heads))
    for b in range(w.B):
        want = O.block_attn(c.z64[b], w.grid, w.ratio, w.window, w.shift, c.w64["psa"],
                            c.w64["cross"], c.w64["wsa"], c.w64["swsa"], w.heads)
        assert rel_err(out[b], want) <= TOL[w.dtype], (name, b)


@pytest.mark.parametrize("name", list(WORKLOADS)[1:])
def test_workload_branches_without_residual(name):
    """Each branch alone at full size and in full, so residual rounding cannot hide
    a small branch (at ratio (1,16,16) the proxies have variance about 1/256)."""
    w = WORKLOADS[name]
    c = Case(1, w.grid, w.D, w.heads, w.dtype)
    g = c.out64(pt.ptdit_giim(c.z[:1], w.grid, w.ratio, c.w["psa"], c.w["cross"], w.heads,
                              pt.PTDIT_NO_RESIDUAL))
    want = O.giim(c.z64[0], w.grid, w.ratio, c.w64["psa"], c.w64["cross"], w.heads,
                  residual=False)
    assert rel_err(g[0], want) <= TOL[w.dtype]
    for shift in [(0, 0, 0), w.shift]:
        a = c.out64(pt.ptdit_window_attn(c.z[:1], w.grid, w.window, shift, c.w["swsa"], w.heads,
                                         pt.PTDIT_NO_RESIDUAL))
        want = O.window_self_attention(c.z64[0], w.grid, w.window, shift, c.w64["swsa"],
                                       w.heads, residual=False)
        assert rel_err(a[0], want) <= TOL[w.dtype], shift


# ---------------------------------------------------------------- long-video ratio sweep

SWEEP = WORKLOADS["video_32x64x64"]


@pytest.mark.parametrize("ratio", RATIO_SWEEP)
def test_ratio_sweep_subgrid(ratio):
    """The long-video ratio sweep on its 4 x 64 x 64 subgrid (M = 4096 .. 64), in full."""
    w = SWEEP.with_(grid=(4, 64, 64), ratio=ratio)
    c = Case(1, w.grid, w.D, w.heads, w.dtype)
    out = c.out64(pt.ptdit_block_attn(c.z, w.grid, w.ratio, w.window, w.shift, c.w["psa"],
                                      c.w["cross"], c.w["wsa"], c.w["swsa"], w.heads))
    want = O.block_attn(c.z64[0], w.grid, w.ratio, w.window, w.shift, c.w64["psa"],
                        c.w64["cross"], c.w64["wsa"], c.w64["swsa"], w.heads)
    assert rel_err(out[0], want) <= TOL[w.dtype]
    g = c.out64(pt.ptdit_giim(c.z, w.grid, w.ratio, c.w["psa"], c.w["cross"], w.heads,
                              pt.PTDIT_NO_RESIDUAL))
    want = O.giim(c.z64[0], w.grid, w.ratio, c.w64["psa"], c.w64["cross"], w.heads,
                  residual=False)
    assert rel_err(g[0], want) <= TOL[w.dtype]


def test_ratio_122_full_grid_sampled():
    """The sweep's largest point: 32768 proxies over the whole 32 x 64 x 64 grid
    (proxy self-attention of 256 x 256 tiles of 128 rows).  Sampled output rows,
    each through its dependency closure (all proxies, both window levels)."""
    w = SWEEP.with_(ratio=(1, 2, 2))
    c = Case(1, w.grid, w.D, w.heads, w.dtype)
    out = pt.ptdit_giim(c.z, w.grid, w.ratio, c.w["psa"], c.w["cross"], w.heads,
                        pt.PTDIT_NO_RESIDUAL)
    rows = sample_rows(w.grid, k=24, seed=11)
    got = c.out64(out[0, torch.from_numpy(rows).cuda()])
    want = O.giim(c.z64[0], w.grid, w.ratio, c.w64["psa"], c.w64["cross"], w.heads,
                  residual=False, rows=rows)[rows]
    assert rel_err(got, want) <= TOL[w.dtype]


# ---------------------------------------------------------------- dense comparator

def test_dense_full_attn_4096():
    """ptdit_full_attn over a 64 x 64 grid (4096 tokens, 32 key tiles), in full."""
    c = Case(1, (1, 64, 64), 1152, 16, "bf16")
    out = c.out64(pt.ptdit_full_attn(c.z, c.grid, c.w["wsa"], 16))
    want = O.masked_self_attention(c.z64[0], c.w64["wsa"], 16, None)
    assert rel_err(out[0], want) <= TOL["bf16"]


@pytest.mark.parametrize("grid", [(1, 128, 128), (4, 64, 64)])
def test_dense_full_attn_16384_sampled(grid):
    """The dense comparator at bench size (16384 tokens): sampled query rows against
    full attention over all keys."""
    c = Case(1, grid, 1152, 16, "bf16")
    out = pt.ptdit_full_attn(c.z, grid, c.w["wsa"], 16, pt.PTDIT_NO_RESIDUAL)
    rows = sample_rows(grid, k=120, seed=5)
    got = c.out64(out[0, torch.from_numpy(rows).cuda()])
    want = O.multihead_attention(c.z64[0][rows], c.z64[0], c.w64["wsa"], 16)
    assert rel_err(got, want) <= TOL["bf16"]


# ---------------------------------------------------------------- proxy extraction variants

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,grid,D,ratio", [
    (2, (4, 8, 12), 40, (2, 4, 3)), (1, (2, 6, 10), 1152, (1, 3, 5)),
    (4, (1, 64, 64), 1152, (1, 4, 4)), (1, (32, 64, 64), 1152, (4, 16, 16)),
    (1, (2, 4, 4), 36, (1, 1, 1)), (1, (1, 8, 8), 2100, (1, 2, 2)),
])
def test_proxy_extract_single_token_bit_exact(dtype, B, grid, D, ratio):
    """'first' and 'random' proxies are copies of one window member: bit for bit."""
    c = Case(B, grid, D, 1, dtype)
    P = ratio[0] * ratio[1] * ratio[2]
    M = c.N // P
    slots = synth.proxy_slots(B, M, P)
    first = c.out64(pt.ptdit_proxy_extract(c.z, grid, ratio, "first"))
    rand = c.out64(pt.ptdit_proxy_extract(c.z, grid, ratio, "random", slots.cuda()))
    mean = c.out64(pt.ptdit_proxy_extract(c.z, grid, ratio, "mean"))
    for b in range(B):
        np.testing.assert_array_equal(first[b], O.proxy_tokens(c.z64[b], grid, ratio, "first"))
        np.testing.assert_array_equal(
            rand[b], O.proxy_tokens(c.z64[b], grid, ratio, "random", slots[b].numpy()))
        assert rel_err(mean[b], O.averaging(c.z64[b], grid, ratio)) <= (1e-5 if dtype == "f32" else 4e-3)


def test_proxy_extract_out_of_range_slot_is_reported():
    c = Case(1, (1, 8, 8), 64, 1, "f32")
    slots = torch.zeros(16, dtype=torch.int32)
    slots[5] = 4   # P = 4: one past the last member
    pt.ptdit_device_status(reset=True)
    out = c.out64(pt.ptdit_proxy_extract(c.z, c.grid, (1, 2, 2), "random", slots.cuda()))
    assert pt.ptdit_device_status(reset=True) == pt.PTDIT_ERR_SHAPE
    assert np.all(out[0, 5] == 0)
    want = O.proxy_tokens(c.z64[0], c.grid, (1, 2, 2), "first")
    np.testing.assert_array_equal(np.delete(out[0], 5, 0), np.delete(want, 5, 0))


@pytest.mark.parametrize("mode", ["first", "random"])
@pytest.mark.parametrize("dtype,B,grid,D,heads,ratio", [
    ("f32", 1, (1, 16, 16), 64, 2, (1, 2, 2)), ("bf16", 2, (2, 16, 16), 1152, 16, (1, 4, 4)),
    ("bf16", 4, (1, 64, 64), 1152, 16, (1, 4, 4)), ("bf16", 1, (16, 32, 48), 1152, 16, (4, 4, 4)),
])
def test_giim_ex_proxy_modes(mode, dtype, B, grid, D, heads, ratio):
    c = Case(B, grid, D, heads, dtype)
    P = ratio[0] * ratio[1] * ratio[2]
    slots = synth.proxy_slots(B, c.N // P, P, seed=99)
    for flags in (0, pt.PTDIT_NO_RESIDUAL):
        out = c.out64(pt.ptdit_giim_ex(c.z, grid, ratio, mode, slots.cuda(), c.w["psa"],
                                       c.w["cross"], heads, flags))
        for b in range(B):
            want = O.giim(c.z64[b], grid, ratio, c.w64["psa"], c.w64["cross"], heads,
                          residual=not flags, proxy_mode=mode, slots=slots[b].numpy())
            assert rel_err(out[b], want) <= TOL[dtype], (b, flags)
