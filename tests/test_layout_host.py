"""Host logic of the CUDA path, checked without a GPU.

The tiled head layout (where each token's 16-byte pieces land in the blocks the
attention kernels load) and the projection GEMM's tile schedule are computed by
host-callable functions of the library; these tests read them through the
ptdit_debug_thl_* and ptdit_debug_gemm_schedule entry points and check them
against the oracle's window partition, the hardware's shared-memory swizzle
written as an address-bit permutation, and scheduling theory.
"""
import itertools

import numpy as np
import pytest

import diffusion_transformer_sparse_b200 as pt
import oracle as O
from diffusion_transformer_sparse_b200 import build

ROWS = 128  # tile rows


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pt.lib()


# ---------------------------------------------------------------- tiled head layout: token maps

@pytest.mark.parametrize("grid", [(1, 16, 16), (1, 20, 40), (2, 16, 32), (1, 3, 5)])
def test_identity_tiles_hold_tokens_in_order(grid):
    N = grid[0] * grid[1] * grid[2]
    row, tok = pt.ptdit_debug_thl_map(grid)
    assert len(tok) == -(-N // ROWS) * ROWS
    assert np.array_equal(row, np.arange(N))
    assert np.array_equal(tok[:N], np.arange(N)) and np.all(tok[N:] == -1)


WINDOWED = [
    # grid, window, shift: 2D and 3D windows of 16, 32, 64 and 128 tokens, shifts of
    # half a window and others, grids whose window count does not fill the last tile
    ((1, 16, 16), (1, 8, 8), (0, 4, 4)),
    ((1, 16, 16), (1, 8, 8), (0, 0, 0)),
    ((1, 24, 8), (1, 8, 8), (0, 4, 4)),
    ((4, 16, 16), (2, 8, 8), (1, 4, 4)),
    ((6, 8, 16), (2, 8, 8), (1, 3, 5)),
    ((2, 16, 32), (2, 4, 16), (1, 1, 4)),
    ((1, 16, 16), (1, 4, 4), (0, 2, 2)),
    ((2, 8, 8), (2, 4, 4), (1, 2, 2)),
    ((1, 12, 20), (1, 4, 4), (0, 1, 3)),
]


@pytest.mark.parametrize("grid,window,shift", WINDOWED)
def test_window_tiles_match_the_oracle_partition(grid, window, shift):
    """Tile rows hold the oracle's (window, slot) tokens of the rolled grid: 128 / n
    windows per tile in window order, slots in order; the rest of the last tile is empty."""
    N = grid[0] * grid[1] * grid[2]
    n = window[0] * window[1] * window[2]
    pack = ROWS // n
    want = O.window_token_map(grid, window, shift)  # [windows, n]
    nwin = want.shape[0]
    row, tok = pt.ptdit_debug_thl_map(grid, window, shift)
    assert len(tok) == -(-nwin // pack) * ROWS
    expect = np.full(len(tok), -1, np.int64)
    for w in range(nwin):
        base = (w // pack) * ROWS + (w % pack) * n
        expect[base:base + n] = want[w]
    assert np.array_equal(tok, expect)
    # row_of_token inverts it
    assert np.array_equal(tok[row], np.arange(N))


def test_window_tiles_need_windows_that_divide_the_tile():
    with pytest.raises(pt.PtditError) as e:
        pt.ptdit_debug_thl_map((1, 12, 12), (1, 3, 3), (0, 1, 1))
    assert e.value.code == 2


# ---------------------------------------------------------------- tiled head layout: swizzle

def _swizzled(canonical, atom_bits):
    """The tensor cores' shared-memory swizzle of a K-major tile, as an address
    permutation: bits [4, 4 + atom_bits) are XORed with the bits 3 places above them
    (atom_bits = 3: 128-byte swizzle, 8 rows of 128 B; 1: 32-byte swizzle, 8 rows of 32 B)."""
    mask = (1 << atom_bits) - 1
    return canonical ^ (((canonical >> 7) & mask) << 4)


def _expected_offsets(d, vpad):
    """Row r, unit p (columns 8p..8p+7) of the swizzled tile: columns 0..63 as 128-byte
    atoms; columns 64.. either 32-byte atoms (16 columns) or a second set of 128-byte atoms."""
    units = 8 if d <= 64 else (16 if vpad else 10)
    off = np.empty((ROWS, units), np.int64)
    for r, p in itertools.product(range(ROWS), range(units)):
        if p < 8:
            off[r, p] = _swizzled((r // 8) * 1024 + (r % 8) * 128 + p * 16, 3)
        elif vpad:
            off[r, p] = 16384 + _swizzled((r // 8) * 1024 + (r % 8) * 128 + (p - 8) * 16, 3)
        else:
            off[r, p] = 16384 + _swizzled((r // 8) * 256 + (r % 8) * 32 + (p - 8) * 16, 1)
    return off


@pytest.mark.parametrize("d,vpad", [(64, 0), (72, 0), (80, 0), (72, 1), (80, 1), (32, 0)])
def test_thl_units_are_the_swizzled_tile(d, vpad):
    off, block = pt.ptdit_debug_thl_units(d, bool(vpad))
    assert np.array_equal(off.astype(np.int64), _expected_offsets(d, vpad and d > 64))
    # every 16-byte unit of the block exactly once
    assert block == off.size * 16
    assert np.array_equal(np.sort(off.ravel()), np.arange(0, block, 16))


@pytest.mark.parametrize("d", [0, 4, 12, 88, 128])
def test_thl_units_reject_unsupported_head_widths(d):
    with pytest.raises(pt.PtditError) as e:
        pt.ptdit_debug_thl_units(d)
    assert e.value.code == 2


# ---------------------------------------------------------------- projection GEMM tile schedule

def _widths(tiles, nseg):
    n_tiles = -(-nseg // 256)
    return np.array([min(256, nseg - 256 * (t % n_tiles)) for t in range(tiles)])


SHAPES = [
    # rows, nseg, nmat, pairs: the block's projections at 1024 px, 2048 px and long video
    # (Q/K/V: three 1152-wide outputs; O: one; proxy K/V: two), and odd cases
    (16384, 1152, 3, 74), (16384, 1152, 1, 74), (1024, 1152, 3, 74), (1024, 1152, 2, 74),
    (256, 1152, 3, 74), (200, 1152, 1, 74), (1, 64, 1, 1), (800, 320, 2, 7),
    (4096, 192, 3, 128), (131072, 1152, 1, 74), (16384, 1024, 3, 74), (3000, 1152, 1, 1),
]


@pytest.mark.parametrize("rows,nseg,nmat,pairs", SHAPES)
def test_gemm_schedule_is_a_balanced_partition(rows, nseg, nmat, pairs):
    tiles, lists = pt.ptdit_debug_gemm_schedule(rows, nseg, nmat, pairs)
    assert tiles == -(-rows // 256) * nmat * -(-nseg // 256)
    if nseg % 256 == 0 or tiles > 4096 or pairs > 128:
        assert lists is None  # equal tiles, or too many to describe: round robin
        return
    assert lists is not None and len(lists) == pairs
    flat = [t for lst in lists for t in lst]
    assert sorted(flat) == list(range(tiles))  # every tile exactly once
    assert all(lst == sorted(lst) for lst in lists)  # each pair sweeps its tiles in order
    w = _widths(tiles, nseg)
    loads = [int(w[lst].sum()) for lst in lists]
    # list scheduling: the busiest pair got its last tile while it was the least loaded
    assert max(loads) <= w.sum() / pairs + w.max()
    # no worse than round robin on these shapes
    rr = [int(w[q::pairs].sum()) for q in range(pairs)]
    assert max(loads) <= max(rr)


@pytest.mark.parametrize("rows,nseg,nmat,pairs", [
    (256, 320, 2, 3), (512, 320, 1, 3), (256, 576, 1, 2), (768, 320, 1, 4), (256, 832, 2, 5),
])
def test_gemm_schedule_within_grahams_bound_of_the_optimum(rows, nseg, nmat, pairs):
    """Longest-processing-time order is within 4/3 - 1/(3 m) of the best makespan on m
    machines (Graham, 1969); the best one is found here by brute force."""
    tiles, lists = pt.ptdit_debug_gemm_schedule(rows, nseg, nmat, pairs)
    w = _widths(tiles, nseg)
    assert tiles <= 8 and lists is not None
    best = min(max(sum(int(w[t]) for t in range(tiles) if a[t] == q) for q in range(pairs))
               for a in itertools.product(range(pairs), repeat=tiles))
    got = max(int(w[lst].sum()) for lst in lists)
    assert got <= (4 / 3 - 1 / (3 * pairs)) * best + 1e-9


@pytest.mark.parametrize("args", [(0, 1152, 1, 74), (1024, 100, 1, 74), (1024, 1152, 4, 74),
                                  (1024, 1152, 1, 0)])
def test_gemm_schedule_rejects_shapes_no_launch_takes(args):
    with pytest.raises(pt.PtditError) as e:
        pt.ptdit_debug_gemm_schedule(*args)
    assert e.value.code == 2
