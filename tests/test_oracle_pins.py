"""Pins of the float64 oracle against things other than itself.

Each test ties one oracle function to what the pages and the mathematics fix:
hand-derived index maps (tests/golden), torch's own multi-head attention as a
library routine, closed forms of degenerate cases, brute force with scalar
loops, invariants, and the pages' printed 2.3% complexity figure.  The last
group plants plausible mistakes in the oracle and checks that a pin catches
each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from diffusion_transformer_sparse_b200 import flops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


def _weights(D, seed, k=4, scale=None):
    rng = np.random.default_rng(seed)
    a = math.sqrt(6.0 / (2 * D)) if scale is None else scale
    return tuple(rng.uniform(-a, a, (D, D)) for _ in range(k))


def torch_mha(xq, xkv, W, heads, allow=None):
    """torch.nn.MultiheadAttention (bias-free, float64) as an independent library routine."""
    D = xq.shape[1]
    mha = torch.nn.MultiheadAttention(D, heads, bias=False, batch_first=True, dtype=torch.float64)
    with torch.no_grad():
        mha.in_proj_weight.copy_(torch.from_numpy(np.concatenate(W[:3], axis=0)))
        mha.out_proj.weight.copy_(torch.from_numpy(W[3]))
        mask = None if allow is None else torch.from_numpy(~allow)
        q = torch.from_numpy(np.ascontiguousarray(xq))[None]
        kv = torch.from_numpy(np.ascontiguousarray(xkv))[None]
        out, _ = mha(q, kv, kv, attn_mask=mask, need_weights=False)
    return out[0].numpy()


def _close(a, b, tol=1e-10):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    err = np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b)))
    assert err <= tol, f"max rel err {err:.3e} > {tol:.1e}"


def _divisors(L):
    return [p for p in range(1, L + 1) if L % p == 0]


# ---------------------------------------------------------------- P1 averaging

def test_proxy_index_golden():
    for name in ("proxy_map_1x4x4_r122.json", "proxy_map_2x2x4_r212.json"):
        g = _golden(name)
        got = O.proxy_index(tuple(g["grid"]), tuple(g["ratio"]))
        np.testing.assert_array_equal(got, np.array(g["proxy_of_token"]))


@pytest.mark.parametrize("grid", [(1, 4, 4), (2, 4, 6), (4, 8, 8), (3, 6, 4)])
def test_averaging_bruteforce(grid):
    f, h, w = grid
    rng = np.random.default_rng(7)
    z = rng.standard_normal((f * h * w, 5))
    for ratio in itertools.product(_divisors(f), _divisors(h), _divisors(w)):
        pf, ph, pw = ratio
        got = O.averaging(z, grid, ratio)
        # scalar loops over each window, written from the definition
        want = []
        for T in range(f // pf):
            for Y in range(h // ph):
                for X in range(w // pw):
                    acc = np.zeros(5)
                    cnt = 0
                    for t in range(T * pf, T * pf + pf):
                        for y in range(Y * ph, Y * ph + ph):
                            for x in range(X * pw, X * pw + pw):
                                acc += z[(t * h + y) * w + x]
                                cnt += 1
                    want.append(acc / cnt)
        _close(got, np.array(want), 1e-14)
        # the index map groups the same tokens
        idx = O.proxy_index(grid, ratio)
        for m in range(got.shape[0]):
            _close(got[m], z[idx == m].mean(axis=0), 1e-14)


def test_averaging_rejects_non_divisible():
    with pytest.raises(ValueError):
        O.averaging(np.zeros((24, 2)), (1, 4, 6), (1, 4, 4))


# ---------------------------------------------------------------- maps and masks

def test_window_map_golden():
    g = _golden("shifted_windows_1x4x4_w122_s011.json")
    grid, window, shift = tuple(g["grid"]), tuple(g["window"]), tuple(g["shift"])
    tok = O.window_token_map(grid, window, shift)
    np.testing.assert_array_equal(tok, np.array(g["token_at_window_slot"]))
    lab = O.window_region_labels(grid, window, shift)
    for k, groups in enumerate(g["allowed_groups"]):
        want = np.zeros((4, 4), bool)
        for grp in groups:
            for i in grp:
                for j in grp:
                    want[i, j] = True
        np.testing.assert_array_equal(lab[k][:, None] == lab[k][None, :], want)


@pytest.mark.parametrize("grid", [(1, 8, 8), (2, 4, 8), (4, 4, 4)])
def test_window_maps_partition_and_match_pair_mask(grid):
    N = O.num_tokens(grid)
    full = O.window_allow_matrix
    for window in itertools.product(*[_divisors(L) for L in grid]):
        for shift in itertools.product(*[range(wd) for wd in window]):
            tok = O.window_token_map(grid, window, shift)
            assert sorted(tok.ravel().tolist()) == list(range(N))
            lab = O.window_region_labels(grid, window, shift)
            allow = np.zeros((N, N), bool)
            for k in range(tok.shape[0]):
                same = lab[k][:, None] == lab[k][None, :]
                allow[np.ix_(tok[k], tok[k])] = same
            np.testing.assert_array_equal(allow, full(grid, window, shift))


# ---------------------------------------------------------------- P2 / cross-attn vs library

def test_ratio_111_proxy_sa_is_full_self_attention():
    grid, D, heads = (2, 4, 4), 8, 2
    z = np.random.default_rng(1).standard_normal((32, D))
    W = _weights(D, 2)
    got = O.proxy_self_attention(z, grid, (1, 1, 1), W, heads)
    _close(got, torch_mha(z, z, W, heads))


@pytest.mark.parametrize("ratio", [(1, 2, 2), (2, 2, 1), (1, 4, 4)])
def test_giim_matches_library_mha(ratio):
    grid, D, heads = (2, 4, 8), 12, 3
    z = np.random.default_rng(3).standard_normal((64, D))
    Wp, Wc = _weights(D, 4), _weights(D, 5)
    Pa = O.averaging(z, grid, ratio)
    Pp = torch_mha(Pa, Pa, Wp, heads)
    _close(O.giim(z, grid, ratio, Wp, Wc, heads, residual=False), torch_mha(z, Pp, Wc, heads))
    _close(O.giim(z, grid, ratio, Wp, Wc, heads), z + torch_mha(z, Pp, Wc, heads))
    _close(O.giim(z, grid, ratio, Wp, Wc, heads, proxy_residual=True, residual=False),
           torch_mha(z, Pp + Pa, Wc, heads))


# ---------------------------------------------------------------- P3 single window

def test_single_window_broadcasts_one_vector():
    grid, D, heads = (2, 4, 4), 8, 2
    z = np.random.default_rng(5).standard_normal((32, D))
    Wp, Wc = _weights(D, 6), _weights(D, 7)
    out = O.giim(z, grid, grid, Wp, Wc, heads, residual=False)
    Pa = z.mean(axis=0)
    # softmax over a single key is 1: SA(P_a) = Wo Wv P_a and CS(z, P') = Wo Wv P'
    Pp = Wp[3] @ (Wp[2] @ Pa)
    want = Wc[3] @ (Wc[2] @ Pp)
    for row in out:
        _close(row, want, 1e-12)


# ---------------------------------------------------------------- P4 special cases

def test_window_equal_grid_is_full_self_attention():
    grid, D, heads = (2, 4, 4), 8, 2
    z = np.random.default_rng(8).standard_normal((32, D))
    W = _weights(D, 9)
    _close(O.window_self_attention(z, grid, grid, (0, 0, 0), W, heads), z + torch_mha(z, z, W, heads))


def test_shift_zero_is_plain_window_attention():
    grid, window, D, heads = (2, 4, 8), (2, 2, 4), 8, 2
    z = np.random.default_rng(10).standard_normal((64, D))
    W = _weights(D, 11)
    got = O.window_self_attention(z, grid, window, (0, 0, 0), W, heads, residual=False)
    assert np.all(O.window_region_labels(grid, window, (0, 0, 0)) == 0)
    # each non-overlapping window attended on its own with the library routine
    f, h, w = grid
    for T, Y, X in itertools.product(range(0, f, 2), range(0, h, 2), range(0, w, 4)):
        toks = [(t * h + y) * w + x for t in range(T, T + 2) for y in range(Y, Y + 2)
                for x in range(X, X + 4)]
        _close(got[toks], torch_mha(z[toks], z[toks], W, heads))


# ---------------------------------------------------------------- P5, P7 two formulations

@pytest.mark.parametrize("grid,window", [((1, 8, 8), (1, 4, 4)), ((4, 4, 8), (2, 2, 4)),
                                         ((2, 6, 6), (2, 2, 2))])
def test_half_shift_direction_does_not_matter(grid, window):
    D, heads = 8, 2
    shift = tuple(wd // 2 for wd in window)
    z = np.random.default_rng(12).standard_normal((O.num_tokens(grid), D))
    W = _weights(D, 13)
    a = O.masked_self_attention(z, W, heads, O.window_allow_matrix(grid, window, shift))
    b = O.masked_self_attention(z, W, heads,
                                O.window_allow_matrix(grid, window, tuple(-s for s in shift)))
    _close(a, b, 1e-13)
    _close(O.window_self_attention(z, grid, window, shift, W, heads), a, 1e-12)


@pytest.mark.parametrize("grid", [(1, 4, 8), (2, 4, 4)])
def test_roll_formulation_matches_pair_mask_and_library(grid):
    D, heads = 6, 2
    z = np.random.default_rng(14).standard_normal((O.num_tokens(grid), D))
    W = _weights(D, 15)
    for window in itertools.product(*[[p for p in _divisors(L) if p > 1 or L == 1] for L in grid]):
        for shift in itertools.product(*[range(wd) for wd in window]):
            allow = O.window_allow_matrix(grid, window, shift)
            got = O.window_self_attention(z, grid, window, shift, W, heads)
            _close(got, O.masked_self_attention(z, W, heads, allow), 1e-12)
            _close(got, z + torch_mha(z, z, W, heads, allow), 1e-10)


# ---------------------------------------------------------------- P6 invariants

def test_giim_permutation_equivariance():
    grid, ratio, D, heads = (1, 4, 8), (1, 2, 2), 8, 2
    f, h, w = grid
    rng = np.random.default_rng(16)
    z = rng.standard_normal((32, D))
    Wp, Wc = _weights(D, 17), _weights(D, 18)
    base = O.giim(z, grid, ratio, Wp, Wc, heads)
    # swap the token blocks of proxy windows (0,0) and (1,3)
    perm = np.arange(32)
    for dy in range(2):
        for dx in range(2):
            a = (0 + dy) * w + (0 + dx)
            b = (2 + dy) * w + (6 + dx)
            perm[a], perm[b] = b, a
    _close(O.giim(z[perm], grid, ratio, Wp, Wc, heads), base[perm], 1e-12)
    # permute tokens inside every window: proxies unchanged, output permuted alike
    perm2 = np.arange(32)
    for Y in range(0, h, 2):
        for X in range(0, w, 2):
            a, b = Y * w + X, (Y + 1) * w + X + 1
            perm2[a], perm2[b] = b, a
    _close(O.averaging(z[perm2], grid, ratio), O.averaging(z, grid, ratio), 1e-15)
    _close(O.giim(z[perm2], grid, ratio, Wp, Wc, heads), base[perm2], 1e-12)


# ---------------------------------------------------------------- P8 brute force

def _scalar_mha_row(zi, keys, W, heads):
    """One query row by scalar loops: projections, per-head softmax with math.exp, output projection."""
    Wq, Wk, Wv, Wo = W
    D = len(zi)
    d = D // heads

    def lin(Wm, x):
        return [sum(Wm[o][k] * x[k] for k in range(D)) for o in range(D)]

    q = lin(Wq, zi)
    ks = [lin(Wk, kj) for kj in keys]
    vs = [lin(Wv, kj) for kj in keys]
    o = [0.0] * D
    for hh in range(heads):
        c0 = hh * d
        s = [sum(q[c0 + c] * kk[c0 + c] for c in range(d)) / math.sqrt(d) for kk in ks]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        tot = sum(e)
        for c in range(d):
            o[c0 + c] = sum(e[j] * vs[j][c0 + c] for j in range(len(ks))) / tot
    return np.array(lin(Wo, o))


def test_bruteforce_tiny_block():
    grid, ratio, window, shift, D, heads = (2, 4, 4), (1, 2, 2), (2, 2, 2), (1, 1, 1), 4, 2
    f, h, w = grid
    N = 32
    rng = np.random.default_rng(19)
    z = rng.standard_normal((N, D))
    Wp, Wc, Wa, Ws = (_weights(D, s) for s in (20, 21, 22, 23))
    coords = [(t, y, x) for t in range(f) for y in range(h) for x in range(w)]

    # GIIM by scalar loops
    proxies = []
    for T in range(0, f, ratio[0]):
        for Y in range(0, h, ratio[1]):
            for X in range(0, w, ratio[2]):
                mem = [i for i, (t, y, x) in enumerate(coords)
                       if T <= t < T + ratio[0] and Y <= y < Y + ratio[1] and X <= x < X + ratio[2]]
                proxies.append(sum(z[i] for i in mem) / len(mem))
    Pp = [_scalar_mha_row(p, proxies, Wp, heads) for p in proxies]
    z1 = np.array([z[i] + _scalar_mha_row(z[i], Pp, Wc, heads) for i in range(N)])

    def window_pass(zin, s):
        # physically shift each token to its place in the rolled grid, remember
        # along which axes the roll wrapped it, and attend among tokens that
        # share a window and the same wrap flags
        out = np.empty_like(zin)
        placed = {}
        for i, (t, y, x) in enumerate(coords):
            pos = ((t - s[0]) % f, (y - s[1]) % h, (x - s[2]) % w)
            wrapped = (t < s[0], y < s[1], x < s[2])
            win = (pos[0] // window[0], pos[1] // window[1], pos[2] // window[2])
            placed[i] = (win, wrapped)
        Wm = Wa if s == (0, 0, 0) else Ws
        for i in range(N):
            keys = [zin[j] for j in range(N) if placed[j] == placed[i]]
            out[i] = zin[i] + _scalar_mha_row(zin[i], keys, Wm, heads)
        return out

    z3 = window_pass(window_pass(z1, (0, 0, 0)), shift)
    got = O.block_attn(z, grid, ratio, window, shift, Wp, Wc, Wa, Ws, heads)
    _close(got, z3, 1e-12)


def test_block_rows_closure_matches_full():
    grid, ratio, window, shift, D, heads = (4, 8, 8), (1, 2, 4), (2, 4, 4), (1, 2, 2), 8, 2
    rng = np.random.default_rng(24)
    z = rng.standard_normal((256, D))
    Ws = [_weights(D, s) for s in (25, 26, 27, 28)]
    full = O.block_attn(z, grid, ratio, window, shift, *Ws, heads)
    rows = np.array([0, 7, 63, 64, 130, 255, 200])
    _close(O.block_attn_rows(z, grid, ratio, window, shift, *Ws, heads, rows), full[rows], 1e-13)


# ---------------------------------------------------------------- P9 the pages' number

def test_complexity_ratio_matches_printed_2_3_percent():
    g = _golden("complexity_ratio_2048.json")
    pct = 100 * flops.core_ratio(16384, 256, 64)
    assert abs(pct - g["printed_percent"]) <= g["printed_resolution_percent"]
    # the counter's own terms give the same ratio against its dense core
    f = flops.block_flops(16384, 256, 64, 1152)
    dense = flops.dense_flops(16384, 1152)
    assert math.isclose(f["core"] / dense["core"], flops.core_ratio(16384, 256, 64))


# ---------------------------------------------------------------- P10 invariants

def test_softmax_rows_and_convex_hull():
    rng = np.random.default_rng(29)
    S = rng.standard_normal((7, 11)) * 5
    S[:, 3] = -np.inf
    Pm = O.softmax_rows(S)
    _close(Pm.sum(axis=1), np.ones(7), 1e-15)
    assert np.all(Pm[:, 3] == 0)
    Q, K, V = (rng.standard_normal((9, 6)) for _ in range(3))
    out = O.attention_heads(Q, K, V, 2)
    for h in range(2):
        cols = slice(3 * h, 3 * h + 3)
        assert np.all(out[:, cols] <= V[:, cols].max(axis=0) + 1e-12)
        assert np.all(out[:, cols] >= V[:, cols].min(axis=0) - 1e-12)


# ---------------------------------------------------------------- planted mistakes

def _pin_fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_pins_catch_a_flipped_roll(monkeypatch):
    roll = np.roll

    def flipped_roll(a, shift, axis):
        return roll(a, tuple(-s for s in shift), axis)

    monkeypatch.setattr(np, "roll", flipped_roll)
    assert _pin_fails(lambda: test_roll_formulation_matches_pair_mask_and_library((1, 4, 8)))


def test_pins_catch_a_dropped_scale(monkeypatch):
    monkeypatch.setattr(math, "sqrt", lambda x: 1.0)
    assert _pin_fails(test_ratio_111_proxy_sa_is_full_self_attention)


def test_pins_catch_a_transposed_weight(monkeypatch):
    monkeypatch.setattr(O.ptdit_oracle, "project", lambda x, W: np.asarray(x, float) @ np.asarray(W, float))
    assert _pin_fails(test_ratio_111_proxy_sa_is_full_self_attention)


def test_pins_catch_a_wrong_proxy_order(monkeypatch):
    real = O.ptdit_oracle.averaging

    def col_major(z, grid, ratio):
        f, h, w = grid
        pf, ph, pw = ratio
        P = real(z, grid, ratio)
        # windows numbered column-major instead of row-major
        return P.reshape(f // pf, h // ph, w // pw, -1).transpose(2, 1, 0, 3).reshape(P.shape)

    monkeypatch.setattr(O, "averaging", col_major)
    assert _pin_fails(lambda: test_averaging_bruteforce((1, 4, 4)))


# ---------------------------------------------------------------- proxy extraction modes

def test_proxy_first_and_members_golden():
    g = _golden("proxy_first_2x4x4.json")
    grid = tuple(g["grid"])
    z = np.arange(O.num_tokens(grid), dtype=np.float64)[:, None] * np.ones((1, 3))
    for case in g["cases"]:
        got = O.proxy_tokens(z, grid, tuple(case["ratio"]), "first")
        np.testing.assert_array_equal(got[:, 0], case["first_token"])
    np.testing.assert_array_equal(O.window_members(grid, (1, 2, 2))[3],
                                  g["members_ratio_122_window_3"])


@pytest.mark.parametrize("grid,ratio", [((2, 4, 6), (1, 2, 3)), ((4, 4, 4), (2, 2, 1)),
                                        ((3, 2, 5), (3, 1, 5)), ((2, 6, 4), (1, 1, 1))])
def test_proxy_random_bruteforce(grid, ratio):
    """Scalar loops: member k of window m is the k-th smallest token index whose
    window (from coordinates) is m."""
    rng = np.random.default_rng(3)
    f, h, w = grid
    pf, ph, pw = ratio
    N, P = f * h * w, pf * ph * pw
    M = N // P
    z = rng.normal(size=(N, 5))
    slots = rng.integers(0, P, M)
    got = O.proxy_tokens(z, grid, ratio, "random", slots)
    for m in range(M):
        members = []
        for t in range(N):
            tt, y, x = t // (h * w), (t // w) % h, t % w
            if ((tt // pf) * (h // ph) + y // ph) * (w // pw) + x // pw == m:
                members.append(t)
        assert len(members) == P
        assert np.array_equal(got[m], z[members[slots[m]]])
    # slot 0 everywhere is the 'first' mode
    assert np.array_equal(O.proxy_tokens(z, grid, ratio, "random", np.zeros(M, int)),
                          O.proxy_tokens(z, grid, ratio, "first"))


def test_mean_of_all_single_token_proxies_is_the_average():
    """Averaging the 'random' extraction over every slot gives the window mean."""
    grid, ratio = (2, 8, 6), (2, 4, 3)
    rng = np.random.default_rng(8)
    z = rng.normal(size=(O.num_tokens(grid), 7))
    P = 24
    M = O.num_tokens(grid) // P
    acc = sum(O.proxy_tokens(z, grid, ratio, "random", np.full(M, k)) for k in range(P)) / P
    _close(acc, O.proxy_tokens(z, grid, ratio, "mean"), 1e-13)


def test_giim_with_first_proxies_matches_library_mha():
    grid, ratio, D, heads = (2, 4, 4), (1, 2, 2), 12, 3
    rng = np.random.default_rng(21)
    z = rng.normal(size=(O.num_tokens(grid), D))
    Wp, Wc = _weights(D, 1), _weights(D, 2)
    Pa = z[[0, 2, 8, 10, 16, 18, 24, 26]]  # golden first tokens
    Pp = torch_mha(Pa, Pa, Wp, heads)
    want = z + torch_mha(z, Pp, Wc, heads)
    _close(O.giim(z, grid, ratio, Wp, Wc, heads, proxy_mode="first"), want, 1e-10)


def test_proxy_modes_reject_bad_input():
    z = np.zeros((16, 2))
    with pytest.raises(ValueError):
        O.proxy_tokens(z, (1, 4, 4), (1, 2, 2), "random", np.array([0, 1, 2, 4]))
    with pytest.raises(ValueError):
        O.proxy_tokens(z, (1, 4, 4), (1, 2, 2), "median")


def test_pins_catch_a_last_token_proxy(monkeypatch):
    """A 'first' mode that took each window's last member is caught by the golden."""
    real = O.window_members
    monkeypatch.setattr(O.ptdit_oracle, "window_members", lambda g, r: real(g, r)[:, ::-1])
    with pytest.raises(AssertionError):
        test_proxy_first_and_members_golden()


# ---------------------------------------------------------------- the complete PT-Block

def _norm_params(D, rng):
    return (1.0 + 0.1 * rng.normal(size=D), 0.1 * rng.normal(size=D))


def test_layer_norm_matches_library():
    rng = np.random.default_rng(5)
    x = rng.normal(size=(37, 24)) * 3 + 1
    g, b = _norm_params(24, rng)
    ln = torch.nn.LayerNorm(24, eps=1e-6, dtype=torch.float64)
    with torch.no_grad():
        ln.weight.copy_(torch.from_numpy(g))
        ln.bias.copy_(torch.from_numpy(b))
        want = ln(torch.from_numpy(x)).numpy()
    _close(O.layer_norm(x, g, b, 1e-6), want, 1e-12)
    # unit scale, zero shift: every row has mean 0 and mean square var / (var + eps)
    y = O.layer_norm(x, np.ones(24), np.zeros(24), 1e-6)
    assert np.allclose(y.mean(axis=1), 0, atol=1e-12)
    var = x.var(axis=1)
    assert np.allclose((y ** 2).mean(axis=1), var / (var + 1e-6), rtol=1e-12)


def test_gelu_tanh_matches_library_and_closed_forms():
    x = np.linspace(-9, 9, 1001)
    want = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    _close(O.gelu_tanh(x), want, 1e-14)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert np.allclose(O.gelu_tanh(x) - O.gelu_tanh(-x), x, atol=1e-14)  # gelu(x) - gelu(-x) = x


def test_mlp_matches_library():
    rng = np.random.default_rng(6)
    D, Dh = 12, 48
    x = rng.normal(size=(9, D))
    W1, W2 = rng.normal(size=(Dh, D)) / 4, rng.normal(size=(D, Dh)) / 7
    b1, b2 = rng.normal(size=Dh), rng.normal(size=D)
    net = torch.nn.Sequential(torch.nn.Linear(D, Dh, dtype=torch.float64),
                              torch.nn.GELU(approximate="tanh"),
                              torch.nn.Linear(Dh, D, dtype=torch.float64))
    with torch.no_grad():
        for lin, W, b in ((net[0], W1, b1), (net[2], W2, b2)):
            lin.weight.copy_(torch.from_numpy(W))
            lin.bias.copy_(torch.from_numpy(b))
        want = net(torch.from_numpy(x)).numpy()
    _close(O.mlp(x, W1, b1, W2, b2), want, 1e-12)


def _block_inputs(D, heads, N, L, seed):
    rng = np.random.default_rng(seed)
    W = {m: _weights(D, 30 + i) for i, m in enumerate(("psa", "cross", "wsa", "swsa", "text"))}
    norms = {k: _norm_params(D, rng) for k in ("proxy", "cross", "wsa", "swsa", "text", "mlp")}
    Dh = 4 * D
    mlp_w = (rng.normal(size=(Dh, D)) / math.sqrt(D), 0.1 * rng.normal(size=Dh),
             rng.normal(size=(D, Dh)) / math.sqrt(Dh), 0.1 * rng.normal(size=D))
    return rng.normal(size=(N, D)), W, norms, mlp_w, rng.normal(size=(L, D))


def test_pt_block_matches_library_composition():
    """The block wired from torch's LayerNorm, MultiheadAttention (window branches
    as full attention under the pinned pair mask) and an nn.Sequential MLP."""
    grid, ratio, window, shift, D, heads = (2, 4, 4), (1, 2, 2), (2, 2, 2), (1, 1, 1), 12, 2
    N = O.num_tokens(grid)
    z, W, norms, mlp_w, text = _block_inputs(D, heads, N, 5, 40)

    def tln(x, key):
        ln = torch.nn.LayerNorm(D, eps=1e-6, dtype=torch.float64)
        with torch.no_grad():
            ln.weight.copy_(torch.from_numpy(norms[key][0]))
            ln.bias.copy_(torch.from_numpy(norms[key][1]))
            return ln(torch.from_numpy(x)).numpy()

    Pa = O.averaging(z, grid, ratio)
    Pp = Pa + torch_mha(tln(Pa, "proxy"), tln(Pa, "proxy"), W["psa"], heads)
    z1 = z + torch_mha(tln(z, "cross"), Pp, W["cross"], heads)
    a0 = O.window_allow_matrix(grid, window, (0, 0, 0))
    a1 = O.window_allow_matrix(grid, window, shift)
    z2 = z1 + torch_mha(tln(z1, "wsa"), tln(z1, "wsa"), W["wsa"], heads, a0)
    z3 = z2 + torch_mha(tln(z2, "swsa"), tln(z2, "swsa"), W["swsa"], heads, a1)
    z4 = z3 + torch_mha(tln(z3, "text"), text, W["text"], heads)
    net = torch.nn.Sequential(torch.nn.Linear(D, 4 * D, dtype=torch.float64),
                              torch.nn.GELU(approximate="tanh"),
                              torch.nn.Linear(4 * D, D, dtype=torch.float64))
    with torch.no_grad():
        net[0].weight.copy_(torch.from_numpy(mlp_w[0]))
        net[0].bias.copy_(torch.from_numpy(mlp_w[1]))
        net[2].weight.copy_(torch.from_numpy(mlp_w[2]))
        net[2].bias.copy_(torch.from_numpy(mlp_w[3]))
        want = z4 + net(torch.from_numpy(tln(z4, "mlp"))).numpy()
    got = O.pt_block(z, grid, ratio, window, shift, W, norms, mlp_w, text, heads)
    _close(got, want, 1e-10)


def test_pins_catch_an_unbiased_variance(monkeypatch):
    real = O.ptdit_oracle.layer_norm

    def wrong(x, g, b, eps=1e-6):
        x = np.asarray(x, dtype=np.float64)
        return (x - x.mean(1, keepdims=True)) / np.sqrt(x.var(1, ddof=1, keepdims=True) + eps) * g + b

    monkeypatch.setattr(O, "layer_norm", wrong)
    with pytest.raises(AssertionError):
        test_layer_norm_matches_library()
    monkeypatch.setattr(O, "layer_norm", real)


def test_pins_catch_a_wrong_mlp_term(monkeypatch):
    real = O.ptdit_oracle.mlp
    monkeypatch.setattr(O.ptdit_oracle, "mlp", lambda x, *w: real(x, *w) - x)
    with pytest.raises(AssertionError):
        test_pt_block_matches_library_composition()


# ---------------------------------------------------------------- backward of a TCM branch

BWD_CASES = [  # grid, window, shift: 2D and 3D windows, with and without the roll's wrap masks
    ((1, 4, 4), (1, 2, 2), (0, 0, 0)),
    ((1, 4, 4), (1, 2, 2), (0, 1, 1)),
    ((2, 4, 4), (2, 2, 2), (1, 1, 1)),
    ((2, 4, 6), (2, 2, 3), (1, 1, 2)),
]


def _bwd_inputs(grid, D, seed):
    rng = np.random.default_rng(seed)
    N = O.num_tokens(grid)
    return rng.standard_normal((N, D)), rng.standard_normal((N, D)), _weights(D, seed + 1, scale=0.5)


@pytest.mark.parametrize("grid,window,shift", BWD_CASES)
def test_window_bwd_matches_finite_differences(grid, window, shift):
    """Directional derivatives of L = <dout, out> by central differences in float64,
    along random directions of z and of each weight matrix."""
    D, heads = 8, 2
    z, dout, W = _bwd_inputs(grid, D, 7)
    dz, dW = O.window_self_attention_bwd(z, grid, window, shift, W, heads, dout)

    def L(zz, WW):
        return float(np.sum(dout * O.window_self_attention(zz, grid, window, shift, WW, heads)))

    rng = np.random.default_rng(11)
    eps = 1e-5
    U = rng.standard_normal(z.shape)
    fd = (L(z + eps * U, W) - L(z - eps * U, W)) / (2 * eps)
    assert abs(fd - np.sum(dz * U)) <= 1e-7 * max(1.0, abs(fd))
    for i in range(4):
        V = rng.standard_normal(W[i].shape)
        Wp, Wm = list(W), list(W)
        Wp[i], Wm[i] = W[i] + eps * V, W[i] - eps * V
        fd = (L(z, tuple(Wp)) - L(z, tuple(Wm))) / (2 * eps)
        assert abs(fd - np.sum(dW[i] * V)) <= 1e-7 * max(1.0, abs(fd)), ("dW", i)


def _torch_window_branch(z, grid, window, shift, W, heads):
    """The TCM branch in torch ops (float64): roll, window partition, masked multi-head
    attention, merge, roll back, residual; differentiated by autograd."""
    f, h, w = grid
    N, D = z.shape
    wf, wh, ww = window
    d = D // heads
    zr = torch.roll(z.reshape(f, h, w, D), shifts=tuple(-s for s in shift), dims=(0, 1, 2))
    x = zr.reshape(f // wf, wf, h // wh, wh, w // ww, ww, D).permute(0, 2, 4, 1, 3, 5, 6)
    x = x.reshape(-1, wf * wh * ww, D)
    # a pair attends iff the roll did not wrap between them along any axis: the last
    # s positions of each axis of the rolled grid hold the tokens that wrapped around
    pos = np.stack(np.meshgrid(np.arange(f), np.arange(h), np.arange(w), indexing="ij"), -1)
    side = np.stack([(pos[..., a] >= [f, h, w][a] - shift[a]) & (shift[a] > 0)
                     for a in range(3)], -1)
    side = torch.from_numpy(side.reshape(f // wf, wf, h // wh, wh, w // ww, ww, 3)
                            .transpose(0, 2, 4, 1, 3, 5, 6).reshape(x.shape[0], -1, 3))
    allow = (side[:, :, None, :] == side[:, None, :, :]).all(-1)
    Wq, Wk, Wv, Wo = W

    def split(t):
        return t.reshape(t.shape[0], t.shape[1], heads, d).transpose(1, 2)

    q, k, v = split(x @ Wq.T), split(x @ Wk.T), split(x @ Wv.T)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(d)
    s = s.masked_fill(~allow[:, None], float("-inf"))
    a = (torch.softmax(s, dim=-1) @ v).transpose(1, 2).reshape(x.shape[0], -1, D)
    y = (a @ Wo.T).reshape(f // wf, h // wh, w // ww, wf, wh, ww, D).permute(0, 3, 1, 4, 2, 5, 6)
    y = torch.roll(y.reshape(f, h, w, D), shifts=tuple(shift), dims=(0, 1, 2)).reshape(N, D)
    return z + y


@pytest.mark.parametrize("grid,window,shift", BWD_CASES)
def test_window_bwd_matches_autograd(grid, window, shift):
    D, heads = 16, 4
    z, dout, W = _bwd_inputs(grid, D, 21)
    dz, dW = O.window_self_attention_bwd(z, grid, window, shift, W, heads, dout)
    zt = torch.from_numpy(z).requires_grad_()
    Wt = tuple(torch.from_numpy(x).requires_grad_() for x in W)
    out = _torch_window_branch(zt, grid, window, shift, Wt, heads)
    _close(out.detach().numpy(), O.window_self_attention(z, grid, window, shift, W, heads))
    out.backward(torch.from_numpy(dout))
    _close(dz, zt.grad.numpy())
    for i in range(4):
        _close(dW[i], Wt[i].grad.numpy())


def test_window_bwd_without_residual_drops_dout():
    grid, window, shift = BWD_CASES[2]
    z, dout, W = _bwd_inputs(grid, 8, 3)
    dz, dW = O.window_self_attention_bwd(z, grid, window, shift, W, 2, dout)
    dz0, dW0 = O.window_self_attention_bwd(z, grid, window, shift, W, 2, dout, residual=False)
    _close(dz0 + dout, dz)
    for a, b in zip(dW, dW0):
        _close(a, b)


def test_pins_catch_a_dropped_softmax_jacobian_term(monkeypatch):
    def no_rowsum(Q, K, V, dA, heads, allow=None):
        d = Q.shape[1] // heads
        c = 1.0 / math.sqrt(d)
        dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
        for h in range(heads):
            cols = slice(h * d, (h + 1) * d)
            S = (Q[:, cols] @ K[:, cols].T) * c
            if allow is not None:
                S = np.where(allow, S, -np.inf)
            P = O.softmax_rows(S)
            dV[:, cols] = P.T @ dA[:, cols]
            dS = P * (dA[:, cols] @ V[:, cols].T)  # the rowsum term is missing
            dQ[:, cols] = c * (dS @ K[:, cols])
            dK[:, cols] = c * (dS.T @ Q[:, cols])
        return dQ, dK, dV

    monkeypatch.setattr(O.ptdit_oracle, "attention_heads_bwd", no_rowsum)
    assert _pin_fails(lambda: test_window_bwd_matches_finite_differences(*BWD_CASES[1]))


def test_pins_catch_swapped_query_and_key_gradients(monkeypatch):
    real = O.ptdit_oracle.attention_heads_bwd

    def swapped(*a, **k):
        dQ, dK, dV = real(*a, **k)
        return dK, dQ, dV

    monkeypatch.setattr(O.ptdit_oracle, "attention_heads_bwd", swapped)
    assert _pin_fails(lambda: test_window_bwd_matches_finite_differences(*BWD_CASES[2]))


def test_tcm_bwd_matches_finite_differences():
    """The two-branch composition: directional derivatives of <dout, tcm(z)> in z and in
    one weight of each module."""
    grid, window, shift = (2, 4, 4), (2, 2, 2), (1, 1, 1)
    D, heads = 8, 2
    z, dout, Wa = _bwd_inputs(grid, D, 31)
    Wb = _weights(D, 77, scale=0.5)
    dz, dWa, dWb = O.tcm_bwd(z, grid, window, shift, Wa, Wb, heads, dout)

    def L(zz, A, Bw):
        return float(np.sum(dout * O.tcm(zz, grid, window, shift, A, Bw, heads)))

    rng = np.random.default_rng(5)
    eps = 1e-5
    U = rng.standard_normal(z.shape)
    fd = (L(z + eps * U, Wa, Wb) - L(z - eps * U, Wa, Wb)) / (2 * eps)
    assert abs(fd - np.sum(dz * U)) <= 1e-7 * max(1.0, abs(fd))
    for which, grads in ((0, dWa), (1, dWb)):
        for i in (0, 3):
            V = rng.standard_normal((D, D))
            P, M = [list(Wa), list(Wb)], [list(Wa), list(Wb)]
            P[which][i] = P[which][i] + eps * V
            M[which][i] = M[which][i] - eps * V
            fd = (L(z, tuple(P[0]), tuple(P[1])) - L(z, tuple(M[0]), tuple(M[1]))) / (2 * eps)
            assert abs(fd - np.sum(grads[i] * V)) <= 1e-7 * max(1.0, abs(fd)), (which, i)



# ---------------------------------------------------------------- backward of GIIM

@pytest.mark.parametrize("proxy_residual", [False, True])
def test_giim_bwd_matches_finite_differences(proxy_residual):
    """Directional derivatives of <dout, giim(z)> in z and in every weight of both modules."""
    grid, ratio, D, heads = (2, 4, 4), (1, 2, 2), 8, 2
    rng = np.random.default_rng(9)
    N = O.num_tokens(grid)
    z, dout = rng.standard_normal((N, D)), rng.standard_normal((N, D))
    Wp, Wc = _weights(D, 41, scale=0.5), _weights(D, 42, scale=0.5)
    dz, dWp, dWc = O.giim_bwd(z, grid, ratio, Wp, Wc, heads, dout, proxy_residual=proxy_residual)

    def L(zz, A, C):
        return float(np.sum(dout * O.giim(zz, grid, ratio, A, C, heads,
                                          proxy_residual=proxy_residual)))

    eps = 1e-5
    U = rng.standard_normal(z.shape)
    fd = (L(z + eps * U, Wp, Wc) - L(z - eps * U, Wp, Wc)) / (2 * eps)
    assert abs(fd - np.sum(dz * U)) <= 1e-7 * max(1.0, abs(fd))
    for which, grads in ((0, dWp), (1, dWc)):
        for i in range(4):
            V = rng.standard_normal((D, D))
            P, M = [list(Wp), list(Wc)], [list(Wp), list(Wc)]
            P[which][i] = P[which][i] + eps * V
            M[which][i] = M[which][i] - eps * V
            fd = (L(z, tuple(P[0]), tuple(P[1])) - L(z, tuple(M[0]), tuple(M[1]))) / (2 * eps)
            assert abs(fd - np.sum(grads[i] * V)) <= 1e-7 * max(1.0, abs(fd)), (which, i)


def test_averaging_bwd_is_the_adjoint():
    """<averaging(z), dP> = <z, averaging_bwd(dP)> for random z, dP."""
    grid, ratio = (4, 6, 4), (2, 3, 2)
    rng = np.random.default_rng(3)
    z = rng.standard_normal((O.num_tokens(grid), 5))
    dP = rng.standard_normal((O.averaging(z, grid, ratio).shape[0], 5))
    lhs = np.sum(O.averaging(z, grid, ratio) * dP)
    rhs = np.sum(z * O.averaging_bwd(dP, grid, ratio))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_pins_catch_an_averaging_adjoint_without_the_divisor(monkeypatch):
    real = O.ptdit_oracle.averaging_bwd

    def no_divisor(dP, grid, ratio):
        return real(dP, grid, ratio) * (ratio[0] * ratio[1] * ratio[2])

    monkeypatch.setattr(O.ptdit_oracle, "averaging_bwd", no_divisor)
    assert _pin_fails(lambda: test_giim_bwd_matches_finite_differences(False))


def test_attention_bwd_ignores_a_common_key_shift():
    """Adding one vector m to every key adds c Q_h m_h to each score row, which the
    row softmax removes: P, A and so dQ, dK, dV are unchanged, and the key
    gradients of every head sum to zero over the keys (each row of dS does).  The
    row-attention backward relies on both: it takes dQ against the keys less their
    mean and centres dK over the keys."""
    rng = np.random.default_rng(11)
    nq, nk, D, heads = 9, 7, 8, 2
    Q, K, V, dA = (rng.standard_normal((n, D)) for n in (nq, nk, nk, nq))
    m = 3.0 + rng.standard_normal(D)
    dQ, dK, dV = O.attention_heads_bwd(Q, K, V, dA, heads)
    dQs, dKs, dVs = O.attention_heads_bwd(Q, K + m, V, dA, heads)
    for got, want in ((dQs, dQ), (dKs, dK), (dVs, dV)):
        assert np.allclose(got, want, rtol=0, atol=1e-12)
    assert np.abs(dK.sum(axis=0)).max() <= 1e-12 * np.abs(dK).max()
    # not a property of any key gradient: a dK without the rowsum term fails it
    d = D // heads
    S = (Q[:, :d] @ K[:, :d].T) / np.sqrt(d)
    P = O.softmax_rows(S)
    wrong = (P * (dA[:, :d] @ V[:, :d].T)).T @ Q[:, :d]
    assert np.abs(wrong.sum(axis=0)).max() > 1e-3


def test_block_attn_bwd_matches_finite_differences():
    """The whole path, GIIM then TCM: directional derivatives of <dout, block_attn(z)>
    in z and in one weight of each of the four modules."""
    grid, ratio, window, shift = (2, 4, 4), (1, 2, 2), (2, 2, 2), (1, 1, 1)
    D, heads = 8, 2
    rng = np.random.default_rng(13)
    N = O.num_tokens(grid)
    z, dout = rng.standard_normal((N, D)), rng.standard_normal((N, D))
    W = [_weights(D, 50 + i, scale=0.5) for i in range(4)]
    dz, *dW = O.block_attn_bwd(z, grid, ratio, window, shift, *W, heads, dout)

    def L(zz, Ws):
        return float(np.sum(dout * O.block_attn(zz, grid, ratio, window, shift, *Ws, heads)))

    eps = 1e-5
    U = rng.standard_normal(z.shape)
    fd = (L(z + eps * U, W) - L(z - eps * U, W)) / (2 * eps)
    assert abs(fd - np.sum(dz * U)) <= 1e-7 * max(1.0, abs(fd))
    for m, i in ((0, 1), (1, 0), (2, 2), (3, 3)):
        V = rng.standard_normal((D, D))
        P, M = [list(w) for w in W], [list(w) for w in W]
        P[m][i] = P[m][i] + eps * V
        M[m][i] = M[m][i] - eps * V
        fd = (L(z, [tuple(w) for w in P]) - L(z, [tuple(w) for w in M])) / (2 * eps)
        assert abs(fd - np.sum(dW[m][i] * V)) <= 1e-7 * max(1.0, abs(fd)), (m, i)
