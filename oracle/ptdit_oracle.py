"""Float64 CPU oracle for the PT-DiT block-attention path (GIIM + TCM).

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the CUDA library computes.  Only the test suite, the
``smoke()`` self-check and the bench's CPU-baseline / reference leg may import
it; the product path never does.  It imports nothing from the product package
and shares no code, table or helper with the CUDA sources.

Sources.  Citations name the page and the part of it that defines the step:

  [T2X]  "Qihoo-T2X -- Proxy-Tokenized DiT for Text-to-Any-Task" (a reading note
         of the PT-DiT paper): §3 Method -- Eq. GIIM, Eq. TCM, the complexity
         paragraph, the compression-ratio schedule; the code-comparison section
         (get_proxy_token, ProxyTokensTransformerBlock.forward); Fig. 2 reading
         (row-major token index).
  [NEWS] "Qihoo-T2X - A high-efficiency multimodal generative model ...":
         Technical Principles (proxy averaging, window + shifted-window SA).

Everything is float64.  Inputs may be float32 or bf16-valued arrays; they are
widened once and never rounded again, so this is the exact result of the
definition up to float64 rounding.

Readings taken where the pages are silent or ambiguous:
  * softmax scale is 1/sqrt(d), d = D / heads (standard multi-head attention);
  * proxy self-attention is SA(P_a) with no norm and no residual, as in
    Eq. GIIM; the code listing's "+ proxy" residual is the option
    ``proxy_residual=True``; layer norms are not part of this path;
  * the zero-initialised ``linear_1_visual`` after the cross-attention is a
    bias-free linear, so it is folded into the cross-attention's W_o; no
    layer has a bias;
  * WSA and SWSA each have their own Q/K/V/O weights (Swin style);
  * the shifted window follows Swin: roll the grid by -s along (f, h, w),
    partition into windows, attend inside each window with the region mask
    (a pair may attend iff it lies in the same slice of the rolled grid along
    every axis, i.e. the roll did not wrap between them), merge, roll by +s;
    masked pairs get probability exactly 0;
  * tokens are flattened row-major over (f, h, w); windows and proxies are
    numbered row-major over the window grid and tokens inside a window
    row-major over (t, y, x);
  * every grid extent must be divisible by its ratio and its window.

Backward (training) of GIIM: ``giim_bwd`` (``averaging_bwd`` is the averaging's
adjoint).  Backward of a TCM branch: ``window_self_attention_bwd`` returns
dL/dz and the four weight gradients for a given dL/dout, by the chain rule
written out per window and head (``attention_heads_bwd`` holds the softmax
Jacobian step); roll and window partition are row permutations, so their
adjoints are the inverse permutations.

Every function here is pinned by the CPU tests (tests/test_oracle_pins.py)
against closed forms, library routines, brute force, hand-derived fixtures or,
for the gradients, central finite differences and torch autograd.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# Query rows are processed in chunks of this many so the score matrix of a
# very long sequence stays small.  Rows are independent, so chunking changes
# no arithmetic.
_ROW_CHUNK = 4096

# Heads are independent: above this many scores per head they run on a pool
# of host threads (numpy releases the GIL in its matrix products and
# element-wise passes).  Each head's arithmetic is the same either way and
# writes its own columns of the result, so the output is bit-identical.
_PARALLEL_SCORES = 1 << 22
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1)))
    return _POOL


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def _check_divisible(grid, part, what):
    for L, p in zip(grid, part):
        if p <= 0 or L % p:
            raise ValueError(f"grid {tuple(grid)} is not divisible by {what} {tuple(part)}")


# --------------------------------------------------------------------------
# Token grid  [T2X Fig. 2 reading: row-major flattening; §3 "reshape z_s to f×h×w"]
# --------------------------------------------------------------------------

def num_tokens(grid) -> int:
    f, h, w = grid
    return f * h * w


def token_coords(grid):
    """(t, y, x) of every token of the flattened f×h×w grid, t slowest, x fastest."""
    f, h, w = grid
    t, y, x = np.meshgrid(np.arange(f), np.arange(h), np.arange(w), indexing="ij")
    return t.ravel(), y.ravel(), x.ravel()


# --------------------------------------------------------------------------
# GIIM step 1: Averaging  [T2X §3 Eq. GIIM "Averaging"; get_proxy_token(mode="mean")]
# --------------------------------------------------------------------------

def proxy_index(grid, ratio) -> np.ndarray:
    """Index m of the proxy token that each latent token is averaged into.

    A proxy window is p_f×p_h×p_w tokens; proxies are numbered row-major over
    the (f/p_f, h/p_h, w/p_w) grid of windows.
    """
    _check_divisible(grid, ratio, "ratio")
    f, h, w = grid
    pf, ph, pw = ratio
    t, y, x = token_coords(grid)
    return ((t // pf) * (h // ph) + (y // ph)) * (w // pw) + (x // pw)


def averaging(z, grid, ratio) -> np.ndarray:
    """P_a: the mean of z_s over each p_f×p_h×p_w window.  z [N, D] -> [M, D]."""
    _check_divisible(grid, ratio, "ratio")
    f, h, w = grid
    pf, ph, pw = ratio
    z = _f64(z)
    D = z.shape[1]
    blocks = z.reshape(f // pf, pf, h // ph, ph, w // pw, pw, D)
    return blocks.mean(axis=(1, 3, 5)).reshape(-1, D)


def window_members(grid, ratio) -> np.ndarray:
    """[M, P]: the tokens of each proxy window, windows row-major over the window
    grid, members row-major (t, y, x) inside the window."""
    _check_divisible(grid, ratio, "ratio")
    f, h, w = grid
    pf, ph, pw = ratio
    idx = np.arange(num_tokens(grid)).reshape(f // pf, pf, h // ph, ph, w // pw, pw)
    return idx.transpose(0, 2, 4, 1, 3, 5).reshape(-1, pf * ph * pw)


def proxy_tokens(z, grid, ratio, mode="mean", slots=None) -> np.ndarray:
    """The proxy tokens of each window under the three extraction modes that the
    pages compare  [T2X code-comparison section, get_proxy_token(mode=...); §3
    Method ablation notes: Average / Top-Left / Random].

    mean:   the window mean (Eq. GIIM, the method's choice);
    first:  the window's first member in (t, y, x) order, i.e. its top-left
            token in its first frame;
    random: member slots[m] of window m; the random draw itself is an input
            (slots, an int array [M] with 0 <= slots[m] < p_f p_h p_w).
    """
    if mode == "mean":
        return averaging(z, grid, ratio)
    z = _f64(z)
    members = window_members(grid, ratio)
    if mode == "first":
        return z[members[:, 0]]
    if mode == "random":
        slots = np.asarray(slots)
        if slots.shape != (members.shape[0],) or np.any(slots < 0) or np.any(slots >= members.shape[1]):
            raise ValueError("slots must hold one member index per window")
        return z[members[np.arange(members.shape[0]), slots]]
    raise ValueError(f"unknown proxy mode {mode!r}")


# --------------------------------------------------------------------------
# Multi-head attention (the SA / CS / WSA / SWSA operator of Eq. GIIM, Eq. TCM)
# --------------------------------------------------------------------------

def project(x, W) -> np.ndarray:
    """y = x W^T: a bias-free linear layer with W stored [out][in]."""
    return _f64(x) @ _f64(W).T


def softmax_rows(S) -> np.ndarray:
    """Row softmax; -inf entries get probability 0."""
    S = S - S.max(axis=1, keepdims=True)
    E = np.exp(S)
    return E / E.sum(axis=1, keepdims=True)


def attention_heads(Q, K, V, heads, allow=None) -> np.ndarray:
    """Per head h: softmax(Q_h K_h^T / sqrt(d)) V_h, heads concatenated (no output projection).

    Q [Nq, D], K and V [Nk, D]; head h owns columns h*d .. h*d+d-1.  ``allow``
    is an optional bool [Nq, Nk]; False removes key j from query i's softmax.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Nq, D = Q.shape
    if D % heads:
        raise ValueError("D must be divisible by heads")
    d = D // heads
    scale = 1.0 / math.sqrt(d)
    out = np.empty((Nq, D))

    parallel = heads > 1 and Nq * K.shape[0] >= _PARALLEL_SCORES
    # concurrent heads each hold one chunk of scores: keep a chunk near 16 M entries
    chunk = max(64, min(_ROW_CHUNK, (1 << 24) // max(1, K.shape[0]))) if parallel else _ROW_CHUNK

    def head(h):
        cols = slice(h * d, (h + 1) * d)
        for q0 in range(0, Nq, chunk):
            q1 = min(Nq, q0 + chunk)
            S = (Q[q0:q1, cols] @ K[:, cols].T) * scale
            if allow is not None:
                S = np.where(allow[q0:q1], S, -np.inf)
            out[q0:q1, cols] = softmax_rows(S) @ V[:, cols]

    if parallel:
        list(_pool().map(head, range(heads)))
    else:
        for h in range(heads):
            head(h)
    return out


def multihead_attention(x_q, x_kv, W, heads, allow=None) -> np.ndarray:
    """MHA with queries from x_q and keys/values from x_kv; W = (Wq, Wk, Wv, Wo), each [D][D]."""
    Wq, Wk, Wv, Wo = W
    O = attention_heads(project(x_q, Wq), project(x_kv, Wk), project(x_kv, Wv), heads, allow)
    return project(O, Wo)


# --------------------------------------------------------------------------
# GIIM  [T2X §3 Eq. GIIM: z_s = CS(z_s, SA(Averaging(z_s))); the code listing's proxy
#        self-attention and cross-attention]
# --------------------------------------------------------------------------

def proxy_self_attention(z, grid, ratio, W_psa, heads, proxy_residual=False, proxy_mode="mean",
                         slots=None) -> np.ndarray:
    """P' = SA(Averaging(z_s)) (+ P_a when proxy_residual); proxy_mode and slots
    select another extraction (proxy_tokens)."""
    Pa = proxy_tokens(z, grid, ratio, proxy_mode, slots)
    Pp = multihead_attention(Pa, Pa, W_psa, heads)
    return Pp + Pa if proxy_residual else Pp


def giim(z, grid, ratio, W_psa, W_cross, heads, *, proxy_residual=False, residual=True,
         rows=None, proxy_mode="mean", slots=None) -> np.ndarray:
    """GIIM of one batch item.  z [N, D] -> [N, D].

    Cross-attention CS takes every latent token as the query and the proxies
    P' as keys and values; its result is added to z_s (``residual``).  With
    ``rows`` given, only those output rows are computed and the others are NaN.
    """
    z = _f64(z)
    Pp = proxy_self_attention(z, grid, ratio, W_psa, heads, proxy_residual, proxy_mode, slots)
    if rows is None:
        cs = multihead_attention(z, Pp, W_cross, heads)
        return z + cs if residual else cs
    rows = np.asarray(rows)
    out = np.full_like(z, np.nan)
    cs = multihead_attention(z[rows], Pp, W_cross, heads)
    out[rows] = z[rows] + cs if residual else cs
    return out


# --------------------------------------------------------------------------
# TCM  [T2X §3 Eq. TCM; window_shift / window_Ishift; NEWS Technical Principles]
# --------------------------------------------------------------------------

def averaging_bwd(dP, grid, ratio) -> np.ndarray:
    """Adjoint of averaging: every token of window m receives dP[m] / (p_f p_h p_w).
    dP [M, D] -> [N, D]."""
    _check_divisible(grid, ratio, "ratio")
    f, h, w = grid
    pf, ph, pw = ratio
    dP = _f64(dP)
    D = dP.shape[1]
    g = dP.reshape(f // pf, 1, h // ph, 1, w // pw, 1, D) / (pf * ph * pw)
    return np.broadcast_to(g, (f // pf, pf, h // ph, ph, w // pw, pw, D)).reshape(-1, D).copy()


def giim_bwd(z, grid, ratio, W_psa, W_cross, heads, dout, *, proxy_residual=False,
             residual=True):
    """Backward of giim (window-mean proxies) on one batch item: the chain rule through
    the cross-attention (queries from z, keys and values from P'), the proxy
    self-attention and the averaging.  Returns (dz, dW_psa, dW_cross), the weight
    gradients in the weights' [out][in] storage.
        out = z + Ac Wco^T,  Ac = MHA core(z Wcq^T, P' Wck^T, P' Wcv^T)
        P'  = Ap Wpo^T (+ P_a),  Ap = MHA core(P_a Wpq^T, P_a Wpk^T, P_a Wpv^T)
        P_a = averaging(z)
    """
    z, dout = _f64(z), _f64(dout)
    Wpq, Wpk, Wpv, Wpo = (_f64(x) for x in W_psa)
    Wcq, Wck, Wcv, Wco = (_f64(x) for x in W_cross)
    # forward, keeping what the backward reads
    Pa = averaging(z, grid, ratio)
    Pq, Pk, Pv = Pa @ Wpq.T, Pa @ Wpk.T, Pa @ Wpv.T
    Ap = attention_heads(Pq, Pk, Pv, heads)
    Pp = Ap @ Wpo.T + (Pa if proxy_residual else 0.0)
    Cq, Ck, Cv = z @ Wcq.T, Pp @ Wck.T, Pp @ Wcv.T
    Ac = attention_heads(Cq, Ck, Cv, heads)
    # cross-attention and its projections
    dWco = dout.T @ Ac
    dCq, dCk, dCv = attention_heads_bwd(Cq, Ck, Cv, dout @ Wco, heads)
    dz = dCq @ Wcq
    dWcq, dWck, dWcv = dCq.T @ z, dCk.T @ Pp, dCv.T @ Pp
    dPp = dCk @ Wck + dCv @ Wcv
    # proxy self-attention and its projections
    dWpo = dPp.T @ Ap
    dPq, dPk, dPv = attention_heads_bwd(Pq, Pk, Pv, dPp @ Wpo, heads)
    dPa = dPq @ Wpq + dPk @ Wpk + dPv @ Wpv + (dPp if proxy_residual else 0.0)
    dWpq, dWpk, dWpv = dPq.T @ Pa, dPk.T @ Pa, dPv.T @ Pa
    # the averaging
    dz = dz + averaging_bwd(dPa, grid, ratio)
    if residual:
        dz = dz + dout
    return dz, (dWpq, dWpk, dWpv, dWpo), (dWcq, dWck, dWcv, dWco)


def _to_windows(g, window) -> np.ndarray:
    """[f, h, w, ...] -> [num_windows, n, ...]: windows row-major, slots row-major (t, y, x)."""
    f, h, w = g.shape[:3]
    wf, wh, ww = window
    rest = g.shape[3:]
    x = g.reshape(f // wf, wf, h // wh, wh, w // ww, ww, *rest)
    x = x.transpose(0, 2, 4, 1, 3, 5, *range(6, 6 + len(rest)))
    return x.reshape((f // wf) * (h // wh) * (w // ww), wf * wh * ww, *rest)


def _from_windows(win, grid, window) -> np.ndarray:
    """Inverse of _to_windows: [num_windows, n, ...] -> [f, h, w, ...]."""
    f, h, w = grid
    wf, wh, ww = window
    rest = win.shape[2:]
    x = win.reshape(f // wf, h // wh, w // ww, wf, wh, ww, *rest)
    x = x.transpose(0, 3, 1, 4, 2, 5, *range(6, 6 + len(rest)))
    return x.reshape(f, h, w, *rest)


def window_token_map(grid, window, shift) -> np.ndarray:
    """[num_windows, n]: the original token index at each (window, slot) of the rolled grid."""
    _check_divisible(grid, window, "window")
    idx = np.arange(num_tokens(grid)).reshape(grid)
    rolled = np.roll(idx, shift=tuple(-s for s in shift), axis=(0, 1, 2))
    return _to_windows(rolled, window)


def _region_labels_1d(L, wsize, s) -> np.ndarray:
    """Swin's three slices of one axis of the rolled grid.

    Positions [0, L-w) -> 0, [L-w, L-s) -> 1, [L-s, L) -> 2.  Only the last
    window of the axis mixes tokens that the roll wrapped (label 2) with
    tokens it did not (label 1).  With s == 0 every position is 0.
    """
    lab = np.zeros(L, dtype=np.int64)
    if s > 0:
        lab[L - wsize:L - s] = 1
        lab[L - s:] = 2
    return lab


def window_region_labels(grid, window, shift) -> np.ndarray:
    """[num_windows, n] region label of each (window, slot); slots attend iff labels are equal."""
    _check_divisible(grid, window, "window")
    f, h, w = grid
    for s, wd in zip(shift, window):
        if not 0 <= s < wd:
            raise ValueError("shift must satisfy 0 <= s < window")
    lt = _region_labels_1d(f, window[0], shift[0])[:, None, None]
    ly = _region_labels_1d(h, window[1], shift[1])[None, :, None]
    lx = _region_labels_1d(w, window[2], shift[2])[None, None, :]
    return _to_windows((lt * 3 + ly) * 3 + lx, window)


def window_self_attention(z, grid, window, shift, W, heads, *, residual=True,
                          windows=None) -> np.ndarray:
    """One TCM branch on one batch item: WSA for shift (0,0,0), SWSA otherwise.

    roll(z, -s) -> partition into windows -> masked MHA inside each window ->
    merge -> roll(+s) (-> + z).  With ``windows`` (indices of rolled-grid
    windows) only those windows are computed and every other row is NaN.
    """
    f, h, w = grid
    z = _f64(z)
    N, D = z.shape
    zr = np.roll(z.reshape(f, h, w, D), shift=tuple(-s for s in shift), axis=(0, 1, 2))
    zw = _to_windows(zr, window)
    lab = window_region_labels(grid, window, shift)
    yw = np.full_like(zw, np.nan)
    for k in (range(zw.shape[0]) if windows is None else windows):
        allow = lab[k][:, None] == lab[k][None, :]
        yw[k] = multihead_attention(zw[k], zw[k], W, heads, allow)
    y = np.roll(_from_windows(yw, grid, window), shift=tuple(shift), axis=(0, 1, 2)).reshape(N, D)
    return z + y if residual else y


def attention_heads_bwd(Q, K, V, dA, heads, allow=None):
    """Gradients of attention_heads with respect to Q, K and V, given dA = dL/dA.

    Per head h, with S = c Q_h K_h^T (c = 1/sqrt(d), masked entries -inf),
    P = softmax(S) row by row and A_h = P V_h, the chain rule gives
        dV_h = P^T dA_h,   dP = dA_h V_h^T,
        dS   = P * (dP - rowsum(P * dP))     (the softmax Jacobian, row by row),
        dQ_h = c dS K_h,   dK_h = c dS^T Q_h.
    Masked entries have P = 0, so they pass no gradient.  Returns (dQ, dK, dV).
    """
    Q, K, V, dA = _f64(Q), _f64(K), _f64(V), _f64(dA)
    d = Q.shape[1] // heads
    c = 1.0 / math.sqrt(d)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for h in range(heads):
        cols = slice(h * d, (h + 1) * d)
        S = (Q[:, cols] @ K[:, cols].T) * c
        if allow is not None:
            S = np.where(allow, S, -np.inf)
        P = softmax_rows(S)
        dV[:, cols] = P.T @ dA[:, cols]
        dP = dA[:, cols] @ V[:, cols].T
        dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
        dQ[:, cols] = c * (dS @ K[:, cols])
        dK[:, cols] = c * (dS.T @ Q[:, cols])
    return dQ, dK, dV


def window_self_attention_bwd(z, grid, window, shift, W, heads, dout, *, residual=True):
    """Backward of window_self_attention on one batch item (one TCM branch).

    out = (z +) roll(+s)(merge(Y_k)), Y_k = MHA(Z_k, Z_k) Wo^T over each window
    Z_k of roll(-s)(z).  Given dout = dL/dout, returns
    (dz, (dWq, dWk, dWv, dWo)): dL/dz and the weight gradients, each [D][D] in
    the [out][in] storage of W.  Roll and window partition are permutations of
    the rows, so their adjoints are the inverse permutations: the gradient rows
    are gathered into windows exactly as z was, and scattered back the same
    way.  Per window, with X = Z_k, A = attention output, dY = the window's
    rows of dout:
        dWo += dY^T A,  dA = dY Wo,  (dQ, dK, dV) = attention_heads_bwd(...),
        dWq += dQ^T X,  dWk += dK^T X,  dWv += dV^T X,
        dX = dQ Wq + dK Wk + dV Wv.
    """
    f, h, w = grid
    z, dout = _f64(z), _f64(dout)
    Wq, Wk, Wv, Wo = (_f64(x) for x in W)
    N, D = z.shape
    back = tuple(-s for s in shift)
    zw = _to_windows(np.roll(z.reshape(f, h, w, D), shift=back, axis=(0, 1, 2)), window)
    gw = _to_windows(np.roll(dout.reshape(f, h, w, D), shift=back, axis=(0, 1, 2)), window)
    lab = window_region_labels(grid, window, shift)
    dWq, dWk, dWv, dWo = (np.zeros((D, D)) for _ in range(4))
    dxw = np.empty_like(zw)
    for k in range(zw.shape[0]):
        allow = lab[k][:, None] == lab[k][None, :]
        X, dY = zw[k], gw[k]
        Q, K, V = X @ Wq.T, X @ Wk.T, X @ Wv.T
        A = attention_heads(Q, K, V, heads, allow)
        dWo += dY.T @ A
        dQ, dK, dV = attention_heads_bwd(Q, K, V, dY @ Wo, heads, allow)
        dWq += dQ.T @ X
        dWk += dK.T @ X
        dWv += dV.T @ X
        dxw[k] = dQ @ Wq + dK @ Wk + dV @ Wv
    dz = np.roll(_from_windows(dxw, grid, window), shift=tuple(shift), axis=(0, 1, 2)).reshape(N, D)
    if residual:
        dz = dz + dout
    return dz, (dWq, dWk, dWv, dWo)


def tcm_bwd(z, grid, window, shift, W_wsa, W_swsa, heads, dout, *, residual=True):
    """Backward of tcm: the chain rule through its two branches.  z^ = WSA(z) (+ z) is
    recomputed; SWSA's backward at z^ gives dL/dz^ and SWSA's weight gradients, WSA's
    backward at z with dL/dz^ gives dL/dz and WSA's.  Returns (dz, dW_wsa, dW_swsa)."""
    zh = window_self_attention(z, grid, window, (0, 0, 0), W_wsa, heads, residual=residual)
    dzh, dW_swsa = window_self_attention_bwd(zh, grid, window, shift, W_swsa, heads, dout,
                                             residual=residual)
    dz, dW_wsa = window_self_attention_bwd(z, grid, window, (0, 0, 0), W_wsa, heads, dzh,
                                           residual=residual)
    return dz, dW_wsa, dW_swsa


def tcm(z, grid, window, shift, W_wsa, W_swsa, heads, *, residual=True) -> np.ndarray:
    """ẑ = WSA(z) + z;  z_w = SWSA(ẑ) + ẑ   [T2X §3 Eq. TCM]."""
    zh = window_self_attention(z, grid, window, (0, 0, 0), W_wsa, heads, residual=residual)
    return window_self_attention(zh, grid, window, shift, W_swsa, heads, residual=residual)


def block_attn(z, grid, ratio, window, shift, W_psa, W_cross, W_wsa, W_swsa, heads, *,
               proxy_residual=False, residual=True) -> np.ndarray:
    """GIIM then TCM on one batch item  [T2X code listing: ProxyTokensTransformerBlock.forward,
    its GIIM and TCM attentions]."""
    z1 = giim(z, grid, ratio, W_psa, W_cross, heads, proxy_residual=proxy_residual,
              residual=residual)
    return tcm(z1, grid, window, shift, W_wsa, W_swsa, heads, residual=residual)


def block_attn_bwd(z, grid, ratio, window, shift, W_psa, W_cross, W_wsa, W_swsa, heads, dout,
                   *, proxy_residual=False, residual=True):
    """Backward of block_attn on one batch item: z1 = giim(z) is recomputed, TCM's
    backward at z1 gives dL/dz1 and both window modules' weight gradients, GIIM's
    backward at z with dL/dz1 gives dL/dz and the proxy and cross modules'.
    Returns (dz, dW_psa, dW_cross, dW_wsa, dW_swsa)."""
    z1 = giim(z, grid, ratio, W_psa, W_cross, heads, proxy_residual=proxy_residual,
              residual=residual)
    dz1, dW_wsa, dW_swsa = tcm_bwd(z1, grid, window, shift, W_wsa, W_swsa, heads, dout,
                                   residual=residual)
    dz, dW_psa, dW_cross = giim_bwd(z, grid, ratio, W_psa, W_cross, heads, dz1,
                                    proxy_residual=proxy_residual, residual=residual)
    return dz, dW_psa, dW_cross, dW_wsa, dW_swsa


def block_attn_rows(z, grid, ratio, window, shift, W_psa, W_cross, W_wsa, W_swsa, heads, rows,
                    *, proxy_residual=False, residual=True) -> np.ndarray:
    """block_attn at the listed token rows only, from the full input z.

    Computes just the dependency closure: the shifted windows holding ``rows``
    need z2 on their tokens; those need the unshifted windows holding them,
    which need z1 on their tokens; z1 rows need the full proxy set.  Every
    row outside the closure stays NaN, so a missed dependency cannot pass.
    Returns [len(rows), D].
    """
    rows = np.asarray(rows)
    smap = window_token_map(grid, window, shift)
    umap = window_token_map(grid, window, (0, 0, 0))
    n = smap.shape[1]
    swin_of = np.empty(num_tokens(grid), dtype=np.int64)
    swin_of[smap.ravel()] = np.repeat(np.arange(smap.shape[0]), n)
    uwin_of = np.empty(num_tokens(grid), dtype=np.int64)
    uwin_of[umap.ravel()] = np.repeat(np.arange(umap.shape[0]), n)
    S2 = np.unique(swin_of[rows])
    T2 = smap[S2].ravel()
    S1 = np.unique(uwin_of[T2])
    T1 = umap[S1].ravel()
    z1 = giim(z, grid, ratio, W_psa, W_cross, heads, proxy_residual=proxy_residual,
              residual=residual, rows=T1)
    z2 = window_self_attention(z1, grid, window, (0, 0, 0), W_wsa, heads, residual=residual,
                               windows=S1)
    z3 = window_self_attention(z2, grid, window, shift, W_swsa, heads, residual=residual,
                               windows=S2)
    return z3[rows]


# --------------------------------------------------------------------------
# Second, independent formulation of TCM: full attention with a pair mask
# --------------------------------------------------------------------------

def window_allow_matrix(grid, window, shift) -> np.ndarray:
    """bool [N, N]: token i may attend token j.

    Derived from coordinates rather than from the roll: i and j must fall in
    the same window of the grid shifted cyclically by s (position (c - s) mod L
    along each axis) AND their offset along every axis must be the same before
    and after the shift, i.e. the shift did not wrap between them.  Any
    integer shift works here, negative ones included.
    """
    _check_divisible(grid, window, "window")
    t, y, x = token_coords(grid)
    allow = np.ones((t.size, t.size), dtype=bool)
    for c, L, wd, s in zip((t, y, x), grid, window, shift):
        cr = (c - s) % L
        allow &= (cr[:, None] // wd) == (cr[None, :] // wd)
        allow &= (cr[:, None] - cr[None, :]) == (c[:, None] - c[None, :])
    return allow


def masked_self_attention(z, W, heads, allow, *, residual=True) -> np.ndarray:
    """Full self-attention over all tokens with a pair mask (+ z)."""
    z = _f64(z)
    y = multihead_attention(z, z, W, heads, allow)
    return z + y if residual else y


# --------------------------------------------------------------------------
# The complete PT-Block  [T2X §3 Method: "PT-Block (GIIM + TCM + text
# cross-attn + MLP)", the block diagram; code-comparison section,
# ProxyTokensTransformerBlock.forward]
#
# Readings (the pages name the sub-layers and their order but not the norms'
# form, the MLP's width or activation, nor where each norm sits):
#   * every sub-layer is pre-norm with a residual: x <- x + F(LN(x)); the proxy
#     self-attention normalises the proxies (proxy_norm1) and adds them back,
#     as the listing's proxy self-attention does;
#   * LN is a LayerNorm over D with a per-channel scale and shift and
#     epsilon eps; its variance is the population (biased) variance;
#   * the text cross-attention takes the normalised latents as queries and the
#     text tokens (already projected to width D outside the block) as keys and
#     values;
#   * the MLP is fc1 (D -> Dh, bias) -> GELU, tanh form -> fc2 (Dh -> D, bias),
#     the feed-forward of the DiT / PixArt-alpha blocks PT-DiT is compared with;
#   * attention projections have no bias (as in the rest of this path).
# --------------------------------------------------------------------------

def layer_norm(x, gamma, beta, eps=1e-6) -> np.ndarray:
    """Per row: (x - mean) / sqrt(var + eps) * gamma + beta, var the mean squared deviation."""
    x = _f64(x)
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * _f64(gamma) + _f64(beta)


def gelu_tanh(x) -> np.ndarray:
    """GELU in its tanh form: x/2 (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = _f64(x)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def mlp(x, W1, b1, W2, b2) -> np.ndarray:
    """fc2(GELU(fc1(x))): W1 [Dh][D], b1 [Dh], W2 [D][Dh], b2 [D]."""
    return project(gelu_tanh(project(x, W1) + _f64(b1)), W2) + _f64(b2)


def pt_block(z, grid, ratio, window, shift, W, norms, mlp_w, text, heads, *, eps=1e-6,
             proxy_mode="mean", slots=None) -> np.ndarray:
    """One complete PT-Block on one batch item.  z [N, D] -> [N, D].

    W: {"psa", "cross", "wsa", "swsa", "text"} -> (Wq, Wk, Wv, Wo);
    norms: {"proxy", "cross", "wsa", "swsa", "text", "mlp"} -> (gamma, beta);
    mlp_w: (W1, b1, W2, b2); text: [L, D] text tokens.
    """
    z = _f64(z)
    ln = {k: (lambda x, g=g, b=b: layer_norm(x, g, b, eps)) for k, (g, b) in norms.items()}
    Pa = proxy_tokens(z, grid, ratio, proxy_mode, slots)
    Pn = ln["proxy"](Pa)
    Pp = Pa + multihead_attention(Pn, Pn, W["psa"], heads)
    z1 = z + multihead_attention(ln["cross"](z), Pp, W["cross"], heads)
    z2 = z1 + window_self_attention(ln["wsa"](z1), grid, window, (0, 0, 0), W["wsa"], heads,
                                    residual=False)
    z3 = z2 + window_self_attention(ln["swsa"](z2), grid, window, shift, W["swsa"], heads,
                                    residual=False)
    z4 = z3 + multihead_attention(ln["text"](z3), _f64(text), W["text"], heads)
    return z4 + mlp(ln["mlp"](z4), *mlp_w)
