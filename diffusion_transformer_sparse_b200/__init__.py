"""PT-DiT block attention (GIIM + TCM) on NVIDIA B200: ctypes binding over libptdit.so.

Every function here only marshals arguments: torch CUDA tensors become device
pointers, the current torch stream becomes the stream argument, and a non-zero
status becomes a PtditError.  All arithmetic runs in the CUDA library; there is
no CPU path.  If libptdit.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libptdit.so")

PTDIT_F32, PTDIT_BF16 = 0, 1
PTDIT_PROXY_RESIDUAL = 0x1
PTDIT_NO_RESIDUAL = 0x2
PTDIT_PROXY_MEAN, PTDIT_PROXY_FIRST, PTDIT_PROXY_RANDOM = 0, 1, 2
PROXY_MODES = {"mean": PTDIT_PROXY_MEAN, "first": PTDIT_PROXY_FIRST, "random": PTDIT_PROXY_RANDOM}
# status codes (include/ptdit.h)
(PTDIT_OK, PTDIT_ERR_NULL, PTDIT_ERR_SHAPE, PTDIT_ERR_DTYPE, PTDIT_ERR_WORKSPACE, PTDIT_ERR_CUDA,
 PTDIT_ERR_TIMEOUT, PTDIT_ERR_ALIGN, PTDIT_ERR_ALIAS) = range(9)
KINDS = ("average", "gemm", "attn_proxy", "attn_cross", "attn_window", "attn_dense", "norm",
         "attn_text", "attn_window_bwd", "wgrad", "transpose", "attn_rows_bwd",
         "attn_window_fused")

# Every symbol declared in include/ptdit.h.
EXPORTS = (
    "ptdit_proxy_average", "ptdit_workspace_bytes", "ptdit_giim", "ptdit_window_attn",
    "ptdit_tcm", "ptdit_block_attn", "ptdit_full_attn", "ptdit_strerror", "ptdit_last_error",
    "ptdit_debug_proxy_map", "ptdit_debug_window_map", "ptdit_device_status", "ptdit_debug_timeout", "ptdit_timing_enable",
    "ptdit_timing_read", "ptdit_launch_count", "ptdit_window_attn_static",
    "ptdit_debug_thl_map", "ptdit_debug_thl_units", "ptdit_debug_gemm_schedule",
    "ptdit_proxy_extract", "ptdit_giim_ex", "ptdit_pt_block", "ptdit_pt_block_workspace_bytes",
    "ptdit_debug_wait_limit", "ptdit_window_attn_bwd", "ptdit_window_attn_bwd_workspace_bytes",
    "ptdit_tcm_bwd", "ptdit_tcm_bwd_workspace_bytes", "ptdit_giim_bwd",
    "ptdit_giim_bwd_workspace_bytes", "ptdit_block_attn_bwd",
    "ptdit_block_attn_bwd_workspace_bytes", "ptdit_window_fused",
    "ptdit_block_attn_train_workspace_bytes", "ptdit_block_attn_fwd_train",
    "ptdit_block_attn_bwd_saved",
)


class PtditError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"ptdit error {code}: {message}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("F", ctypes.c_int), ("H", ctypes.c_int),
                ("W", ctypes.c_int), ("D", ctypes.c_int), ("heads", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class AttnW(ctypes.Structure):
    _fields_ = [("wq", ctypes.c_void_p), ("wk", ctypes.c_void_p), ("wv", ctypes.c_void_p),
                ("wo", ctypes.c_void_p)]


class AttnWgrad(ctypes.Structure):
    _fields_ = [("dwq", ctypes.c_void_p), ("dwk", ctypes.c_void_p), ("dwv", ctypes.c_void_p),
                ("dwo", ctypes.c_void_p)]


class NormW(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p)]


class BlockW(ctypes.Structure):
    _fields_ = ([(m, AttnW) for m in ("psa", "cross", "wsa", "swsa", "text")] +
                [("norm_" + k, NormW) for k in ("proxy", "cross", "wsa", "swsa", "text", "mlp")] +
                [("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                 ("b2", ctypes.c_void_p), ("mlp_hidden", ctypes.c_int), ("eps", ctypes.c_float)])


_lib = None
Int3 = ctypes.c_int * 3
_P = ctypes.c_void_p
_S = ctypes.POINTER(Shape)
_W = ctypes.POINTER(AttnW)
_I3 = ctypes.POINTER(ctypes.c_int)
_IP = ctypes.POINTER(ctypes.c_int)  # an int the call writes


def lib() -> ctypes.CDLL:
    """The loaded libptdit.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "diffusion_transformer_sparse_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "ptdit_proxy_average": (ctypes.c_int, [_S, _I3, _P, _P, _P]),
            "ptdit_workspace_bytes": (ctypes.c_size_t, [_S, _I3, _I3]),
            "ptdit_proxy_extract": (ctypes.c_int, [_S, _I3, ctypes.c_int, _P, _P, _P, _P]),
            "ptdit_pt_block_workspace_bytes": (ctypes.c_size_t, [_S, _I3, ctypes.c_int,
                                                                 ctypes.c_int]),
            "ptdit_pt_block": (ctypes.c_int, [_S, _I3, _I3, _I3, ctypes.POINTER(BlockW), _P,
                                              ctypes.c_int, ctypes.c_int, _P, _P, _P, _P,
                                              ctypes.c_size_t, _P]),
            "ptdit_giim_ex": (ctypes.c_int, [_S, _I3, ctypes.c_int, _P, _W, _W, ctypes.c_uint, _P,
                                             _P, _P, ctypes.c_size_t, _P]),
            "ptdit_giim": (ctypes.c_int, [_S, _I3, _W, _W, ctypes.c_uint, _P, _P, _P,
                                          ctypes.c_size_t, _P]),
            "ptdit_window_attn": (ctypes.c_int, [_S, _I3, _I3, _W, ctypes.c_uint, _P, _P, _P,
                                                 ctypes.c_size_t, _P]),
            "ptdit_tcm": (ctypes.c_int, [_S, _I3, _I3, _W, _W, ctypes.c_uint, _P, _P, _P,
                                         ctypes.c_size_t, _P]),
            "ptdit_window_attn_bwd_workspace_bytes": (ctypes.c_size_t, [_S, _I3]),
            "ptdit_tcm_bwd_workspace_bytes": (ctypes.c_size_t, [_S, _I3]),
            "ptdit_giim_bwd_workspace_bytes": (ctypes.c_size_t, [_S, _I3]),
            "ptdit_block_attn_bwd_workspace_bytes": (ctypes.c_size_t, [_S, _I3, _I3]),
            "ptdit_block_attn_train_workspace_bytes": (ctypes.c_size_t, [_S, _I3, _I3]),
            "ptdit_block_attn_fwd_train": (ctypes.c_int, [_S, _I3, _I3, _I3, _W, _W, _W, _W,
                                                          ctypes.c_uint, _P, _P, _P,
                                                          ctypes.c_size_t, _P]),
            "ptdit_block_attn_bwd_saved": (ctypes.c_int, [_S, _I3, _I3, _I3, _W, _W, _W, _W,
                                                          ctypes.c_uint, _P, _P, _P]
                                           + [ctypes.POINTER(AttnWgrad)] * 4
                                           + [_P, ctypes.c_size_t, _P]),
            "ptdit_block_attn_bwd": (ctypes.c_int, [_S, _I3, _I3, _I3, _W, _W, _W, _W,
                                                    ctypes.c_uint, _P, _P, _P]
                                     + [ctypes.POINTER(AttnWgrad)] * 4
                                     + [_P, ctypes.c_size_t, _P]),
            "ptdit_giim_bwd": (ctypes.c_int, [_S, _I3, _W, _W, ctypes.c_uint, _P, _P, _P,
                                              ctypes.POINTER(AttnWgrad), ctypes.POINTER(AttnWgrad),
                                              _P, ctypes.c_size_t, _P]),
            "ptdit_tcm_bwd": (ctypes.c_int, [_S, _I3, _I3, _W, _W, ctypes.c_uint, _P, _P, _P,
                                             ctypes.POINTER(AttnWgrad), ctypes.POINTER(AttnWgrad),
                                             _P, ctypes.c_size_t, _P]),
            "ptdit_window_attn_bwd": (ctypes.c_int, [_S, _I3, _I3, _W, ctypes.c_uint, _P, _P, _P,
                                                     ctypes.POINTER(AttnWgrad), _P,
                                                     ctypes.c_size_t, _P]),
            "ptdit_block_attn": (ctypes.c_int, [_S, _I3, _I3, _I3, _W, _W, _W, _W, ctypes.c_uint,
                                                _P, _P, _P, ctypes.c_size_t, _P]),
            "ptdit_full_attn": (ctypes.c_int, [_S, _W, ctypes.c_uint, _P, _P, _P,
                                               ctypes.c_size_t, _P]),
            "ptdit_strerror": (ctypes.c_char_p, [ctypes.c_int]),
            "ptdit_last_error": (ctypes.c_char_p, []),
            "ptdit_debug_proxy_map": (ctypes.c_int, [_I3, _I3, _P, _P]),
            "ptdit_debug_window_map": (ctypes.c_int, [_I3, _I3, _I3, _P, _P, _P]),
            "ptdit_device_status": (ctypes.c_int, [ctypes.c_int]),
            "ptdit_debug_timeout": (ctypes.c_int, [ctypes.c_longlong, _P]),
            "ptdit_debug_wait_limit": (ctypes.c_int, [ctypes.c_longlong]),
            "ptdit_window_fused": (ctypes.c_int, [ctypes.c_int]),
            "ptdit_timing_enable": (ctypes.c_int, [ctypes.c_int]),
            "ptdit_timing_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int),
                                                 ctypes.POINTER(ctypes.c_float), ctypes.c_int]),
            "ptdit_launch_count": (ctypes.c_longlong, []),
            "ptdit_window_attn_static": (ctypes.c_int, [_S, _I3, _I3, _W, ctypes.c_uint, _P, _P,
                                                        _P]),
            "ptdit_debug_thl_map": (ctypes.c_int, [_I3, _I3, _I3, ctypes.c_int, _P, _P, _IP]),
            "ptdit_debug_thl_units": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, _IP, _IP]),
            "ptdit_debug_gemm_schedule": (ctypes.c_int, [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                                         ctypes.c_int, _P, _P, _IP, _IP]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int):
    if code != 0:
        raise PtditError(code, lib().ptdit_last_error().decode())


def _i3(v) -> Int3:
    return Int3(*[int(x) for x in v]) if v is not None else None


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return PTDIT_BF16
    if t.dtype == torch.float32:
        return PTDIT_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_shape(z, grid, heads) -> Shape:
    """Shape of a [B, N, D] latent tensor on the (f, h, w) grid."""
    B, N, D = z.shape
    f, h, w = grid
    if f * h * w != N:
        raise ValueError(f"grid {tuple(grid)} does not hold {N} tokens")
    return Shape(B, f, h, w, D, heads, _dtype_code(z))


def attn_w(ws) -> AttnW:
    """AttnW from a (Wq, Wk, Wv, Wo) tuple of [D, D] CUDA tensors."""
    for w in ws:
        if not w.is_contiguous():
            raise ValueError("weights must be contiguous")
    return AttnW(*[w.data_ptr() for w in ws])


def _check_z(z):
    if not z.is_cuda or not z.is_contiguous() or z.dim() != 3:
        raise ValueError("latents must be a contiguous [B, N, D] CUDA tensor")


def workspace_bytes(shape: Shape, ratio=None, window=None) -> int:
    return int(lib().ptdit_workspace_bytes(ctypes.byref(shape), _i3(ratio), _i3(window)))


def workspace(shape: Shape, ratio=None, window=None):
    """A caller-owned workspace tensor of ptdit_workspace_bytes() bytes."""
    import torch
    n = workspace_bytes(shape, ratio, window)
    if n == 0:
        raise PtditError(2, lib().ptdit_last_error().decode())
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def ptdit_proxy_average(z, grid, ratio, proxies=None, stream=None):
    """[B, N, D] -> [B, M, D] window means (GIIM Averaging)."""
    import torch
    _check_z(z)
    shape = make_shape(z, grid, 1)
    P = ratio[0] * ratio[1] * ratio[2]
    if proxies is None:
        proxies = torch.empty(z.shape[0], z.shape[1] // P, z.shape[2], dtype=z.dtype,
                              device=z.device)
    _check(lib().ptdit_proxy_average(ctypes.byref(shape), _i3(ratio), _ptr(z), _ptr(proxies),
                                     _stream(stream)))
    return proxies


def _slots(mode, slots, B, M):
    """Device int32 slot array for PTDIT_PROXY_RANDOM (None otherwise)."""
    if PROXY_MODES[mode] != PTDIT_PROXY_RANDOM:
        return None
    if slots is None or not slots.is_cuda or slots.dtype.is_floating_point:
        raise ValueError("mode 'random' needs a CUDA int32 slots tensor of B * M entries")
    if slots.numel() != B * M:
        raise ValueError(f"slots holds {slots.numel()} entries, expected {B * M}")
    return slots.contiguous()


def ptdit_proxy_extract(z, grid, ratio, mode="mean", slots=None, proxies=None, stream=None):
    """[B, N, D] -> [B, M, D] proxy tokens: window mean, first token or the slot-th
    member of each window (slots: CUDA int32 [B, M])."""
    import torch
    _check_z(z)
    shape = make_shape(z, grid, 1)
    P = ratio[0] * ratio[1] * ratio[2]
    M = z.shape[1] // P
    if proxies is None:
        proxies = torch.empty(z.shape[0], M, z.shape[2], dtype=z.dtype, device=z.device)
    sl = _slots(mode, slots, z.shape[0], M)
    _check(lib().ptdit_proxy_extract(ctypes.byref(shape), _i3(ratio), PROXY_MODES[mode],
                                     _ptr(sl), _ptr(z), _ptr(proxies), _stream(stream)))
    return proxies


def _prep(z_in, grid, heads, z_out, ws, ratio, window):
    import torch
    _check_z(z_in)
    shape = make_shape(z_in, grid, heads)
    if z_out is None:
        z_out = torch.empty_like(z_in)
    if ws is None:
        ws = workspace(shape, ratio, window)
    return shape, z_out, ws


def ptdit_giim(z_in, grid, ratio, psa, cross, heads, flags=0, z_out=None, ws=None,
               stream=None):
    shape, z_out, ws = _prep(z_in, grid, heads, z_out, ws, ratio, None)
    wp, wc = attn_w(psa), attn_w(cross)
    _check(lib().ptdit_giim(ctypes.byref(shape), _i3(ratio), ctypes.byref(wp), ctypes.byref(wc),
                            flags, _ptr(z_in), _ptr(z_out), _ptr(ws), ws.numel(),
                            _stream(stream)))
    return z_out


def ptdit_giim_ex(z_in, grid, ratio, mode, slots, psa, cross, heads, flags=0, z_out=None,
                  ws=None, stream=None):
    shape, z_out, ws = _prep(z_in, grid, heads, z_out, ws, ratio, None)
    P = ratio[0] * ratio[1] * ratio[2]
    sl = _slots(mode, slots, z_in.shape[0], z_in.shape[1] // P)
    wp, wc = attn_w(psa), attn_w(cross)
    _check(lib().ptdit_giim_ex(ctypes.byref(shape), _i3(ratio), PROXY_MODES[mode], _ptr(sl),
                               ctypes.byref(wp), ctypes.byref(wc), flags, _ptr(z_in), _ptr(z_out),
                               _ptr(ws), ws.numel(), _stream(stream)))
    return z_out


def block_w(attn: dict, norms: dict, mlp, eps: float = 1e-6) -> BlockW:
    """BlockW from {"psa", "cross", "wsa", "swsa", "text"} -> (Wq, Wk, Wv, Wo), {norm name}
    -> (gamma, beta) and (W1, b1, W2, b2), all contiguous CUDA tensors."""
    bw = BlockW()
    for m in ("psa", "cross", "wsa", "swsa", "text"):
        setattr(bw, m, attn_w(attn[m]))
    for k in ("proxy", "cross", "wsa", "swsa", "text", "mlp"):
        g, b = norms[k]
        setattr(bw, "norm_" + k, NormW(g.data_ptr(), b.data_ptr()))
    W1, b1, W2, b2 = mlp
    for t in (W1, b1, W2, b2):
        if not t.is_contiguous():
            raise ValueError("MLP parameters must be contiguous")
    bw.w1, bw.b1, bw.w2, bw.b2 = W1.data_ptr(), b1.data_ptr(), W2.data_ptr(), b2.data_ptr()
    bw.mlp_hidden = int(W1.shape[0])
    bw.eps = float(eps)
    return bw


def pt_block_workspace(shape: Shape, ratio, text_len: int, mlp_hidden: int):
    import torch
    n = int(lib().ptdit_pt_block_workspace_bytes(ctypes.byref(shape), _i3(ratio), int(text_len),
                                                 int(mlp_hidden)))
    if n == 0:
        raise PtditError(2, "invalid arguments for the block workspace")
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def ptdit_pt_block(z_in, grid, ratio, window, shift, attn: dict, norms: dict, mlp, text, heads,
                   eps=1e-6, mode="mean", slots=None, z_out=None, ws=None, stream=None):
    """One complete PT-Block (GIIM, TCM, text cross-attention, MLP; pre-norm residual
    sub-layers).  text: [B, L, D] CUDA tensor of text tokens at the model width."""
    import torch
    _check_z(z_in)
    shape = make_shape(z_in, grid, heads)
    if not text.is_cuda or not text.is_contiguous() or text.dim() != 3:
        raise ValueError("text must be a contiguous [B, L, D] CUDA tensor")
    bw = block_w(attn, norms, mlp, eps)
    if z_out is None:
        z_out = torch.empty_like(z_in)
    if ws is None:
        ws = pt_block_workspace(shape, ratio, text.shape[1], bw.mlp_hidden)
    P = ratio[0] * ratio[1] * ratio[2]
    sl = _slots(mode, slots, z_in.shape[0], z_in.shape[1] // P)
    _check(lib().ptdit_pt_block(ctypes.byref(shape), _i3(ratio), _i3(window), _i3(shift),
                                ctypes.byref(bw), _ptr(text), int(text.shape[1]),
                                PROXY_MODES[mode], _ptr(sl), _ptr(z_in), _ptr(z_out), _ptr(ws),
                                ws.numel(), _stream(stream)))
    return z_out


def ptdit_window_attn(z_in, grid, window, shift, w, heads, flags=0, z_out=None, ws=None,
                      stream=None):
    shape, z_out, ws = _prep(z_in, grid, heads, z_out, ws, None, window)
    ww = attn_w(w)
    _check(lib().ptdit_window_attn(ctypes.byref(shape), _i3(window), _i3(shift),
                                   ctypes.byref(ww), flags, _ptr(z_in), _ptr(z_out), _ptr(ws),
                                   ws.numel(), _stream(stream)))
    return z_out


def window_attn_bwd_workspace(shape: Shape, window):
    """A uint8 device buffer of ptdit_window_attn_bwd_workspace_bytes()."""
    import torch
    n = lib().ptdit_window_attn_bwd_workspace_bytes(ctypes.byref(shape), _i3(window))
    if n == 0:
        raise PtditError(PTDIT_ERR_SHAPE, "invalid shape or window")
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def ptdit_window_attn_bwd(z_in, dz_out, grid, window, shift, w, heads, flags=0, dz_in=None,
                          dw=None, ws=None, stream=None):
    """Backward of ptdit_window_attn: returns (dz_in, (dWq, dWk, dWv, dWo)), the weight
    gradients fp32 [D, D]."""
    import torch
    _check_z(z_in)
    _check_z(dz_out)
    shape = make_shape(z_in, grid, heads)
    if dz_in is None:
        dz_in = torch.empty_like(z_in)
    if dw is None:
        dw = tuple(torch.empty(z_in.shape[-1], z_in.shape[-1], dtype=torch.float32,
                               device=z_in.device) for _ in range(4))
    if ws is None:
        ws = window_attn_bwd_workspace(shape, window)
    ww = attn_w(w)
    g = AttnWgrad(*[_ptr(x) for x in dw])
    _check(lib().ptdit_window_attn_bwd(ctypes.byref(shape), _i3(window), _i3(shift),
                                       ctypes.byref(ww), flags, _ptr(z_in), _ptr(dz_out),
                                       _ptr(dz_in), ctypes.byref(g), _ptr(ws), ws.numel(),
                                       _stream(stream)))
    return dz_in, tuple(dw)


def ptdit_giim_bwd(z_in, dz_out, grid, ratio, psa, cross, heads, flags=0, dz_in=None, ws=None,
                   stream=None):
    """Backward of ptdit_giim (window-mean proxies): returns (dz_in, dW_psa, dW_cross), each
    dW four fp32 [D, D]."""
    import torch
    _check_z(z_in)
    _check_z(dz_out)
    shape = make_shape(z_in, grid, heads)
    if dz_in is None:
        dz_in = torch.empty_like(z_in)
    D = z_in.shape[-1]
    dwp = tuple(torch.empty(D, D, dtype=torch.float32, device=z_in.device) for _ in range(4))
    dwc = tuple(torch.empty(D, D, dtype=torch.float32, device=z_in.device) for _ in range(4))
    if ws is None:
        n = lib().ptdit_giim_bwd_workspace_bytes(ctypes.byref(shape), _i3(ratio))
        if n == 0:
            raise PtditError(PTDIT_ERR_SHAPE, "invalid shape or ratio")
        ws = torch.empty(n, dtype=torch.uint8, device=z_in.device)
    wp, wc = attn_w(psa), attn_w(cross)
    gp, gc = AttnWgrad(*[_ptr(x) for x in dwp]), AttnWgrad(*[_ptr(x) for x in dwc])
    _check(lib().ptdit_giim_bwd(ctypes.byref(shape), _i3(ratio), ctypes.byref(wp),
                                ctypes.byref(wc), flags, _ptr(z_in), _ptr(dz_out), _ptr(dz_in),
                                ctypes.byref(gp), ctypes.byref(gc), _ptr(ws), ws.numel(),
                                _stream(stream)))
    return dz_in, dwp, dwc


def ptdit_tcm_bwd(z_in, dz_out, grid, window, shift, wsa, swsa, heads, flags=0, dz_in=None,
                  ws=None, stream=None):
    """Backward of ptdit_tcm: returns (dz_in, dW_wsa, dW_swsa), each dW four fp32 [D, D]."""
    import torch
    _check_z(z_in)
    _check_z(dz_out)
    shape = make_shape(z_in, grid, heads)
    if dz_in is None:
        dz_in = torch.empty_like(z_in)
    D = z_in.shape[-1]
    dwa = tuple(torch.empty(D, D, dtype=torch.float32, device=z_in.device) for _ in range(4))
    dwb = tuple(torch.empty(D, D, dtype=torch.float32, device=z_in.device) for _ in range(4))
    if ws is None:
        n = lib().ptdit_tcm_bwd_workspace_bytes(ctypes.byref(shape), _i3(window))
        if n == 0:
            raise PtditError(PTDIT_ERR_SHAPE, "invalid shape or window")
        ws = torch.empty(n, dtype=torch.uint8, device=z_in.device)
    wa, wb = attn_w(wsa), attn_w(swsa)
    ga, gb = AttnWgrad(*[_ptr(x) for x in dwa]), AttnWgrad(*[_ptr(x) for x in dwb])
    _check(lib().ptdit_tcm_bwd(ctypes.byref(shape), _i3(window), _i3(shift), ctypes.byref(wa),
                               ctypes.byref(wb), flags, _ptr(z_in), _ptr(dz_out), _ptr(dz_in),
                               ctypes.byref(ga), ctypes.byref(gb), _ptr(ws), ws.numel(),
                               _stream(stream)))
    return dz_in, dwa, dwb


def ptdit_block_attn_bwd(z_in, dz_out, grid, ratio, window, shift, psa, cross, wsa, swsa, heads,
                         flags=0, dz_in=None, ws=None, stream=None):
    """Backward of ptdit_block_attn: returns (dz_in, dW_psa, dW_cross, dW_wsa, dW_swsa),
    each dW four fp32 [D, D]."""
    import torch
    _check_z(z_in)
    _check_z(dz_out)
    shape = make_shape(z_in, grid, heads)
    if dz_in is None:
        dz_in = torch.empty_like(z_in)
    D = z_in.shape[-1]
    dws = [tuple(torch.empty(D, D, dtype=torch.float32, device=z_in.device) for _ in range(4))
           for _ in range(4)]
    if ws is None:
        n = lib().ptdit_block_attn_bwd_workspace_bytes(ctypes.byref(shape), _i3(ratio),
                                                      _i3(window))
        if n == 0:
            raise PtditError(PTDIT_ERR_SHAPE, "invalid shape, ratio or window")
        ws = torch.empty(n, dtype=torch.uint8, device=z_in.device)
    w = [attn_w(x) for x in (psa, cross, wsa, swsa)]
    g = [AttnWgrad(*[_ptr(x) for x in dw]) for dw in dws]
    _check(lib().ptdit_block_attn_bwd(ctypes.byref(shape), _i3(ratio), _i3(window), _i3(shift),
                                      *[ctypes.byref(x) for x in w], flags, _ptr(z_in),
                                      _ptr(dz_out), _ptr(dz_in), *[ctypes.byref(x) for x in g],
                                      _ptr(ws), ws.numel(), _stream(stream)))
    return (dz_in, *dws)


def train_workspace(z_in, grid, ratio, window, heads):
    """A uint8 device buffer of ptdit_block_attn_train_workspace_bytes()."""
    import torch
    shape = make_shape(z_in, grid, heads)
    n = lib().ptdit_block_attn_train_workspace_bytes(ctypes.byref(shape), _i3(ratio), _i3(window))
    if n == 0:
        raise PtditError(PTDIT_ERR_SHAPE, "invalid shape, ratio or window")
    return torch.empty(n, dtype=torch.uint8, device=z_in.device)


def ptdit_block_attn_fwd_train(z_in, grid, ratio, window, shift, psa, cross, wsa, swsa, heads, ws,
                               flags=0, z_out=None, stream=None):
    """The block-attention forward that keeps its activations in ws (train_workspace) for
    ptdit_block_attn_bwd_saved; returns z_out."""
    import torch
    _check_z(z_in)
    shape = make_shape(z_in, grid, heads)
    if z_out is None:
        z_out = torch.empty_like(z_in)
    w = [attn_w(x) for x in (psa, cross, wsa, swsa)]
    _check(lib().ptdit_block_attn_fwd_train(ctypes.byref(shape), _i3(ratio), _i3(window),
                                            _i3(shift), *[ctypes.byref(x) for x in w], flags,
                                            _ptr(z_in), _ptr(z_out), _ptr(ws), ws.numel(),
                                            _stream(stream)))
    return z_out


def ptdit_block_attn_bwd_saved(z_in, dz_out, grid, ratio, window, shift, psa, cross, wsa, swsa,
                               heads, ws, flags=0, dz_in=None, stream=None):
    """The block-attention backward from the activations ptdit_block_attn_fwd_train kept in
    ws: returns (dz_in, dW_psa, dW_cross, dW_wsa, dW_swsa), each dW four fp32 [D, D]."""
    import torch
    _check_z(z_in)
    _check_z(dz_out)
    shape = make_shape(z_in, grid, heads)
    if dz_in is None:
        dz_in = torch.empty_like(z_in)
    D = z_in.shape[-1]
    dws = [tuple(torch.empty(D, D, dtype=torch.float32, device=z_in.device) for _ in range(4))
           for _ in range(4)]
    w = [attn_w(x) for x in (psa, cross, wsa, swsa)]
    g = [AttnWgrad(*[_ptr(x) for x in dw]) for dw in dws]
    _check(lib().ptdit_block_attn_bwd_saved(ctypes.byref(shape), _i3(ratio), _i3(window),
                                            _i3(shift), *[ctypes.byref(x) for x in w], flags,
                                            _ptr(z_in), _ptr(dz_out), _ptr(dz_in),
                                            *[ctypes.byref(x) for x in g], _ptr(ws), ws.numel(),
                                            _stream(stream)))
    return (dz_in, *dws)


def ptdit_tcm(z_in, grid, window, shift, wsa, swsa, heads, flags=0, z_out=None, ws=None,
              stream=None):
    shape, z_out, ws = _prep(z_in, grid, heads, z_out, ws, None, window)
    wa, wb = attn_w(wsa), attn_w(swsa)
    _check(lib().ptdit_tcm(ctypes.byref(shape), _i3(window), _i3(shift), ctypes.byref(wa),
                           ctypes.byref(wb), flags, _ptr(z_in), _ptr(z_out), _ptr(ws),
                           ws.numel(), _stream(stream)))
    return z_out


def ptdit_block_attn(z_in, grid, ratio, window, shift, psa, cross, wsa, swsa, heads, flags=0,
                     z_out=None, ws=None, stream=None):
    shape, z_out, ws = _prep(z_in, grid, heads, z_out, ws, ratio, window)
    w = [attn_w(x) for x in (psa, cross, wsa, swsa)]
    _check(lib().ptdit_block_attn(ctypes.byref(shape), _i3(ratio), _i3(window), _i3(shift),
                                  *[ctypes.byref(x) for x in w], flags, _ptr(z_in), _ptr(z_out),
                                  _ptr(ws), ws.numel(), _stream(stream)))
    return z_out


def ptdit_full_attn(z_in, grid, w, heads, flags=0, z_out=None, ws=None, stream=None):
    shape, z_out, ws = _prep(z_in, grid, heads, z_out, ws, None, None)
    ww = attn_w(w)
    _check(lib().ptdit_full_attn(ctypes.byref(shape), ctypes.byref(ww), flags, _ptr(z_in),
                                 _ptr(z_out), _ptr(ws), ws.numel(), _stream(stream)))
    return z_out


def ptdit_debug_proxy_map(grid, ratio, stream=None):
    import torch
    N = grid[0] * grid[1] * grid[2]
    out = torch.empty(N, dtype=torch.int32, device="cuda")
    _check(lib().ptdit_debug_proxy_map(_i3(grid), _i3(ratio), _ptr(out), _stream(stream)))
    return out


def ptdit_debug_window_map(grid, window, shift, with_mask=True, stream=None):
    import torch
    N = grid[0] * grid[1] * grid[2]
    n = window[0] * window[1] * window[2]
    tok = torch.empty(N, dtype=torch.int32, device="cuda")
    allowed = torch.empty((N // n) * n * n, dtype=torch.uint8, device="cuda") if with_mask else None
    _check(lib().ptdit_debug_window_map(_i3(grid), _i3(window), _i3(shift), _ptr(tok),
                                        _ptr(allowed), _stream(stream)))
    return tok, allowed


def ptdit_debug_thl_map(grid, window=None, shift=None):
    """Tiled head layout of one batch item (host only): (row_of_token[N],
    token_of_row[tiles * 128]) as int32 arrays, rows numbered tile * 128 + row and
    -1 for rows that hold no token.  Identity tiles without `window`; with it, the
    window tiles of the grid rolled by -shift."""
    import numpy as np
    N = grid[0] * grid[1] * grid[2]
    windowed = 1 if window is not None else 0
    w3 = _i3(window) if windowed else None
    s3 = _i3(shift if shift is not None else (0, 0, 0)) if windowed else None
    tiles = ctypes.c_int(0)
    _check(lib().ptdit_debug_thl_map(_i3(grid), w3, s3, windowed, None, None, ctypes.byref(tiles)))
    row = np.empty(N, np.int32)
    tok = np.empty(tiles.value * 128, np.int32)
    _check(lib().ptdit_debug_thl_map(_i3(grid), w3, s3, windowed, row.ctypes.data, tok.ctypes.data,
                                     ctypes.byref(tiles)))
    return row, tok


def ptdit_debug_thl_units(d: int, vpad: bool = False):
    """(offset[128, units] uint32, block_bytes): byte offset, inside one (tile, head)
    block, of the 16-byte unit p of tile row r (host only)."""
    import numpy as np
    units, block = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().ptdit_debug_thl_units(int(d), int(vpad), None, ctypes.byref(units),
                                       ctypes.byref(block)))
    off = np.empty((128, units.value), np.uint32)
    _check(lib().ptdit_debug_thl_units(int(d), int(vpad), off.ctypes.data, ctypes.byref(units),
                                       ctypes.byref(block)))
    return off, block.value


def ptdit_debug_gemm_schedule(rows: int, nseg: int, nmat: int, pairs: int):
    """Tile order of the 2-SM projection GEMM (host only): (tiles, None) when the
    launch runs round robin, else (tiles, per-pair lists of tile indices)."""
    import numpy as np
    tiles, sched = ctypes.c_int(0), ctypes.c_int(0)
    args = (int(rows), int(nseg), int(nmat), int(pairs))
    _check(lib().ptdit_debug_gemm_schedule(*args, None, None, ctypes.byref(tiles),
                                           ctypes.byref(sched)))
    if not sched.value:
        return tiles.value, None
    first = np.empty(pairs + 1, np.int32)
    tile = np.empty(tiles.value, np.int32)
    _check(lib().ptdit_debug_gemm_schedule(*args, first.ctypes.data, tile.ctypes.data,
                                           ctypes.byref(tiles), ctypes.byref(sched)))
    return tiles.value, [tile[first[q]:first[q + 1]].tolist() for q in range(pairs)]


def ptdit_device_status(reset: bool = False) -> int:
    """The device status word (0, or PTDIT_ERR_TIMEOUT after a bounded wait gave up);
    synchronises the device; reset clears it."""
    v = int(lib().ptdit_device_status(1 if reset else 0))
    if v == PTDIT_ERR_CUDA:
        raise PtditError(v, lib().ptdit_last_error().decode())
    return v


def ptdit_debug_timeout(limit_ns: int, stream=None):
    """Launch one bounded wait that nothing releases (gives up after limit_ns)."""
    _check(lib().ptdit_debug_timeout(int(limit_ns), _stream(stream)))


def ptdit_debug_wait_limit(limit_ns: int):
    """Limit of the window kernel's waits for work on this thread (0: the default 2 s)."""
    _check(lib().ptdit_debug_wait_limit(int(limit_ns)))


def ptdit_timing_enable(max_launches: int):
    _check(lib().ptdit_timing_enable(int(max_launches)))


def ptdit_timing_read(max_records: int = 4096):
    """[(kind name, milliseconds)] of the launches recorded since the last read."""
    kinds = (ctypes.c_int * max_records)()
    ms = (ctypes.c_float * max_records)()
    n = lib().ptdit_timing_read(kinds, ms, max_records)
    if n < 0:
        raise PtditError(5, lib().ptdit_last_error().decode())
    return [(KINDS[kinds[i]], ms[i]) for i in range(n)]


def ptdit_launch_count() -> int:
    return int(lib().ptdit_launch_count())
