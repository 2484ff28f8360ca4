/*
 * ptdit.h -- PT-DiT block attention (GIIM + TCM) for NVIDIA B200 (sm_100a).
 *
 * The operation is the attention half of a PT-Block of the Proxy-Tokenized
 * Diffusion Transformer, as stated in "Qihoo-T2X -- Proxy-Tokenized DiT for
 * Text-to-Any-Task", §3 Method:
 *
 *   GIIM (Eq. GIIM)  z_s <- z_s + CS(z_s, SA(Averaging(z_s)))
 *       Averaging: the mean of z_s over each p_f x p_h x p_w window gives the
 *       proxy tokens P_a; SA: multi-head self-attention among the proxies;
 *       CS: multi-head cross-attention, every latent token the query, the
 *       proxies keys and values.
 *   TCM  (Eq. TCM)   z^ = WSA(z_s) + z_s ;  z_w = SWSA(z^) + z^
 *       WSA: self-attention inside non-overlapping windows; SWSA: the same
 *       after a Swin-style cyclic roll of the grid by -s, with the pairs that
 *       the roll wrapped masked out, followed by the roll back by +s.
 *
 * Conventions shared by every entry point
 *   - Latents are [B, N, D], contiguous, N = F*H*W flattened row-major over
 *     the (f, h, w) token grid (t slowest, x fastest).  Proxies are [B, M, D],
 *     M = N / (p_f p_h p_w), numbered row-major over the grid of windows.
 *   - A module's weights are four [D][D] row-major matrices, applied as
 *     y = x W^T (PyTorch Linear layout), with no bias.  Head h owns columns
 *     h*d .. h*d+d-1 of Q, K, V, d = D / heads.  The softmax scale is
 *     1/sqrt(d).  The zero-initialised linear after the cross-attention of
 *     the official code is folded into the cross-attention's W_o.
 *   - dtype PTDIT_BF16: bf16 storage, bf16 tensor-core inputs, fp32
 *     accumulation and softmax.  dtype PTDIT_F32: fp32 storage and fp32 FMA
 *     arithmetic throughout (no TF32).
 *   - Every data pointer is a DEVICE pointer owned by the caller; the
 *     library never allocates device memory and keeps no pointer after the
 *     call returns.  Pointers must be 16-byte aligned.  z_out must not
 *     overlap z_in, the weights or the workspace.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream).  Arguments are validated on the host first; on any error
 *     nothing is launched and a PTDIT_ERR_* code is returned.
 *     ptdit_last_error() gives a one-line description (per host thread).
 *   - Every grid extent must be divisible by its proxy ratio and by its TCM
 *     window, and 0 <= shift < window on every axis (else PTDIT_ERR_SHAPE).
 */
#ifndef PTDIT_H
#define PTDIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *ptdit_stream_t; /* a cudaStream_t */

enum { PTDIT_F32 = 0, PTDIT_BF16 = 1 };

typedef struct {
    int B;          /* batch items (independent) */
    int F, H, W;    /* token grid f x h x w; N = F*H*W */
    int D;          /* model width */
    int heads;      /* attention heads; d = D / heads */
    int dtype;      /* PTDIT_F32 or PTDIT_BF16 */
} ptdit_shape;

/* One attention module's projections: Q = x Wq^T, K = x Wk^T, V = x Wv^T,
 * out = A Wo^T, each W a [D][D] row-major device array of the call's dtype. */
typedef struct {
    const void *wq, *wk, *wv, *wo;
} ptdit_attn_w;

/* Status codes. */
#define PTDIT_OK            0
#define PTDIT_ERR_NULL      1  /* a required pointer is NULL */
#define PTDIT_ERR_SHAPE     2  /* sizes, ratios, windows or shifts are invalid */
#define PTDIT_ERR_DTYPE     3  /* unknown dtype */
#define PTDIT_ERR_WORKSPACE 4  /* workspace smaller than ptdit_workspace_bytes() */
#define PTDIT_ERR_CUDA      5  /* a CUDA call or launch failed */
#define PTDIT_ERR_TIMEOUT   6  /* a bounded device-side wait gave up */
#define PTDIT_ERR_ALIGN     7  /* a pointer is not 16-byte aligned */
#define PTDIT_ERR_ALIAS     8  /* z_out overlaps an input or the workspace */

/* Flags. */
#define PTDIT_PROXY_RESIDUAL 0x1u /* proxy SA adds its input: P' = SA(P_a) + P_a
                                     (the official code listing); default P' = SA(P_a) (Eq. GIIM) */
#define PTDIT_NO_RESIDUAL    0x2u /* drop every residual add on the latent stream:
                                     each module returns only its attention branch */

/*
 * ptdit_proxy_average -- GIIM "Averaging" (Eq. GIIM; get_proxy_token mode "mean").
 *   proxies[b, m, :] = mean of z[b, t, :] over the tokens t of window m.
 *   ratio = {p_f, p_h, p_w}.  z: [B, N, D] (in), proxies: [B, M, D] (out).
 *   Sums in fp32 in a fixed order (bitwise deterministic), one rounding.
 */
int ptdit_proxy_average(const ptdit_shape *shape, const int ratio[3], const void *z,
                        void *proxies, ptdit_stream_t stream);

/*
 * Proxy extraction modes (Qihoo-T2X reading note, code-comparison section,
 * get_proxy_token(mode=...), and the proxy-extraction ablation of §3 Method:
 * Average / Top-Left / Random).
 *   PTDIT_PROXY_MEAN    the window mean (Eq. GIIM; the method's choice)
 *   PTDIT_PROXY_FIRST   the window's first token in (t, y, x) order: its
 *                       top-left token in its first frame
 *   PTDIT_PROXY_RANDOM  the window member the caller's slots array names:
 *                       slots is a DEVICE int32 array [B * M] (batch item
 *                       major), slots[b*M + m] in [0, p_f p_h p_w) counting
 *                       the window's members row-major over (t, y, x).  The
 *                       random draw is the caller's; a slot outside the range
 *                       leaves that proxy zero and records PTDIT_ERR_SHAPE in
 *                       the device status word (ptdit_device_status).
 */
#define PTDIT_PROXY_MEAN   0
#define PTDIT_PROXY_FIRST  1
#define PTDIT_PROXY_RANDOM 2

/*
 * ptdit_proxy_extract -- the proxy tokens under any of the three modes.
 *   mode PTDIT_PROXY_MEAN is ptdit_proxy_average.  Single-token modes copy
 *   their token bit for bit.  slots: see PTDIT_PROXY_RANDOM (NULL otherwise;
 *   ignored).  Errors as ptdit_proxy_average, plus PTDIT_ERR_SHAPE for an
 *   unknown mode and PTDIT_ERR_NULL for RANDOM without slots.
 */
int ptdit_proxy_extract(const ptdit_shape *shape, const int ratio[3], int mode,
                        const int32_t *slots, const void *z, void *proxies,
                        ptdit_stream_t stream);

/*
 * ptdit_workspace_bytes -- device scratch that every call below needs for
 * this shape (the maximum over them), or 0 for an invalid shape.  The
 * workspace must be 256-byte aligned; its contents need no initialisation
 * and are garbage after a call.  For a window of 128 tokens in bf16 the size
 * includes the heads' repacked Q/K/V weight rows (3 d rounded up to 16 rows of
 * D per head) that the fused projection + window-attention kernel reads
 * (ptdit_window_fused); a smaller workspace that holds everything else is
 * accepted and runs the two-kernel form.
 */
size_t ptdit_workspace_bytes(const ptdit_shape *shape, const int ratio[3], const int window[3]);

/*
 * ptdit_giim -- Eq. GIIM: z_out = z_in + CS(z_in, SA(Averaging(z_in))).
 *   psa:   the proxy self-attention's weights; cross: the cross-attention's.
 *   flags: PTDIT_PROXY_RESIDUAL, PTDIT_NO_RESIDUAL (z_out = CS(...) only).
 */
int ptdit_giim(const ptdit_shape *shape, const int ratio[3], const ptdit_attn_w *psa,
               const ptdit_attn_w *cross, unsigned flags, const void *z_in, void *z_out,
               void *ws, size_t ws_bytes, ptdit_stream_t stream);

/*
 * ptdit_giim_ex -- ptdit_giim with the proxy tokens extracted by `mode`
 *   (and `slots`, for PTDIT_PROXY_RANDOM) instead of the window mean.
 */
int ptdit_giim_ex(const ptdit_shape *shape, const int ratio[3], int mode, const int32_t *slots,
                  const ptdit_attn_w *psa, const ptdit_attn_w *cross, unsigned flags,
                  const void *z_in, void *z_out, void *ws, size_t ws_bytes,
                  ptdit_stream_t stream);

/*
 * ptdit_window_attn -- one TCM branch (Eq. TCM): z_out = z_in + WSA(z_in)
 *   for shift {0,0,0}, else SWSA: Swin-style roll by -shift, attention
 *   inside each window of window[] tokens with wrapped pairs masked out,
 *   roll back.  flags: PTDIT_NO_RESIDUAL.
 */
int ptdit_window_attn(const ptdit_shape *shape, const int window[3], const int shift[3],
                      const ptdit_attn_w *w, unsigned flags, const void *z_in, void *z_out,
                      void *ws, size_t ws_bytes, ptdit_stream_t stream);

/*
 * ptdit_window_attn_static -- ptdit_window_attn without a workspace argument,
 *   for callers that cannot allocate device memory: code that runs where
 *   cudaMalloc is not allowed or must not be called (it can synchronise the
 *   device), or that only receives input and output buffers from a host
 *   framework whose allocator it cannot reach.  The paper has no counterpart;
 *   this is a packaging of the same computation.
 *   Scratch is a static device array of PTDIT_STATIC_SCRATCH_BYTES inside the
 *   library (enough for one 64x64-token grid at D = 1152 in bf16); every GPU
 *   that loads the library's device code holds it until the process exits.  The caller still
 *   passes z_in and z_out.  A shape whose workspace (ptdit_workspace_bytes
 *   with ratio NULL) exceeds the maximum returns PTDIT_ERR_WORKSPACE and
 *   launches nothing.  Nothing is allocated: no cudaMalloc, no cudaFree.
 *   The first call on a device looks up the array's device address with
 *   cudaGetSymbolAddress (and may load the library's device code), so make
 *   it before any stream capture.  All calls share the one array: calls that
 *   overlap on the GPU (unordered streams or host threads) race.
 */
#define PTDIT_STATIC_SCRATCH_BYTES (48u << 20)
int ptdit_window_attn_static(const ptdit_shape *shape, const int window[3], const int shift[3],
                             const ptdit_attn_w *w, unsigned flags, const void *z_in,
                             void *z_out, ptdit_stream_t stream);

/*
 * ptdit_window_attn_bwd -- backward (training) of ptdit_window_attn: given the
 *   branch input z_in and dz_out = dL/dz_out, writes dz_in = dL/dz_in and the
 *   four weight gradients dL/dWq, dL/dWk, dL/dWv, dL/dWo.  With
 *   PTDIT_NO_RESIDUAL the branch had no residual (dz_in then omits dz_out).
 *   The branch is recomputed from z_in (Q, K, V and the attention output);
 *   per window and head the chain rule is the standard one for softmax
 *   attention: dV = P^T dA, dP = dA V^T, dS = P * (dP - rowsum(P * dP)),
 *   dQ = c dS K, dK = c dS^T Q (c = 1/sqrt(d), dA = dz_out Wo), then
 *   dz_in = (dz_out +) roll back of [dQ dK dV] [Wq; Wk; Wv] and
 *   dW = (gradient)^T (input) summed over all B N tokens.
 *   Arguments: z_in, dz_out [B, N, D] bf16; dz_in [B, N, D] bf16 (must not
 *   overlap any other argument); dw: four fp32 [D][D] row-major arrays in
 *   the weights' [out][in] layout, overwritten (zeroed on `stream`, then the
 *   token slices' contributions are added with atomic vector reductions, so
 *   the summation order varies from run to run at fp32 rounding level).
 *   Workspace: ptdit_window_attn_bwd_workspace_bytes(shape, window) bytes,
 *   256-byte aligned, contents garbage after the call.
 *   Supported: dtype PTDIT_BF16 only, D a multiple of 128, head widths 8..80
 *   in steps of 8, windows of 16, 32, 64 or 128 tokens; anything else returns
 *   PTDIT_ERR_SHAPE (PTDIT_ERR_DTYPE for PTDIT_F32) and launches nothing.
 */
typedef struct {
    float *dwq, *dwk, *dwv, *dwo;
} ptdit_attn_wgrad;
size_t ptdit_window_attn_bwd_workspace_bytes(const ptdit_shape *shape, const int window[3]);
int ptdit_window_attn_bwd(const ptdit_shape *shape, const int window[3], const int shift[3],
                          const ptdit_attn_w *w, unsigned flags, const void *z_in,
                          const void *dz_out, void *dz_in, const ptdit_attn_wgrad *dw, void *ws,
                          size_t ws_bytes, ptdit_stream_t stream);

/*
 * ptdit_giim_bwd -- backward (training) of ptdit_giim with window-mean proxies:
 *   given z_in and dz_out = dL/dz_out, writes dz_in = dL/dz_in and both modules'
 *   weight gradients (fp32 [D][D], overwritten).  The forward is recomputed
 *   (keeping each query row's log-sum-exp); per head the attention backward is
 *   the softmax chain rule with delta = rowsum(dO * O); dK and dV of each
 *   128-key tile are summed over all queries, dQ over the key tiles through a
 *   projection over the stacked weights; the averaging's adjoint hands every
 *   token dP_a[window] / P.  flags: PTDIT_PROXY_RESIDUAL, PTDIT_NO_RESIDUAL.
 *   Workspace: ptdit_giim_bwd_workspace_bytes(shape, ratio).  Supported: bf16,
 *   D a multiple of 128, head widths 8..80 in steps of 8, at most 8192
 *   proxies; else PTDIT_ERR_SHAPE / PTDIT_ERR_DTYPE, nothing launched.
 */
size_t ptdit_giim_bwd_workspace_bytes(const ptdit_shape *shape, const int ratio[3]);
int ptdit_giim_bwd(const ptdit_shape *shape, const int ratio[3], const ptdit_attn_w *psa,
                   const ptdit_attn_w *cross, unsigned flags, const void *z_in,
                   const void *dz_out, void *dz_in, const ptdit_attn_wgrad *dw_psa,
                   const ptdit_attn_wgrad *dw_cross, void *ws, size_t ws_bytes,
                   ptdit_stream_t stream);

/*
 * ptdit_tcm_bwd -- backward of ptdit_tcm: z^ = WSA(z_in) (+ z_in) is recomputed
 *   (WSA's Q, K, V and attention output kept in the workspace), then the SWSA
 *   branch's backward at z^ and the WSA branch's backward at z_in (each as
 *   ptdit_window_attn_bwd; WSA's reuses the kept forward).  dw_wsa and dw_swsa receive the two
 *   modules' weight gradients (fp32, overwritten).  Workspace:
 *   ptdit_tcm_bwd_workspace_bytes(shape, window).  Restrictions and errors as
 *   ptdit_window_attn_bwd.
 */
size_t ptdit_tcm_bwd_workspace_bytes(const ptdit_shape *shape, const int window[3]);
int ptdit_tcm_bwd(const ptdit_shape *shape, const int window[3], const int shift[3],
                  const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
                  const void *z_in, const void *dz_out, void *dz_in,
                  const ptdit_attn_wgrad *dw_wsa, const ptdit_attn_wgrad *dw_swsa, void *ws,
                  size_t ws_bytes, ptdit_stream_t stream);

/*
 * ptdit_block_attn_bwd -- backward (training) of ptdit_block_attn: GIIM's forward
 *   is recomputed once (z1 = GIIM(z_in) and what GIIM's backward reads), then
 *   ptdit_tcm_bwd's steps at z1 give dL/dz1 and the WSA and SWSA weight
 *   gradients, then GIIM's backward with dL/dz1 gives dz_in and the proxy and
 *   cross modules' weight gradients (Qihoo-T2X reading note, §3 Method, Eq. GIIM
 *   and Eq. TCM: the chain rule through the block's forward order).  The 16 weight
 *   gradients (fp32 [D][D], overwritten) must not overlap one another or any
 *   other argument.  Workspace: ptdit_block_attn_bwd_workspace_bytes(shape,
 *   ratio, window): z1, dL/dz1, ptdit_giim_bwd's workspace and ptdit_tcm_bwd's.
 *   Restrictions and errors: those of ptdit_giim_bwd and ptdit_tcm_bwd together.
 */
size_t ptdit_block_attn_bwd_workspace_bytes(const ptdit_shape *shape, const int ratio[3],
                                            const int window[3]);
int ptdit_block_attn_bwd(const ptdit_shape *shape, const int ratio[3], const int window[3],
                         const int shift[3], const ptdit_attn_w *psa, const ptdit_attn_w *cross,
                         const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
                         const void *z_in, const void *dz_out, void *dz_in,
                         const ptdit_attn_wgrad *dw_psa, const ptdit_attn_wgrad *dw_cross,
                         const ptdit_attn_wgrad *dw_wsa, const ptdit_attn_wgrad *dw_swsa, void *ws,
                         size_t ws_bytes, ptdit_stream_t stream);

/*
 * The training pair: ptdit_block_attn_fwd_train runs the block-attention path's
 *   forward (z_out as ptdit_block_attn, up to rounding order) and keeps what the
 *   backward reads in the workspace (GIIM's intermediates with each query row's
 *   log-sum-exp, z1, z^, both window branches' Q, K, V window tiles and attention
 *   outputs); ptdit_block_attn_bwd_saved then computes what ptdit_block_attn_bwd
 *   computes without recomputing the forward.  The second call must get the same
 *   shape, ratio, window, shift, weights, flags, z_in and workspace, with nothing
 *   written to the workspace in between.  Workspace:
 *   ptdit_block_attn_train_workspace_bytes(shape, ratio, window).  Restrictions
 *   and errors: those of ptdit_block_attn_bwd (fwd_train checks z_out as
 *   ptdit_block_attn does).
 */
size_t ptdit_block_attn_train_workspace_bytes(const ptdit_shape *shape, const int ratio[3],
                                              const int window[3]);
int ptdit_block_attn_fwd_train(const ptdit_shape *shape, const int ratio[3], const int window[3],
                               const int shift[3], const ptdit_attn_w *psa,
                               const ptdit_attn_w *cross, const ptdit_attn_w *wsa,
                               const ptdit_attn_w *swsa, unsigned flags, const void *z_in,
                               void *z_out, void *ws, size_t ws_bytes, ptdit_stream_t stream);
int ptdit_block_attn_bwd_saved(const ptdit_shape *shape, const int ratio[3], const int window[3],
                               const int shift[3], const ptdit_attn_w *psa,
                               const ptdit_attn_w *cross, const ptdit_attn_w *wsa,
                               const ptdit_attn_w *swsa, unsigned flags, const void *z_in,
                               const void *dz_out, void *dz_in, const ptdit_attn_wgrad *dw_psa,
                               const ptdit_attn_wgrad *dw_cross, const ptdit_attn_wgrad *dw_wsa,
                               const ptdit_attn_wgrad *dw_swsa, void *ws, size_t ws_bytes,
                               ptdit_stream_t stream);

/*
 * ptdit_tcm -- Eq. TCM: WSA with weights wsa, then SWSA with weights swsa
 *   and the given shift, each with its residual (unless PTDIT_NO_RESIDUAL).
 */
int ptdit_tcm(const ptdit_shape *shape, const int window[3], const int shift[3],
              const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
              const void *z_in, void *z_out, void *ws, size_t ws_bytes, ptdit_stream_t stream);

/*
 * ptdit_block_attn -- the PT-Block attention path: GIIM then TCM, in the
 *   order the block's forward pass runs them (Qihoo-T2X reading note, §3
 *   Method, Eq. GIIM and Eq. TCM).
 */
int ptdit_block_attn(const ptdit_shape *shape, const int ratio[3], const int window[3],
                     const int shift[3], const ptdit_attn_w *psa, const ptdit_attn_w *cross,
                     const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
                     const void *z_in, void *z_out, void *ws, size_t ws_bytes,
                     ptdit_stream_t stream);

/*
 * The complete PT-Block (Qihoo-T2X reading note, §3 Method: "PT-Block (GIIM +
 * TCM + text cross-attn + MLP)" and the block diagram; code-comparison
 * section, ProxyTokensTransformerBlock.forward).  Every sub-layer is pre-norm
 * with a residual (the pages name the sub-layers and their order; the norm
 * form, the MLP's activation and the position of each norm are this library's
 * reading, stated here):
 *   P_a = proxies of z (proxy_mode)      P' = P_a + SA(LN_proxy(P_a))
 *   z1 = z  + CS(LN_cross(z), P')        z2 = z1 + WSA(LN_wsa(z1))
 *   z3 = z2 + SWSA(LN_swsa(z2))          z4 = z3 + MHA(LN_text(z3), text)
 *   z_out = z4 + fc2(GELU(fc1(LN_mlp(z4))))
 * LN(x) = (x - mean) / sqrt(var + eps) * gamma + beta over the D channels of
 * a token (var: mean squared deviation); GELU in its tanh form; fc1 = x W1^T
 * + b1 (W1 [mlp_hidden][D]), fc2 = h W2^T + b2 (W2 [D][mlp_hidden]).  The
 * attention projections have no bias.  The text tokens are [B, text_len, D]
 * (already projected to the model width), keys and values of the text
 * cross-attention.  All parameters are DEVICE arrays of the call's dtype,
 * 16-byte aligned.
 */
typedef struct {
    const void *gamma, *beta;  /* [D] each */
} ptdit_norm_w;

typedef struct {
    ptdit_attn_w psa, cross, wsa, swsa, text;
    ptdit_norm_w norm_proxy, norm_cross, norm_wsa, norm_swsa, norm_text, norm_mlp;
    const void *w1, *b1;  /* [mlp_hidden][D], [mlp_hidden] */
    const void *w2, *b2;  /* [D][mlp_hidden], [D] */
    int mlp_hidden;       /* width of the MLP's hidden layer (4 D in DiT-style blocks) */
    float eps;            /* LayerNorm epsilon, in (0, 1] (1e-6 in DiT-style blocks) */
} ptdit_block_w;

/*
 * ptdit_pt_block_workspace_bytes -- workspace of ptdit_pt_block for this
 *   shape, ratio, text length and MLP width (0 for invalid arguments).
 */
size_t ptdit_pt_block_workspace_bytes(const ptdit_shape *shape, const int ratio[3],
                                      int text_len, int mlp_hidden);

/*
 * ptdit_pt_block -- one complete PT-Block (above).  proxy_mode / slots as in
 *   ptdit_giim_ex (PTDIT_PROXY_MEAN is the method).  z_out must not overlap
 *   z_in, any parameter, the text tokens or the workspace.  Errors as
 *   ptdit_block_attn, plus PTDIT_ERR_SHAPE for text_len < 1, mlp_hidden < 1
 *   or eps outside (0, 1].
 */
int ptdit_pt_block(const ptdit_shape *shape, const int ratio[3], const int window[3],
                   const int shift[3], const ptdit_block_w *w, const void *text, int text_len,
                   int proxy_mode, const int32_t *slots, const void *z_in, void *z_out, void *ws,
                   size_t ws_bytes, ptdit_stream_t stream);

/*
 * ptdit_full_attn -- the dense comparator the pages measure against
 *   (§3 complexity: full self-attention, 2 N^2 D): z_out = z_in + MHA(z_in)
 *   over all N tokens of each batch item.  Needs ptdit_workspace_bytes().
 */
int ptdit_full_attn(const ptdit_shape *shape, const ptdit_attn_w *w, unsigned flags,
                    const void *z_in, void *z_out, void *ws, size_t ws_bytes,
                    ptdit_stream_t stream);

/* ptdit_strerror -- static text for a status code. */
const char *ptdit_strerror(int status);

/* ptdit_last_error -- description of this host thread's last failed call. */
const char *ptdit_last_error(void);

/*
 * Debug index maps, computed on the device by the same address functions the
 * kernels use (for bit-exact comparison with an independent derivation).
 *   ptdit_debug_proxy_map: proxy_of_token[N] (device int32).
 *   ptdit_debug_window_map: token_at_slot[nW * n] (device int32), the
 *     original token index at each (window, slot) of the rolled grid, windows
 *     and slots row-major; allowed[nW * n * n] (device uint8, may be NULL),
 *     1 where slot i may attend slot j of the same window.
 */
int ptdit_debug_proxy_map(const int grid[3], const int ratio[3], int32_t *proxy_of_token,
                          ptdit_stream_t stream);
int ptdit_debug_window_map(const int grid[3], const int window[3], const int shift[3],
                           int32_t *token_at_slot, uint8_t *allowed, ptdit_stream_t stream);

/*
 * Host-only views of the data layout and the projection schedule, computed by
 * the same host functions the launches use (no GPU, no CUDA call; for tests).
 * All arrays are host memory owned by the caller; a NULL array skips that
 * output, so a first call with NULL arrays returns the sizes.  Errors:
 * PTDIT_ERR_NULL for a NULL count pointer, PTDIT_ERR_SHAPE for arguments no
 * launch takes; nothing is written then.
 *
 *   ptdit_debug_thl_map -- the tiled head layout (THL) of the Q, K and V
 *     operands of one batch item of the grid: one block per (128-row tile,
 *     head), each the shared-memory tile the attention kernels read.
 *     windowed = 0: identity tiles (tile t holds tokens 128 t .. 128 t + 127,
 *     the layout of the proxy self-attention and cross-attention operands);
 *     windowed = 1: window tiles of the grid rolled by -shift (window and shift
 *     as in ptdit_window_attn; the window size must divide 128): 128 / n
 *     windows per tile in window order, slots row-major inside a window.
 *     Writes *tiles, row_of_token[N] = tile * 128 + row, and
 *     token_of_row[*tiles * 128] = the token held by each tile row, or -1.
 *   ptdit_debug_thl_units -- byte offset, inside one (tile, head) block of
 *     head width d (8 .. 80, a multiple of 8; vpad: the V operand of the row
 *     kernel, columns padded to 128), of the 16-byte unit p (head columns
 *     8 p .. 8 p + 7) of tile row r: offset[r * units + p] for r < 128 and
 *     p < units.  Writes *units and *block_bytes.
 *   ptdit_debug_gemm_schedule -- the order in which the 2-SM projection GEMM
 *     (256 x 256 output tiles; a matrix's last tile narrower when nseg is not a
 *     multiple of 256) hands its rows x nseg outputs of nmat matrices to
 *     `pairs` CTA pairs.  Writes *tiles and *scheduled: 1 when the launch runs
 *     a longest-processing-time schedule, pair q taking tile[first[q]] ..
 *     tile[first[q + 1] - 1] (first[pairs + 1], tile[*tiles]); 0 when it runs
 *     round robin (tile t on pair t mod pairs; first and tile untouched).
 *     Tile t covers row block t / (nmat * n_tiles), matrix (t / n_tiles) mod
 *     nmat and column block t mod n_tiles, n_tiles = ceil(nseg / 256).
 */
int ptdit_debug_thl_map(const int grid[3], const int window[3], const int shift[3], int windowed,
                        int32_t *row_of_token, int32_t *token_of_row, int *tiles);
int ptdit_debug_thl_units(int d, int vpad, uint32_t *offset, int *units, int *block_bytes);
int ptdit_debug_gemm_schedule(long rows, int nseg, int nmat, int pairs, int32_t *first,
                              int32_t *tile, int *tiles, int *scheduled);


/*
 * Kernel timing for measurement.  ptdit_timing_enable(n) makes the calling
 * host thread's later calls record a CUDA event pair around each kernel
 * launch on the launching stream, up to n launches (0 turns it off and
 * frees the events).  ptdit_timing_read() synchronises on the recorded
 * events, writes up to `max` (kind, milliseconds) pairs and clears the list;
 * it returns the count, or -1 on error.  Kinds are PTDIT_K_*.
 */
enum {
    PTDIT_K_AVERAGE = 0,   /* window averaging */
    PTDIT_K_GEMM = 1,      /* QKV / O projections */
    PTDIT_K_ATTN_PROXY = 2,/* proxy self-attention core */
    PTDIT_K_ATTN_CROSS = 3,/* latent -> proxy cross-attention core */
    PTDIT_K_ATTN_WINDOW = 4,/* window / shifted-window attention core */
    PTDIT_K_ATTN_DENSE = 5,/* full self-attention core */
    PTDIT_K_NORM = 6,      /* LayerNorm of the complete block */
    PTDIT_K_ATTN_TEXT = 7, /* text cross-attention core of the complete block */
    PTDIT_K_ATTN_WINDOW_BWD = 8, /* window attention core, backward */
    PTDIT_K_WGRAD = 9,     /* weight gradients of the projections */
    PTDIT_K_TRANSPOSE = 10,/* weight transposes of the backward */
    PTDIT_K_ATTN_ROWS_BWD = 11, /* cross / proxy attention core, backward */
    PTDIT_K_ATTN_WINDOW_FUSED = 12, /* window Q/K/V projection + window attention, fused */
    PTDIT_K_COUNT = 13
};
int ptdit_timing_enable(int max_launches);
int ptdit_timing_read(int *kind, float *ms, int max);

/* ptdit_launch_count -- kernels this host thread has launched through the library. */
long long ptdit_launch_count(void);

/*
 * ptdit_device_status -- the library's device status word on the current
 *   device: PTDIT_OK, or PTDIT_ERR_TIMEOUT once a bounded device-side wait
 *   (2 s in the kernels) has given up since the last reset; such a kernel
 *   stops issuing work and returns instead of hanging, so its outputs are
 *   incomplete.  Synchronises the device.  reset != 0 clears the word after
 *   reading it.  Returns the word, or PTDIT_ERR_CUDA if it cannot be read.
 */
int ptdit_device_status(int reset);

/*
 * ptdit_debug_timeout -- launches one thread whose bounded wait, on a barrier
 *   nothing arrives on, gives up after limit_ns nanoseconds and records
 *   PTDIT_ERR_TIMEOUT in the device status word, exactly as a stalled kernel
 *   would (no trap, no fault; the context stays usable).  The paper has no
 *   counterpart: it lets tests exercise the timeout path.  Asynchronous on
 *   `stream`.  Errors: PTDIT_ERR_SHAPE (limit_ns <= 0 or above 10 s),
 *   PTDIT_ERR_CUDA.
 */
int ptdit_debug_timeout(long long limit_ns, ptdit_stream_t stream);

/*
 * ptdit_window_fused -- selects, for this host thread's later calls, how a TCM
 *   branch with windows of 128 tokens runs in bf16 (Qihoo-T2X reading note, §3
 *   Method, Eq. TCM): enable = 1 takes one kernel per branch for the window Q/K/V
 *   projection and the window attention (Q, K and V stay on chip; the heads'
 *   weight rows are repacked into the workspace first), 0 (the default) the
 *   projection kernel then the window-attention kernel (Q, K and V through the
 *   workspace), which is the faster form on B200: the fused kernel streams a
 *   head's weight rows for every window.  Both give the same result up to
 *   rounding order.  Other window
 *   sizes, fp32, and the forward that ptdit_tcm_bwd recomputes (whose Q, K and V
 *   its backward reuses) always take the second form.  Any other value of enable
 *   only reads the setting.  Returns the previous setting (0 or 1).
 */
int ptdit_window_fused(int enable);

/*
 * ptdit_debug_wait_limit -- sets, for this host thread's later launches of
 *   the window-attention kernel (ptdit_window_attn, ptdit_tcm,
 *   ptdit_block_attn and ptdit_window_attn_static), the limit of every
 *   device-side wait for work to limit_ns nanoseconds; 0 restores the default
 *   (2 s).  A limit shorter than the work makes those waits give up: the
 *   kernel records PTDIT_ERR_TIMEOUT in the device status word, waits (2 s at
 *   most) for the tensor-core work it issued, and returns with its output
 *   incomplete; the context stays usable.  The paper has no counterpart: it
 *   lets tests exercise the give-up path of a real kernel.  Errors:
 *   PTDIT_ERR_SHAPE (limit_ns < 0 or above 10 s).
 */
int ptdit_debug_wait_limit(long long limit_ns);

/*
 * Host-side fault injection for tests: with the environment variable
 * PTDIT_FAULT set to "workspace", every call that takes a workspace reports
 * PTDIT_ERR_WORKSPACE; set to "launch", every kernel launch is refused with
 * PTDIT_ERR_CUDA before anything reaches the device.  Read on each call.
 */

#ifdef __cplusplus
}
#endif

#endif /* PTDIT_H */
