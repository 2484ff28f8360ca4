// Shared device helpers of the PT-DiT kernels: index maps of the token grid,
// element conversions and the internal launcher interfaces.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace ptdit {

// ---------------------------------------------------------------------------
// Division by a runtime-invariant divisor d >= 1, for numerators below 2^31:
// q = umulhi(2n, m) >> s with s = ceil(log2 d) and m = ceil(2^(31+s) / d)
// (Granlund & Montgomery, "Division by Invariant Integers using
// Multiplication", PLDI 1994).  The index maps divide by grid and window
// extents on every row address, so this replaces ~20-instruction divides.
// ---------------------------------------------------------------------------
struct FastDiv {
    uint32_t d, m, s;
};

inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t s = 0;
    while ((1ull << s) < d) ++s;
    const uint64_t m = ((1ull << (31 + s)) + d - 1) / d;
    return FastDiv{d, static_cast<uint32_t>(m), s};
}

__host__ __device__ __forceinline__ uint32_t fdiv(const FastDiv &f, uint32_t n) {
#ifdef __CUDA_ARCH__
    return __umulhi(n << 1, f.m) >> f.s;
#else
    return static_cast<uint32_t>((static_cast<uint64_t>(n << 1) * f.m) >> 32) >> f.s;
#endif
}

// ---------------------------------------------------------------------------
// Token grid and index maps
//
// Tokens are flattened row-major over the (f, h, w) grid (Qihoo-T2X reading
// note, Fig. 2 reading).  Proxy windows and TCM windows are numbered row-major
// over their window grid, and the tokens inside a window row-major over
// (t, y, x).
// ---------------------------------------------------------------------------

// Proxy windows of p_f x p_h x p_w tokens (§3 Method, Eq. GIIM "Averaging").
struct ProxyGeom {
    int f, h, w;      // token grid
    int pf, ph, pw;   // proxy ratio
    int mf, mh, mw;   // windows per axis
    int M, P;         // proxies, tokens per proxy window
    FastDiv f_mw, f_mh, f_pw, f_ph;
};

__host__ __device__ __forceinline__ int proxy_token(const ProxyGeom &g, int m, int k) {
    // k-th token (row-major inside the window) of proxy window m
    const int r = fdiv(g.f_mw, m), X = m - r * g.mw;
    const int T = fdiv(g.f_mh, r), Y = r - T * g.mh;
    const int q = fdiv(g.f_pw, k), c = k - q * g.pw;
    const int a = fdiv(g.f_ph, q), b = q - a * g.ph;
    return ((T * g.pf + a) * g.h + Y * g.ph + b) * g.w + X * g.pw + c;
}

__host__ __device__ __forceinline__ int proxy_of_token(const ProxyGeom &g, int tok) {
    int x = tok % g.w, r = tok / g.w, y = r % g.h, t = r / g.h;
    return ((t / g.pf) * g.mh + y / g.ph) * g.mw + x / g.pw;
}

// TCM windows of w_f x w_h x w_w tokens on the grid rolled by -shift
// (§3 Method, Eq. TCM; Swin-style cyclic shift).
struct WinGeom {
    int f, h, w;      // token grid
    int wf, wh, ww;   // window
    int sf, sh, sw;   // shift: window origin of the rolled grid is token (s_f, s_h, s_w)
    int nwf, nwh, nww;// windows per axis
    int n, nwin;      // tokens per window, windows per batch item
    FastDiv f_ww, f_wh, f_nww, f_nwh, f_n;
};

// Original token index held by slot `slot` of rolled-grid window `win`.
// *wrap gets one bit per axis (t: 4, y: 2, x: 1), set where the roll carried
// the token across the grid edge.  Two slots of one window may attend each
// other iff their wrap bits are equal: the shift mask is this comparison.
__host__ __device__ __forceinline__ int window_token(const WinGeom &g, int win, int slot,
                                                     int *wrap) {
    const int r = fdiv(g.f_nww, win), wx = win - r * g.nww;
    const int wt = fdiv(g.f_nwh, r), wy = r - wt * g.nwh;
    const int q = fdiv(g.f_ww, slot), sx = slot - q * g.ww;
    const int st = fdiv(g.f_wh, q), sy = q - st * g.wh;
    int t = wt * g.wf + st + g.sf;
    int y = wy * g.wh + sy + g.sh;
    int x = wx * g.ww + sx + g.sw;
    int c = 0;
    if (t >= g.f) { t -= g.f; c |= 4; }
    if (y >= g.h) { y -= g.h; c |= 2; }
    if (x >= g.w) { x -= g.w; c |= 1; }
    *wrap = c;
    return (t * g.h + y) * g.w + x;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  pdl_wait: block until the grids this one
// depends on (the previous kernel in the stream, when launched with
// launch_pdl) have completed and their writes are visible; a no-op otherwise.
// pdl_trigger: let the next kernel of the stream be scheduled (its CTAs run
// their prologue on SMs this grid has left, then wait in pdl_wait).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launches `kernel` with programmatic stream serialization: it may start while
// the previous kernel of the stream finishes, and must call pdl_wait() before
// it reads or writes anything that kernel (or an earlier one) touches.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Element conversions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// Internal launcher interfaces (host side); each returns a cudaError_t.
// ---------------------------------------------------------------------------
enum DType { DT_F32 = 0, DT_BF16 = 1 };

// out[b, m, :] = mean over window m of z[b, tok, :]
cudaError_t launch_proxy_average(int dtype, const ProxyGeom &g, int B, int D, const void *z,
                                 void *proxies, cudaStream_t s);

// out[b, m, :] = z[b, member slots[b * M + m] of window m, :] (member 0, the
// window's first token, when slots is null); a slot outside [0, P) leaves the
// row zero and sets *status to PTDIT_ERR_SHAPE.
cudaError_t launch_proxy_select(int dtype, const ProxyGeom &g, int B, int D, const void *z,
                                void *proxies, const int32_t *slots, int *status, cudaStream_t s);

// Device address of the library's status word on the current device.
int *device_status_ptr();

// SMs of the current device (0 if it cannot be read).
int num_sms();

// Tile geometry of an operand stored in tiled head layout (thl.cuh).
struct ThlDesc {
    int mode;      // 0: plain row-major; 1: identity tiles; 2: window tiles
    int vpad;      // columns 64.. padded to 128 (the row kernel's V)
    int ones;      // column d of every token row holds 1 (V: P V then also sums P)
    int tiles;     // 128-row tiles per batch item
    long rows_pb;  // rows per batch item
    int pack;      // windows per tile (window tiles)
    WinGeom g;     // window tiles
};
// C_s[rows, nseg] = A[rows, K] * W_s[nseg, K]^T (+ R_s), s < nmat.
// A has row stride lda; C_s and R_s share row stride ldc.  R_s may equal C_s
// (in-place residual) or be null.  thl[s] (or null) asks for
// C_s in tiled head layout instead (heads of width d, no residual); only the
// launchers that report support for it accept one.
// bias[s] (or null), a vector of nseg values of the call's dtype, is added to
// C_s before the activation `act` and before the residual:
// C_s = act(A W_s^T + bias_s) + R_s.
enum GemmAct { ACT_NONE = 0, ACT_GELU_TANH = 1 };
struct GemmArgs {
    int dtype;
    const void *A;
    long lda;
    const void *W[3];
    void *C[3];
    const void *R[3];
    long ldc;
    int rows, nseg, K, nmat;
    const ThlDesc *thl[3];
    int heads, d;
    const void *bias[3];
    int act;
};

// GELU, tanh form: x/2 (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).  The fp32
// path calls tanhf; the bf16 paths, whose result is rounded to bf16 (relative
// step 2^-8) right after, use the hardware tanh approximation (relative error
// about 2^-11).
__device__ __forceinline__ float gelu_tanh_arg(float x) {
    return 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
}
__device__ __forceinline__ float gelu_tanh_exact(float x) {
    return 0.5f * x * (1.f + tanhf(gelu_tanh_arg(x)));
}
__device__ __forceinline__ float gelu_tanh_fast(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(gelu_tanh_arg(x)));
    return 0.5f * x * (1.f + t);
}

// y[r, :] = LayerNorm(x[r, :]) * gamma + beta over D columns (rows x D, contiguous).
cudaError_t launch_layer_norm(int dtype, long rows, int D, const void *x, const void *gamma,
                              const void *beta, float eps, void *y, cudaStream_t s);
cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t s);

// Weight gradients dW_i = G_i^T X_i (fp32 [M][N], added into zeroed outputs):
// G_i is columns gcol[i] .. gcol[i] + M - 1 of the row-major gradient buffer
// G[src[i]] (ldg columns), X_i the first N columns of X[src[i]] (ldx columns),
// both over `rows` token rows (the reduction).
constexpr int kWgradMax = 4;
struct WgradArgs {
    const void *G[2];
    int ldg[2];
    const void *X[2];
    int ldx[2];
    int nmat;
    int src[kWgradMax], gcol[kWgradMax];
    float *dW[kWgradMax];
    int M, N, rows;
};
bool wgrad_supported(const WgradArgs &a);
cudaError_t launch_wgrad(const WgradArgs &a, cudaStream_t s);

// GIIM backward's element-wise steps (bf16): delta[b][h][q] = dO . O over head h's
// columns of row q of item b (dO in tiled head layout, identity tiles without
// padding; O row-major with row stride ld); dz = (dout +) dPa[proxy] / P.
cudaError_t launch_row_delta(const void *dO_tiles, const void *O, int B, int nq, int heads,
                             int d, long ld, float *delta, cudaStream_t s);
cudaError_t launch_proxy_broadcast(const ProxyGeom &g, int B, int D, const void *dPa,
                                   const void *dout, void *dz, cudaStream_t s);

// dst[c][r] = src[r][c] for row-major bf16 [rows][cols] matrices (dst has row
// stride ldd >= rows, so several transposes can fill one wider matrix), up to
// kTransposeMax in one launch; rows, cols and ldd multiples of 8, src and dst
// 16-byte aligned.
constexpr int kTransposeMax = 8;
struct TransposeJob {
    const void *src;
    void *dst;
    int rows, cols;
    long ldd;
};
struct TransposeBatch {
    TransposeJob job[kTransposeMax];
    int n;
};
cudaError_t launch_transpose_batch_bf16(const TransposeBatch &jb, cudaStream_t s);
// The 2-SM projection GEMM's tile order for rows x nseg outputs of nmat
// matrices on `pairs` CTA pairs (host only): *tiles, and *scheduled = 1 with
// pair q taking tile[first[q]] .. tile[first[q+1] - 1] when the launch runs a
// schedule (first and tile may be NULL to ask only), 0 for round robin.
// Returns -1 for arguments no launch takes.
int gemm_tc2_schedule(long rows, int nseg, int nmat, int pairs, int32_t *first, int32_t *tile,
                      int *tiles, int *scheduled);

// Attention core.  Head h uses columns h*d .. h*d+d-1 of q, k, v, o.
//   ATT_ROWS:   queries are rows [0, nq) and keys rows [0, nk) of each batch
//               item (proxy SA, cross-attention, full SA).
//   ATT_WINDOW: queries and keys are the tokens of one TCM window (geom),
//               pairs with different wrap bits masked.
enum AttnMode { ATT_ROWS = 0, ATT_WINDOW = 1 };
struct AttnArgs {
    int dtype, mode;
    const void *q, *k, *v;
    void *o;
    long ldq, ldk, ldv, ldo;       // row strides (elements)
    long q_bstride, k_bstride;     // rows per batch item of q/o and of k/v
    int B, heads, d;
    int nq, nk;                    // ATT_ROWS sizes per batch item
    WinGeom geom;                  // ATT_WINDOW geometry
    float scale;                   // 1/sqrt(d)
    ThlDesc tq, tk, tv;            // layouts of q, k, v (mode 0: row-major with ldq...)
    // ATT_ROWS on the tensor cores, when set: each query row's log2-sum-exp2 of its
    // scaled scores, [B][heads][nq] (the backward recomputes P from it)
    float *lse;
};
cudaError_t launch_attention(const AttnArgs &a, cudaStream_t s);
// Backward of window attention: a holds the window tiles of Q, K, V (tiled
// head layout), dout those of dL/dO; writes dQ, dK, dV as the column blocks
// [0, D), [D, 2D), [2D, 3D) of the row-major [B N][ldg] buffer dqkv.
cudaError_t launch_attention_win_bwd(const AttnArgs &a, const void *dout, void *dqkv, long ldg,
                                     cudaStream_t s);
// Backward of row attention: a holds identity tiles of Q (nq rows), K and V (nk
// rows, V without padding), dout those of dL/dO; lse and delta are [B][heads][nq].
// Writes dQ of key tile j into columns [j D, (j + 1) D) of the bf16 [B nq][ldq]
// buffer dq and adds dK, dV into the zeroed fp32 [B nk][D] buffers dk, dv.
cudaError_t launch_attention_rows_bwd(const AttnArgs &a, const void *dout, const float *lse,
                                      const float *delta, void *dq, long ldq, float *dk, float *dv,
                                      cudaStream_t s);
// dst[r][c] = sum over j < nblk of src[r][j D + c], bf16 in and out (fp32 sums); src
// has row stride lds, dst ldd.
cudaError_t launch_sum_blocks_bf16(const void *src, long rows, int nblk, int D, long lds,
                                  void *dst, long ldd, cudaStream_t s);
// mean[b][h d + c] = the mean over the nk key rows of item b of column c of head h,
// K in tiled head layout (identity tiles, no padding).
cudaError_t launch_key_mean(const void *K_tiles, int B, int nk, int heads, int d, float *mean,
                            cudaStream_t s);
// K[b][k][h d + c] -= mean[b][h d + c] for the nk valid key rows of the tiled head
// layout (identity tiles, no padding), in bf16 through fp32.
cudaError_t launch_center_keys(void *K_tiles, int B, int nk, int heads, int d, const float *mean,
                               cudaStream_t s);
// dst[b M + r][c] = bf16(src[b M + r][c] - mean over r' of src[b M + r'][c]) for the
// fp32 row-major [B M][cols] src; dst has row stride ldd.
cudaError_t launch_center_to_bf16(const float *src, int B, int M, int cols, void *dst, long ldd,
                                  cudaStream_t s);
// fp32 -> bf16, n elements (a multiple of 8), into a strided destination: element
// i of row i / cols goes to dst[(i / cols) ldd + i % cols].
cudaError_t launch_to_bf16(const float *src, long rows, int cols, void *dst, long ldd,
                           cudaStream_t s);

// Fused window Q/K/V projection + window attention (windows of 128 tokens):
// win_fused_plan fills the geometry (sub-boxes a rolled window is loaded as) or
// returns false for shapes it does not take; launch_repack_qkv writes the heads'
// [Wq_h; Wk_h; Wv_h] rows (N per head) into win_fused_weight_bytes(p) bytes;
// launch_win_fused writes the attention output, [B N, D] row-major with row
// stride p.ldo, for the token grid z ([B, F, H, W, D]).
struct WinFusedParams {
    int B, F, H, W, D, heads, d, N;  // N: weight rows per head, 3 d rounded up to 16
    int wt, wy, wx;                  // window
    int st, sy, sx;                  // shift (roll by -shift)
    int bt, by, bx;                  // sub-box of a window
    int nb, R;                       // sub-boxes per window, rows per sub-box
    int units;                       // B x windows (set by the launcher)
    float scale;                     // 1/sqrt(d)
    __nv_bfloat16 *o;
    long ldo;
    int *status;
    unsigned long long wait_ns;
};
bool win_fused_plan(int D, int heads, int d, const int window[3], const int shift[3],
                    WinFusedParams *p);
size_t win_fused_weight_bytes(const WinFusedParams &p);
cudaError_t launch_repack_qkv(const void *wq, const void *wk, const void *wv,
                              const WinFusedParams &p, void *out, cudaStream_t s);
cudaError_t launch_win_fused(const void *z, const void *wr, WinFusedParams p, cudaStream_t s);

// Debug maps written with the kernels' own index functions.
cudaError_t launch_debug_proxy_map(const ProxyGeom &g, int32_t *out, cudaStream_t s);
cudaError_t launch_debug_window_map(const WinGeom &g, int32_t *tok, uint8_t *allowed,
                                    cudaStream_t s);

// Per-launch timing hooks (no-ops unless enabled by ptdit_timing_enable).
void timing_begin(int kind, cudaStream_t s);
void timing_end(cudaStream_t s);
void timing_drop();  // forget the last record (its launch did not happen)
void count_launch();

}  // namespace ptdit
