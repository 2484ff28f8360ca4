// C ABI of the PT-DiT block-attention library: argument validation, workspace
// layout, launch ordering on the caller's stream, error reporting and the
// optional per-launch timing hooks.
//
// Launch order of ptdit_block_attn (Qihoo-T2X reading note, §3 Method and the
// code listing of ProxyTokensTransformerBlock.forward):
//   GIIM  1 average z -> P          2 Q,K,V = P W_psa^T     3 proxy SA core
//         4 P' = A W_psa,o^T (+P)   5 K_c,V_c = P' W^T      6 Q_c = z W_c,q^T
//         7 cross-attention core    8 z_out = z + O W_c,o^T
//   TCM   9 Q,K,V = z_out W_wsa^T  10 window core (shift 0) 11 z_out += O W_wsa,o^T
//        12 Q,K,V = z_out W_swsa^T 13 window core (shift s) 14 z_out += O W_swsa,o^T
// The residual stream lives in z_out from step 8 on; steps 11 and 14 add in
// place (each output element is read and written by the same thread).
// Where the tensor-core attention kernels run (bf16, head width 64..80), the
// projections write Q, K and V in tiled head layout (thl.cuh): one block per
// (tile, head) in the order the attention kernel reads them.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <vector>

#include "common.cuh"
#include "ptdit.h"
#include "thl.cuh"

namespace ptdit {
cudaError_t launch_gemm_simt(const GemmArgs &a, cudaStream_t s);
cudaError_t launch_attention_simt(const AttnArgs &a, cudaStream_t s);
bool gemm_tc2_supported(const GemmArgs &a);
cudaError_t launch_gemm_tc2(const GemmArgs &a, cudaStream_t s);
bool attention_tc_supported(const AttnArgs &a);
bool attention_thl_supported(const AttnArgs &a);
cudaError_t launch_attention_tc(const AttnArgs &a, cudaStream_t s);

// bf16 projections run on the tensor cores (2-SM kernel); fp32 projections are
// the CUDA-core FMA path.  A bf16 shape the tensor-core kernel does not take
// is refused by the API before anything is launched.
cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t s) {
    if (a.dtype == DT_BF16)
        return gemm_tc2_supported(a) ? launch_gemm_tc2(a, s) : cudaErrorNotSupported;
    for (int i = 0; i < a.nmat; ++i)  // only the 2-SM kernel writes tiled head layout
        if (a.thl[i]) return cudaErrorNotSupported;
    return launch_gemm_simt(a, s);
}

// bf16 attention runs on the tensor cores (operands in tiled head layout);
// fp32 attention is the CUDA-core FMA path.  A bf16 shape without a
// tensor-core kernel is refused by the API before anything is launched.
cudaError_t launch_attention(const AttnArgs &a, cudaStream_t s) {
    if (a.dtype == DT_BF16)
        return attention_tc_supported(a) ? launch_attention_tc(a, s) : cudaErrorNotSupported;
    return launch_attention_simt(a, s);
}

// ------------------------------------------------------------------ timing hooks
namespace {
struct TimingState {
    int max = 0;
    int count = 0;
    int open_kind = -1;
    std::vector<cudaEvent_t> ev0, ev1;
    std::vector<int> kind;
};
thread_local TimingState g_timing;
thread_local long long g_launches = 0;
}  // namespace

void timing_begin(int kind, cudaStream_t s) {
    TimingState &t = g_timing;
    if (t.max == 0 || t.count >= t.max) return;
    t.open_kind = kind;
    cudaEventRecord(t.ev0[t.count], s);
}

void timing_end(cudaStream_t s) {
    TimingState &t = g_timing;
    if (t.open_kind < 0) return;
    cudaEventRecord(t.ev1[t.count], s);
    t.kind[t.count] = t.open_kind;
    t.open_kind = -1;
    ++t.count;
}

void timing_drop() {
    TimingState &t = g_timing;
    if (t.count > 0 && t.open_kind < 0) --t.count;
}

void count_launch() { ++g_launches; }

}  // namespace ptdit

using namespace ptdit;

// ------------------------------------------------------------------ errors
namespace {
thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(PTDIT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Host-side fault injection (tests): PTDIT_FAULT=workspace or PTDIT_FAULT=launch.
bool fault(const char *kind) {
    const char *v = getenv("PTDIT_FAULT");
    return v && strcmp(v, kind) == 0;
}

// Whether this host thread's window branches may take the fused projection +
// attention kernel (ptdit_window_fused).
thread_local bool g_window_fused = false;
bool fused_window_disabled() { return !g_window_fused; }

int launch_fault(const char *what) {
    return fault("launch") ? fail(PTDIT_ERR_CUDA, "%s: launch refused (PTDIT_FAULT=launch)", what)
                           : PTDIT_OK;
}

// ------------------------------------------------------------------ validation
struct Dims {
    int B, f, h, w, D, heads, d, dtype;
    long N;
    size_t elem;
};

int check_shape(const ptdit_shape *s, Dims *o, bool attention = true) {
    if (!s) return fail(PTDIT_ERR_NULL, "shape is NULL");
    if (s->dtype != PTDIT_F32 && s->dtype != PTDIT_BF16)
        return fail(PTDIT_ERR_DTYPE, "dtype %d is neither PTDIT_F32 nor PTDIT_BF16", s->dtype);
    if (s->B < 1 || s->F < 1 || s->H < 1 || s->W < 1 || s->D < 1 || s->heads < 1)
        return fail(PTDIT_ERR_SHAPE, "B, F, H, W, D and heads must all be positive");
    if (s->D % s->heads)
        return fail(PTDIT_ERR_SHAPE, "D=%d is not divisible by heads=%d", s->D, s->heads);
    const long N = (long)s->F * s->H * s->W;
    if (N > (1L << 30) || (long)s->B * N > (1L << 31) - 1)
        return fail(PTDIT_ERR_SHAPE, "B*N=%ld tokens exceeds 2^31-1", (long)s->B * N);
    if (s->D > 16384) return fail(PTDIT_ERR_SHAPE, "D=%d above 16384", s->D);
    if (attention && s->D / s->heads > 128)
        return fail(PTDIT_ERR_SHAPE, "head dim %d above 128", s->D / s->heads);
    o->B = s->B; o->f = s->F; o->h = s->H; o->w = s->W; o->D = s->D;
    o->heads = s->heads; o->d = s->D / s->heads; o->dtype = s->dtype; o->N = N;
    o->elem = s->dtype == PTDIT_BF16 ? 2 : 4;
    return PTDIT_OK;
}

int make_proxy(const Dims &d, const int ratio[3], ProxyGeom *g) {
    if (!ratio) return fail(PTDIT_ERR_NULL, "ratio is NULL");
    const int L[3] = {d.f, d.h, d.w};
    for (int i = 0; i < 3; ++i)
        if (ratio[i] < 1 || L[i] % ratio[i])
            return fail(PTDIT_ERR_SHAPE, "grid axis %d (%d) is not divisible by ratio %d", i,
                        L[i], ratio[i]);
    g->f = d.f; g->h = d.h; g->w = d.w;
    g->pf = ratio[0]; g->ph = ratio[1]; g->pw = ratio[2];
    g->mf = d.f / ratio[0]; g->mh = d.h / ratio[1]; g->mw = d.w / ratio[2];
    g->M = g->mf * g->mh * g->mw;
    g->P = ratio[0] * ratio[1] * ratio[2];
    g->f_mw = make_fastdiv(g->mw);
    g->f_mh = make_fastdiv(g->mh);
    g->f_pw = make_fastdiv(g->pw);
    g->f_ph = make_fastdiv(g->ph);
    return PTDIT_OK;
}

int make_window(const Dims &d, const int window[3], const int shift[3], WinGeom *g) {
    if (!window) return fail(PTDIT_ERR_NULL, "window is NULL");
    if (!shift) return fail(PTDIT_ERR_NULL, "shift is NULL");
    const int L[3] = {d.f, d.h, d.w};
    for (int i = 0; i < 3; ++i) {
        if (window[i] < 1 || L[i] % window[i])
            return fail(PTDIT_ERR_SHAPE, "grid axis %d (%d) is not divisible by window %d", i,
                        L[i], window[i]);
        if (shift[i] < 0 || shift[i] >= window[i])
            return fail(PTDIT_ERR_SHAPE, "shift %d on axis %d is outside [0, window=%d)",
                        shift[i], i, window[i]);
    }
    g->f = d.f; g->h = d.h; g->w = d.w;
    g->wf = window[0]; g->wh = window[1]; g->ww = window[2];
    g->sf = shift[0]; g->sh = shift[1]; g->sw = shift[2];
    g->nwf = d.f / window[0]; g->nwh = d.h / window[1]; g->nww = d.w / window[2];
    g->n = window[0] * window[1] * window[2];
    g->nwin = g->nwf * g->nwh * g->nww;
    g->f_ww = make_fastdiv(g->ww);
    g->f_wh = make_fastdiv(g->wh);
    g->f_nww = make_fastdiv(g->nww);
    g->f_nwh = make_fastdiv(g->nwh);
    g->f_n = make_fastdiv(g->n);
    return PTDIT_OK;
}

int check_ptr(const void *p, const char *name) {
    if (!p) return fail(PTDIT_ERR_NULL, "%s is NULL", name);
    if ((uintptr_t)p % 16) return fail(PTDIT_ERR_ALIGN, "%s is not 16-byte aligned", name);
    return PTDIT_OK;
}

int check_weights(const ptdit_attn_w *w, const char *name) {
    if (!w) return fail(PTDIT_ERR_NULL, "%s weights are NULL", name);
    const void *p[4] = {w->wq, w->wk, w->wv, w->wo};
    const char *nm[4] = {"wq", "wk", "wv", "wo"};
    for (int i = 0; i < 4; ++i) {
        if (!p[i]) return fail(PTDIT_ERR_NULL, "%s.%s is NULL", name, nm[i]);
        if ((uintptr_t)p[i] % 16)
            return fail(PTDIT_ERR_ALIGN, "%s.%s is not 16-byte aligned", name, nm[i]);
    }
    return PTDIT_OK;
}

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + nb && y < x + na;
}

// ------------------------------------------------------------------ workspace
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Ws {
    size_t P, Qp, Kp, Vp, Ap, Pp, Kc, Vc, Q, K, V, O;
    size_t Xn, H, Kt, Vt;  // the complete block only: norm output, MLP hidden, text K and V
    size_t total;
    // past total: the heads' repacked Q/K/V weight rows of the fused window kernel
    // (a workspace of total_fused bytes lets windows of 128 tokens take it)
    size_t Wr, total_fused;
};

// Whether the attention operands of this shape go through tiled head layout.
bool thl_shape(const Dims &d) { return d.dtype == PTDIT_BF16 && d.d >= 8 && d.d <= 80 && d.d % 8 == 0; }

// bf16 attention has tensor-core kernels for head widths 8 .. 80 in steps of 8
// and windows of 16, 32, 64 or 128 tokens; other bf16 shapes are refused.
int check_bf16_attention(const Dims &d, const WinGeom *wg = nullptr) {
    if (d.dtype != PTDIT_BF16) return PTDIT_OK;
    if (d.D % 16)
        return fail(PTDIT_ERR_SHAPE,
                    "bf16 projections take widths D that are multiples of 16 (tensor cores); "
                    "D=%d has no bf16 kernel (PTDIT_F32 takes any width)", d.D);
    if (!thl_shape(d))
        return fail(PTDIT_ERR_SHAPE,
                    "bf16 attention takes head widths 8..80 in steps of 8 (tensor cores); "
                    "head width %d has no bf16 kernel (PTDIT_F32 takes any width)", d.d);
    if (wg && wg->n != 16 && wg->n != 32 && wg->n != 64 && wg->n != 128)
        return fail(PTDIT_ERR_SHAPE,
                    "bf16 window attention takes windows of 16, 32, 64 or 128 tokens "
                    "(tensor cores); a window of %d tokens has no bf16 kernel "
                    "(PTDIT_F32 takes any window)", wg->n);
    return PTDIT_OK;
}

// Bytes of `rows_pb` rows per batch item in tiled head layout.
size_t thl_bytes(const Dims &d, long rows_pb, int vpad) {
    return (size_t)d.B * ((rows_pb + kThlRows - 1) / kThlRows) * d.heads *
           thl_block_bytes(d.d, vpad);
}

// L, Dh: text tokens and MLP width of the complete block (0 for the attention path).
Ws ws_layout(const Dims &d, long M, long Lt = 0, long Dh = 0) {
    Ws L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    auto mx = [](size_t a, size_t b) { return a > b ? a : b; };
    const size_t pm = (size_t)d.B * M * d.D * d.elem, tn = (size_t)d.B * d.N * d.D * d.elem;
    const bool t = thl_shape(d);
    // Q and K blocks of 80 columns; V blocks padded to 128 for the row kernel
    const size_t pq = t ? thl_bytes(d, M, 0) : 0, pv = t ? thl_bytes(d, M, 1) : 0;
    const size_t tq = t ? thl_bytes(d, d.N, 0) : 0, tv = t ? thl_bytes(d, d.N, 1) : 0;
    L.P = take(pm); L.Qp = take(mx(pm, pq)); L.Kp = take(mx(pm, pq)); L.Vp = take(mx(pm, pv));
    L.Ap = take(pm); L.Pp = take(pm); L.Kc = take(mx(pm, pq)); L.Vc = take(mx(pm, pv));
    L.Q = take(mx(tn, tq)); L.K = take(mx(tn, tq)); L.V = take(mx(tn, tv)); L.O = take(tn);
    L.Xn = L.H = L.Kt = L.Vt = 0;
    if (Dh > 0) {
        const size_t tl = (size_t)d.B * Lt * d.D * d.elem;
        L.Xn = take(mx(tn, pm));
        L.H = take((size_t)d.B * d.N * Dh * d.elem);
        L.Kt = take(mx(tl, t ? thl_bytes(d, Lt, 0) : 0));
        L.Vt = take(mx(tl, t ? thl_bytes(d, Lt, 1) : 0));
    }
    L.total = off;
    L.Wr = off;
    L.total_fused = off;
    if (thl_shape(d) && d.D % 64 == 0) {  // the fused window kernel's weight rows
        const size_t N = (size_t)(3 * d.d + 15) / 16 * 16;
        L.total_fused += align256((size_t)d.heads * N * d.D * d.elem);
    }
    return L;
}

ThlDesc thl_identity(long rows_pb, int vpad, int ones = 0) {
    ThlDesc t;
    memset(&t, 0, sizeof t);
    t.mode = THL_IDENTITY;
    t.vpad = vpad;
    t.ones = ones;
    t.rows_pb = rows_pb;
    t.tiles = (int)((rows_pb + kThlRows - 1) / kThlRows);
    t.pack = 1;
    return t;
}

ThlDesc thl_window(const WinGeom &g, long N, int vpad, int ones = 0) {
    ThlDesc t;
    memset(&t, 0, sizeof t);
    t.mode = THL_WINDOW;
    t.vpad = vpad;
    t.ones = ones;
    t.rows_pb = N;
    t.pack = kThlRows / g.n;
    t.tiles = (g.nwin + t.pack - 1) / t.pack;
    t.g = g;
    return t;
}

// V operands carry a column of ones (row sums of P from the P V product) when
// the head is narrower than its 16-column-aligned tile width.
int v_ones(const Dims &d) { return d.d % 16 != 0; }

// Whether some tile rows of this layout hold no token (they must read as zeros).
bool thl_has_empty_rows(const ThlDesc &t) {
    return t.mode == THL_IDENTITY ? t.rows_pb % kThlRows != 0 : t.g.nwin % t.pack != 0;
}

int check_ws(const Dims &d, long M, const void *ws, size_t ws_bytes, Ws *L, long Lt = 0,
             long Dh = 0) {
    *L = ws_layout(d, M, Lt, Dh);
    if (fault("workspace"))
        return fail(PTDIT_ERR_WORKSPACE, "workspace refused (PTDIT_FAULT=workspace)");
    if (!ws) return fail(PTDIT_ERR_NULL, "workspace is NULL");
    if ((uintptr_t)ws % 256) return fail(PTDIT_ERR_ALIGN, "workspace is not 256-byte aligned");
    if (ws_bytes < L->total)
        return fail(PTDIT_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L->total);
    return PTDIT_OK;
}

// ------------------------------------------------------------------ launch helpers
#define TRY(x)                         \
    do {                               \
        int _rc = (x);                 \
        if (_rc != PTDIT_OK) return _rc; \
    } while (0)

struct Run {
    const Dims &d;
    cudaStream_t s;
    char *ws;
    const Ws &L;
    size_t cap = 0;  // the caller's workspace bytes (0: only L.total known)
    char *at(size_t off) const { return ws + off; }
};

// C = act(A W^T + bias) + R for one weight matrix of nseg x K (row stride K);
// A has row stride lda = K, C and R row stride ldc = nseg.
int gemm_ex(const Run &r, int kind, const void *A, long rows, int K, int nseg, const void *W,
            void *C, const void *R, const void *bias, int act, const char *what) {
    GemmArgs g;
    memset(&g, 0, sizeof g);
    g.dtype = r.d.dtype;
    g.A = A;
    g.lda = K;
    g.W[0] = W;
    g.C[0] = C;
    g.R[0] = R;
    g.bias[0] = bias;
    g.act = act;
    g.ldc = nseg;
    g.rows = (int)rows;
    g.nseg = nseg;
    g.K = K;
    g.nmat = 1;
    TRY(launch_fault(what));
    timing_begin(kind, r.s);
    cudaError_t e = launch_gemm(g, r.s);
    timing_end(r.s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, what);
}

int gemm(const Run &r, int kind, const void *A, long rows, int nmat, const void *const W[3],
         void *const C[3], const void *const R[3], const char *what) {
    GemmArgs g;
    memset(&g, 0, sizeof g);
    g.dtype = r.d.dtype;
    g.A = A;
    g.lda = r.d.D;
    for (int i = 0; i < nmat; ++i) {
        g.W[i] = W[i];
        g.C[i] = C[i];
        g.R[i] = R ? R[i] : nullptr;
    }
    g.ldc = r.d.D;
    g.rows = (int)rows;
    g.nseg = r.d.D;
    g.K = r.d.D;
    g.nmat = nmat;
    TRY(launch_fault(what));
    timing_begin(kind, r.s);
    cudaError_t e = launch_gemm(g, r.s);
    timing_end(r.s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, what);
}

// Projections whose outputs C_i are in tiled head layout where thl[i] is set:
// one fused launch of the 2-SM kernel (row-major outputs of the fp32 path: one
// projection per output).  Tile rows that hold no token are zeroed.
int gemm_thl(const Run &r, int kind, const void *A, long rows, int nmat, const void *const W[3],
             void *const C[3], const ThlDesc *const thl[3], const char *what) {
    GemmArgs g;
    memset(&g, 0, sizeof g);
    g.dtype = r.d.dtype;
    g.A = A;
    g.lda = r.d.D;
    for (int i = 0; i < nmat; ++i) {
        g.W[i] = W[i];
        g.C[i] = C[i];
        g.thl[i] = thl[i];
    }
    g.ldc = r.d.D;
    g.rows = (int)rows;
    g.nseg = r.d.D;
    g.K = r.d.D;
    g.nmat = nmat;
    g.heads = r.d.heads;
    g.d = r.d.d;
    TRY(launch_fault(what));
    cudaError_t e = cudaErrorNotSupported;
    if (gemm_tc2_supported(g)) {
        timing_begin(kind, r.s);
        e = launch_gemm_tc2(g, r.s);
        timing_end(r.s);
        if (e == cudaErrorNotSupported) {  // tensor maps refused: nothing was launched
            (void)cudaGetLastError();
            timing_drop();
        } else {
            count_launch();
        }
        if (e != cudaSuccess && e != cudaErrorNotSupported) return cuda_fail(e, what);
    }
    if (e == cudaErrorNotSupported) {
        // row-major outputs (the fp32 path): one projection per output; tiled outputs
        // exist only where the 2-SM kernel runs (every bf16 shape the API accepts)
        for (int i = 0; i < nmat; ++i) {
            if (thl[i]) return cuda_fail(cudaErrorNotSupported, what);
            const void *Wi[3] = {W[i], nullptr, nullptr};
            void *Ci[3] = {C[i], nullptr, nullptr};
            TRY(gemm(r, kind, A, rows, 1, Wi, Ci, nullptr, what));
        }
        return PTDIT_OK;
    }
    for (int i = 0; i < nmat; ++i) {
        if (!thl[i] || !thl_has_empty_rows(*thl[i])) continue;
        timing_begin(kind, r.s);
        cudaError_t e = launch_thl_zero_rows(*thl[i], r.d.B, r.d.heads, r.d.d, C[i], r.s);
        timing_end(r.s);
        count_launch();
        if (e != cudaSuccess) return cuda_fail(e, "tiled head layout");
    }
    return PTDIT_OK;
}

int attention(const Run &r, int kind, AttnArgs a, const char *what) {
    a.dtype = r.d.dtype;
    a.heads = r.d.heads;
    a.d = r.d.d;
    a.B = r.d.B;
    a.ldq = a.ldk = a.ldv = a.ldo = r.d.D;
    a.scale = 1.0f / sqrtf((float)r.d.d);
    TRY(launch_fault(what));
    timing_begin(kind, r.s);
    cudaError_t e = launch_attention(a, r.s);
    timing_end(r.s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, what);
}

// The pre-norms of the complete block (null members: the attention path, no norm).
struct NormSet {
    const ptdit_norm_w *proxy, *cross, *wsa, *swsa, *text, *mlp;
    float eps;
};

// y = LayerNorm(x) * gamma + beta over the model width, rows x D.
int layer_norm(const Run &r, const ptdit_norm_w *nw, float eps, const void *x, long rows, void *y,
               const char *what) {
    TRY(launch_fault(what));
    timing_begin(PTDIT_K_NORM, r.s);
    cudaError_t e = launch_layer_norm(r.d.dtype, rows, r.d.D, x, nw->gamma, nw->beta, eps, y, r.s);
    timing_end(r.s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, what);
}


// GIIM: z_out = (z_in +) CS(z_in, SA(Average(z_in)) (+ P_a)).
// The proxy tokens P_a of every window: the mean (the method), or one member
// of the window (the pages' Top-Left and Random ablation variants).
int extract_proxies(const Dims &d, const ProxyGeom &pg, int mode, const int32_t *slots,
                    const void *z, void *proxies, cudaStream_t s) {
    TRY(launch_fault("proxy extraction"));
    cudaError_t e;
    timing_begin(PTDIT_K_AVERAGE, s);
    if (mode == PTDIT_PROXY_MEAN) {
        e = launch_proxy_average(d.dtype, pg, d.B, d.D, z, proxies, s);
    } else {
        int *status = device_status_ptr();
        e = status ? launch_proxy_select(d.dtype, pg, d.B, d.D, z, proxies,
                                         mode == PTDIT_PROXY_RANDOM ? slots : nullptr, status, s)
                   : cudaErrorInvalidValue;
    }
    timing_end(s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, "proxy extraction");
}

int check_proxy_mode(int mode, const int32_t *slots) {
    if (mode != PTDIT_PROXY_MEAN && mode != PTDIT_PROXY_FIRST && mode != PTDIT_PROXY_RANDOM)
        return fail(PTDIT_ERR_SHAPE, "proxy mode %d is not MEAN, FIRST or RANDOM", mode);
    if (mode == PTDIT_PROXY_RANDOM) {
        if (!slots) return fail(PTDIT_ERR_NULL, "PTDIT_PROXY_RANDOM needs a slots array");
        if ((uintptr_t)slots % 4) return fail(PTDIT_ERR_ALIGN, "slots is not 4-byte aligned");
    }
    return PTDIT_OK;
}

// With norms (the complete block): the proxy self-attention reads LN(P_a) and
// adds P_a; the cross-attention's queries come from LN(z_in).
int run_giim(const Run &r, const ProxyGeom &pg, const ptdit_attn_w *psa,
             const ptdit_attn_w *cross, unsigned flags, const void *z_in, void *z_out,
             int mode = PTDIT_PROXY_MEAN, const int32_t *slots = nullptr,
             const NormSet *nm = nullptr) {
    const Dims &d = r.d;
    const long BM = (long)d.B * pg.M, BN = (long)d.B * d.N;
    TRY(extract_proxies(d, pg, mode, slots, z_in, r.at(r.L.P), r.s));
    const void *pin = r.at(r.L.P), *zq = z_in;
    if (nm) {
        TRY(layer_norm(r, nm->proxy, nm->eps, r.at(r.L.P), BM, r.at(r.L.Xn), "proxy norm"));
        pin = r.at(r.L.Xn);
    }
    AttnArgs pa;  // proxy self-attention
    memset(&pa, 0, sizeof pa);
    pa.mode = ATT_ROWS;
    pa.dtype = d.dtype;
    pa.d = d.d;
    pa.q = r.at(r.L.Qp); pa.k = r.at(r.L.Kp); pa.v = r.at(r.L.Vp); pa.o = r.at(r.L.Ap);
    pa.q_bstride = pa.k_bstride = pg.M;
    pa.nq = pa.nk = pg.M;
    const bool tiled = attention_thl_supported(pa);
    const ThlDesc tp = thl_identity(pg.M, 0), tpv = thl_identity(pg.M, 1, v_ones(d));
    if (tiled) {
        pa.tq = pa.tk = tp;
        pa.tv = tpv;
    }
    {
        const void *W[3] = {psa->wq, psa->wk, psa->wv};
        void *C[3] = {r.at(r.L.Qp), r.at(r.L.Kp), r.at(r.L.Vp)};
        const ThlDesc *T[3] = {tiled ? &tp : nullptr, tiled ? &tp : nullptr, tiled ? &tpv : nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, pin, BM, 3, W, C, T, "proxy QKV projection"));
    }
    TRY(attention(r, PTDIT_K_ATTN_PROXY, pa, "proxy self-attention"));
    {
        const void *W[3] = {psa->wo, nullptr, nullptr};
        void *C[3] = {r.at(r.L.Pp), nullptr, nullptr};
        const void *R[3] = {(nm || (flags & PTDIT_PROXY_RESIDUAL)) ? r.at(r.L.P) : nullptr,
                            nullptr, nullptr};
        TRY(gemm(r, PTDIT_K_GEMM, r.at(r.L.Ap), BM, 1, W, C, R, "proxy output projection"));
    }
    AttnArgs ca;  // cross-attention: latent queries, proxy keys and values
    memset(&ca, 0, sizeof ca);
    ca.mode = ATT_ROWS;
    ca.q = r.at(r.L.Q); ca.k = r.at(r.L.Kc); ca.v = r.at(r.L.Vc); ca.o = r.at(r.L.O);
    ca.q_bstride = d.N;
    ca.k_bstride = pg.M;
    ca.nq = (int)d.N;
    ca.nk = pg.M;
    const ThlDesc tn = thl_identity(d.N, 0);
    if (tiled) {
        ca.tq = tn;
        ca.tk = tp;
        ca.tv = tpv;
    }
    {
        const void *W[3] = {cross->wk, cross->wv, nullptr};
        void *C[3] = {r.at(r.L.Kc), r.at(r.L.Vc), nullptr};
        const ThlDesc *T[3] = {tiled ? &tp : nullptr, tiled ? &tpv : nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, r.at(r.L.Pp), BM, 2, W, C, T, "proxy K/V projection"));
    }
    if (nm) {
        TRY(layer_norm(r, nm->cross, nm->eps, z_in, BN, r.at(r.L.Xn), "cross-attention norm"));
        zq = r.at(r.L.Xn);
    }
    {
        const void *W[3] = {cross->wq, nullptr, nullptr};
        void *C[3] = {r.at(r.L.Q), nullptr, nullptr};
        const ThlDesc *T[3] = {tiled ? &tn : nullptr, nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, zq, BN, 1, W, C, T, "latent Q projection"));
    }
    TRY(attention(r, PTDIT_K_ATTN_CROSS, ca, "cross-attention"));
    {
        const void *W[3] = {cross->wo, nullptr, nullptr};
        void *C[3] = {z_out, nullptr, nullptr};
        const void *R[3] = {(flags & PTDIT_NO_RESIDUAL) ? nullptr : z_in, nullptr, nullptr};
        TRY(gemm(r, PTDIT_K_GEMM, r.at(r.L.O), BN, 1, W, C, R, "cross output projection"));
    }
    return PTDIT_OK;
}

// One TCM branch: x_out = (x_in +) WSA_or_SWSA(x_in), or, with a norm (the
// complete block), x_out = x_in + WSA_or_SWSA(LN(x_in)).  x_out may equal x_in.
// fused_ok = false: Q, K and V must come out in the workspace (a caller reuses them),
// so the fused projection + attention kernel is not taken.
int run_window(const Run &r, const WinGeom &wg, const ptdit_attn_w *w, unsigned flags,
               const void *x_in, void *x_out, const ptdit_norm_w *nw = nullptr, float eps = 0.f,
               bool fused_ok = true) {
    const Dims &d = r.d;
    const long BN = (long)d.B * d.N;
    const void *xa = x_in;
    if (nw) {
        TRY(layer_norm(r, nw, eps, x_in, BN, r.at(r.L.Xn), "window norm"));
        xa = r.at(r.L.Xn);
    }
    // windows of 128 tokens in bf16, given the workspace for the heads' repacked weight
    // rows: the projection and the attention in one kernel
    WinFusedParams fp;
    const int win3[3] = {wg.wf, wg.wh, wg.ww}, sh3[3] = {wg.sf, wg.sh, wg.sw};
    if (fused_ok && d.dtype == PTDIT_BF16 && !fused_window_disabled() &&
        win_fused_plan(d.D, d.heads, d.d, win3, sh3, &fp) && r.cap >= r.L.total_fused &&
        r.L.Wr + win_fused_weight_bytes(fp) <= r.L.total_fused) {
        void *wr = r.at(r.L.Wr);
        TRY(launch_fault("weight repack"));
        cudaError_t e = launch_repack_qkv(w->wq, w->wk, w->wv, fp, wr, r.s);
        count_launch();
        if (e != cudaSuccess) return cuda_fail(e, "weight repack");
        fp.B = d.B; fp.F = d.f; fp.H = d.h; fp.W = d.w;
        fp.scale = 1.0f / sqrtf((float)d.d);
        fp.o = reinterpret_cast<__nv_bfloat16 *>(r.at(r.L.O));
        fp.ldo = d.D;
        TRY(launch_fault("fused window attention"));
        timing_begin(PTDIT_K_ATTN_WINDOW_FUSED, r.s);
        e = launch_win_fused(xa, wr, fp, r.s);
        timing_end(r.s);
        count_launch();
        if (e != cudaSuccess) return cuda_fail(e, "fused window projection + attention");
        const void *W[3] = {w->wo, nullptr, nullptr};
        void *C[3] = {x_out, nullptr, nullptr};
        const void *R[3] = {(flags & PTDIT_NO_RESIDUAL) ? nullptr : x_in, nullptr, nullptr};
        return gemm(r, PTDIT_K_GEMM, r.at(r.L.O), BN, 1, W, C, R, "window output projection");
    }
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.mode = ATT_WINDOW;
    a.dtype = d.dtype;
    a.d = d.d;
    a.q = r.at(r.L.Q); a.k = r.at(r.L.K); a.v = r.at(r.L.V); a.o = r.at(r.L.O);
    a.q_bstride = a.k_bstride = d.N;
    a.geom = wg;
    const bool tiled = attention_thl_supported(a);
    const ThlDesc tw = thl_window(wg, d.N, 0);  // V too: the window kernel splits its P V
    const ThlDesc twv = thl_window(wg, d.N, 0, v_ones(d));
    if (tiled) {
        a.tq = a.tk = tw;
        a.tv = twv;
    }
    {
        const void *W[3] = {w->wq, w->wk, w->wv};
        void *C[3] = {r.at(r.L.Q), r.at(r.L.K), r.at(r.L.V)};
        const ThlDesc *T[3] = {tiled ? &tw : nullptr, tiled ? &tw : nullptr, tiled ? &twv : nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, xa, BN, 3, W, C, T, "window QKV projection"));
    }
    TRY(attention(r, PTDIT_K_ATTN_WINDOW, a, "window attention"));
    {
        const void *W[3] = {w->wo, nullptr, nullptr};
        void *C[3] = {x_out, nullptr, nullptr};
        const void *R[3] = {(flags & PTDIT_NO_RESIDUAL) ? nullptr : x_in, nullptr, nullptr};
        TRY(gemm(r, PTDIT_K_GEMM, r.at(r.L.O), BN, 1, W, C, R, "window output projection"));
    }
    return PTDIT_OK;
}

// Text cross-attention of the complete block, in place on z:
// z += MHA(LN(z) as queries, text tokens [B, Lt, D] as keys and values).
int run_text(const Run &r, const ptdit_attn_w *w, const ptdit_norm_w *nw, float eps,
             const void *text, int Lt, void *z) {
    const Dims &d = r.d;
    const long BN = (long)d.B * d.N, BL = (long)d.B * Lt;
    TRY(layer_norm(r, nw, eps, z, BN, r.at(r.L.Xn), "text-attention norm"));
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.mode = ATT_ROWS;
    a.dtype = d.dtype;
    a.d = d.d;
    a.q = r.at(r.L.Q); a.k = r.at(r.L.Kt); a.v = r.at(r.L.Vt); a.o = r.at(r.L.O);
    a.q_bstride = d.N;
    a.k_bstride = Lt;
    a.nq = (int)d.N;
    a.nk = Lt;
    const bool tiled = attention_thl_supported(a);
    const ThlDesc tn = thl_identity(d.N, 0), tt = thl_identity(Lt, 0),
                  ttv = thl_identity(Lt, 1, v_ones(d));
    if (tiled) {
        a.tq = tn;
        a.tk = tt;
        a.tv = ttv;
    }
    {
        const void *W[3] = {w->wk, w->wv, nullptr};
        void *C[3] = {r.at(r.L.Kt), r.at(r.L.Vt), nullptr};
        const ThlDesc *T[3] = {tiled ? &tt : nullptr, tiled ? &ttv : nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, text, BL, 2, W, C, T, "text K/V projection"));
    }
    {
        const void *W[3] = {w->wq, nullptr, nullptr};
        void *C[3] = {r.at(r.L.Q), nullptr, nullptr};
        const ThlDesc *T[3] = {tiled ? &tn : nullptr, nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, r.at(r.L.Xn), BN, 1, W, C, T,
                     "text-attention Q projection"));
    }
    TRY(attention(r, PTDIT_K_ATTN_TEXT, a, "text cross-attention"));
    return gemm_ex(r, PTDIT_K_GEMM, r.at(r.L.O), BN, d.D, d.D, w->wo, z, z, nullptr, ACT_NONE,
                   "text-attention output projection");
}

// MLP of the complete block, in place on z: z += fc2(GELU(fc1(LN(z)) + b1)) + b2.
int run_mlp(const Run &r, const ptdit_block_w *w, float eps, void *z) {
    const Dims &d = r.d;
    const long BN = (long)d.B * d.N;
    TRY(layer_norm(r, &w->norm_mlp, eps, z, BN, r.at(r.L.Xn), "MLP norm"));
    TRY(gemm_ex(r, PTDIT_K_GEMM, r.at(r.L.Xn), BN, d.D, w->mlp_hidden, w->w1, r.at(r.L.H),
                nullptr, w->b1, ACT_GELU_TANH, "MLP fc1"));
    return gemm_ex(r, PTDIT_K_GEMM, r.at(r.L.H), BN, w->mlp_hidden, d.D, w->w2, z, z, w->b2,
                   ACT_NONE, "MLP fc2");
}

int check_io(const Dims &d, const void *z_in, const void *z_out, const void *ws, size_t ws_bytes) {
    TRY(check_ptr(z_in, "z_in"));
    TRY(check_ptr(z_out, "z_out"));
    const size_t zb = (size_t)d.B * d.N * d.D * d.elem;
    if (overlap(z_in, zb, z_out, zb)) return fail(PTDIT_ERR_ALIAS, "z_out overlaps z_in");
    if (ws && overlap(ws, ws_bytes, z_out, zb))
        return fail(PTDIT_ERR_ALIAS, "z_out overlaps the workspace");
    if (ws && overlap(ws, ws_bytes, z_in, zb))
        return fail(PTDIT_ERR_ALIAS, "z_in overlaps the workspace");
    return PTDIT_OK;
}

int check_w_alias(const Dims &d, const ptdit_attn_w *w, const void *z_out) {
    const size_t wb = (size_t)d.D * d.D * d.elem, zb = (size_t)d.B * d.N * d.D * d.elem;
    const void *p[4] = {w->wq, w->wk, w->wv, w->wo};
    for (int i = 0; i < 4; ++i)
        if (overlap(p[i], wb, z_out, zb)) return fail(PTDIT_ERR_ALIAS, "z_out overlaps a weight");
    return PTDIT_OK;
}

// ------------------------------------------------------------------ backward of a TCM branch
struct WsBwd {
    size_t Q, K, V, dO, A, G, WoT, WqkvT, total;
};

// Q, K, V and dO window tiles, the recomputed attention output A, the
// gradient rows [dQ dK dV] (B N x 3 D) and the transposed weights.
WsBwd ws_layout_bwd(const Dims &d) {
    WsBwd L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t tq = thl_bytes(d, d.N, 0), tn = (size_t)d.B * d.N * d.D * d.elem;
    L.Q = take(tq); L.K = take(tq); L.V = take(tq); L.dO = take(tq);
    L.A = take(tn); L.G = take(3 * tn);
    L.WoT = take((size_t)d.D * d.D * d.elem);
    L.WqkvT = take((size_t)3 * d.D * d.D * d.elem);
    L.total = off;
    return L;
}

int check_bwd_shape(const Dims &d, const WinGeom &wg) {
    if (d.dtype != PTDIT_BF16)
        return fail(PTDIT_ERR_DTYPE, "the backward runs in bf16 only (tensor cores)");
    TRY(check_bf16_attention(d, &wg));
    if (d.D % 128)
        return fail(PTDIT_ERR_SHAPE,
                    "the backward's weight-gradient kernel takes D a multiple of 128; D=%d", d.D);
    return PTDIT_OK;
}

// The D x D weights' transposes: src[i]^T into dst[i] (row stride ldd[i]), one launch.
int transposes(const Run &r, int n, const void *const *src, void *const *dst, const long *ldd) {
    TransposeBatch jb;
    memset(&jb, 0, sizeof jb);
    jb.n = n;
    for (int i = 0; i < n; ++i) jb.job[i] = TransposeJob{src[i], dst[i], r.d.D, r.d.D, ldd[i]};
    TRY(launch_fault("weight transposes"));
    timing_begin(PTDIT_K_TRANSPOSE, r.s);
    cudaError_t e = launch_transpose_batch_bf16(jb, r.s);
    timing_end(r.s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, "weight transposes");
}

// recompute = false: Q, K, V and A already hold the branch's forward at z_in.
int run_window_bwd(const Run &r, const WsBwd &Lb, const WinGeom &wg, const ptdit_attn_w *w,
                   unsigned flags, const void *z_in, const void *dz_out, void *dz_in,
                   const ptdit_attn_wgrad *dw, bool recompute = true) {
    const Dims &d = r.d;
    const long BN = (long)d.B * d.N;
    void *Q = r.at(Lb.Q), *K = r.at(Lb.K), *V = r.at(Lb.V), *dO = r.at(Lb.dO);
    void *A = r.at(Lb.A), *G = r.at(Lb.G), *WoT = r.at(Lb.WoT), *WqkvT = r.at(Lb.WqkvT);
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.mode = ATT_WINDOW;
    a.dtype = d.dtype;
    a.d = d.d;
    a.q = Q; a.k = K; a.v = V; a.o = A;
    a.q_bstride = a.k_bstride = d.N;
    a.geom = wg;
    const ThlDesc tw = thl_window(wg, d.N, 0);
    const ThlDesc twv = thl_window(wg, d.N, 0, v_ones(d));
    a.tq = a.tk = tw;
    a.tv = twv;
    // the branch recomputed from its input: Q, K, V and the attention output A
    if (recompute) {
        const void *W[3] = {w->wq, w->wk, w->wv};
        void *C[3] = {Q, K, V};
        const ThlDesc *T[3] = {&tw, &tw, &twv};
        TRY(gemm_thl(r, PTDIT_K_GEMM, z_in, BN, 3, W, C, T, "backward: QKV projection"));
        TRY(attention(r, PTDIT_K_ATTN_WINDOW, a, "backward: window attention"));
    }
    // W^T for the input gradients: dA = dz_out Wo, dx = [dQ dK dV] [Wq; Wk; Wv]
    {
        char *qkv = static_cast<char *>(WqkvT);
        const size_t blk = (size_t)d.D * d.elem;
        const void *src[4] = {w->wo, w->wq, w->wk, w->wv};
        void *dst[4] = {WoT, qkv, qkv + blk, qkv + 2 * blk};
        const long ld[4] = {d.D, 3L * d.D, 3L * d.D, 3L * d.D};
        TRY(transposes(r, 4, src, dst, ld));
    }
    {
        const void *W[3] = {WoT, nullptr, nullptr};
        void *C[3] = {dO, nullptr, nullptr};
        const ThlDesc *T[3] = {&tw, nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, dz_out, BN, 1, W, C, T, "backward: dA = dz_out Wo"));
    }
    // dQ, dK, dV per window and head
    a.heads = d.heads;
    a.B = d.B;
    a.ldq = a.ldk = a.ldv = a.ldo = d.D;
    a.scale = 1.0f / sqrtf((float)d.d);
    TRY(launch_fault("window attention backward"));
    timing_begin(PTDIT_K_ATTN_WINDOW_BWD, r.s);
    cudaError_t e = launch_attention_win_bwd(a, dO, G, 3L * d.D, r.s);
    timing_end(r.s);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "window attention backward");
    // dz_in = (dz_out +) [dQ dK dV] [Wq; Wk; Wv]
    TRY(gemm_ex(r, PTDIT_K_GEMM, G, BN, 3 * d.D, d.D, WqkvT, dz_in,
                (flags & PTDIT_NO_RESIDUAL) ? nullptr : dz_out, nullptr, ACT_NONE,
                "backward: input gradient"));
    // weight gradients: dW{q,k,v} = [dQ dK dV]^T z_in, dWo = dz_out^T A
    float *outs[4] = {dw->dwq, dw->dwk, dw->dwv, dw->dwo};
    for (int i = 0; i < 4; ++i) {
        cudaError_t em = cudaMemsetAsync(outs[i], 0, (size_t)d.D * d.D * sizeof(float), r.s);
        if (em != cudaSuccess) return cuda_fail(em, "zeroing the weight gradients");
    }
    WgradArgs g;
    memset(&g, 0, sizeof g);
    g.G[0] = G; g.ldg[0] = 3 * d.D; g.X[0] = z_in; g.ldx[0] = d.D;
    g.G[1] = dz_out; g.ldg[1] = d.D; g.X[1] = A; g.ldx[1] = d.D;
    g.nmat = 4;
    const int src[4] = {0, 0, 0, 1}, col[4] = {0, d.D, 2 * d.D, 0};
    for (int i = 0; i < 4; ++i) {
        g.src[i] = src[i];
        g.gcol[i] = col[i];
        g.dW[i] = outs[i];
    }
    g.M = g.N = d.D;
    g.rows = (int)BN;
    if (!wgrad_supported(g)) return cuda_fail(cudaErrorNotSupported, "weight gradients");
    TRY(launch_fault("weight gradients"));
    timing_begin(PTDIT_K_WGRAD, r.s);
    e = launch_wgrad(g, r.s);
    timing_end(r.s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, "weight gradients");
}

// The TCM backward's workspace: the branch backward's, then z^ and dL/dz^.
// The SWSA branch's backward buffers, z^ and dL/dz^, and WSA's forward at z_in (its Q,
// K, V window tiles and attention output, which WSA's backward then reuses).
struct TcmBwd {
    WsBwd bwd;
    size_t zh, dzh, wq, wk, wv, wa, total;
};
TcmBwd tcm_bwd_layout(const Dims &d) {
    TcmBwd T;
    T.bwd = ws_layout_bwd(d);
    const size_t tn = align256((size_t)d.B * d.N * d.D * d.elem), tq = align256(thl_bytes(d, d.N, 0));
    T.zh = T.bwd.total;
    T.dzh = T.zh + tn;
    T.wq = T.dzh + tn;
    T.wk = T.wq + tq;
    T.wv = T.wk + tq;
    T.wa = T.wv + tq;
    T.total = T.wa + tn;
    return T;
}

// TCM's backward in the workspace at ws (tcm_bwd_layout): z^ = WSA(z_in) (+ z_in) with
// the forward's buffers laid over the backward's, then SWSA's backward at z^ and
// WSA's at z_in.
int run_tcm_bwd(const Dims &d, cudaStream_t s, char *ws, const WinGeom &wg0, const WinGeom &wg1,
                const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
                const void *z_in, const void *dz_out, void *dz_in, const ptdit_attn_wgrad *dw_wsa,
                const ptdit_attn_wgrad *dw_swsa) {
    const TcmBwd T = tcm_bwd_layout(d);
    Ws Lf{};
    Lf.Q = T.wq; Lf.K = T.wk; Lf.V = T.wv; Lf.O = T.wa;
    Run rf{d, s, ws, Lf};
    void *zh = rf.at(T.zh), *dzh = rf.at(T.dzh);
    TRY(run_window(rf, wg0, wsa, flags, z_in, zh, nullptr, 0.f, false));
    const Ws none{};
    Run r{d, s, ws, none};
    TRY(run_window_bwd(r, T.bwd, wg1, swsa, flags, zh, dz_out, dzh, dw_swsa));
    WsBwd Lw = T.bwd;  // WSA's backward on the forward kept above
    Lw.Q = T.wq; Lw.K = T.wk; Lw.V = T.wv; Lw.A = T.wa;
    return run_window_bwd(r, Lw, wg0, wsa, flags, z_in, dzh, dz_in, dw_wsa, false);
}

int check_bwd_io(const Dims &d, const ptdit_attn_w *w, const void *z_in, const void *dz_out,
                 void *dz_in, const void *ws, size_t ws_bytes) {
    TRY(check_io(d, z_in, dz_in, ws, ws_bytes));
    TRY(check_ptr(dz_out, "dz_out"));
    TRY(check_w_alias(d, w, dz_in));
    const size_t zb = (size_t)d.B * d.N * d.D * d.elem;
    if (overlap(dz_out, zb, dz_in, zb)) return fail(PTDIT_ERR_ALIAS, "dz_in overlaps dz_out");
    if (ws && overlap(ws, ws_bytes, dz_out, zb))
        return fail(PTDIT_ERR_ALIAS, "dz_out overlaps the workspace");
    return PTDIT_OK;
}

int check_wgrad(const Dims &d, const ptdit_attn_wgrad *dw, const char *name, const void *z_in,
                const void *dz_out, const void *dz_in, const void *ws, size_t ws_bytes) {
    if (!dw) return fail(PTDIT_ERR_NULL, "%s is NULL", name);
    const size_t zb = (size_t)d.B * d.N * d.D * d.elem, gb = (size_t)d.D * d.D * sizeof(float);
    const float *outs[4] = {dw->dwq, dw->dwk, dw->dwv, dw->dwo};
    const char *nm[4] = {"dwq", "dwk", "dwv", "dwo"};
    for (int i = 0; i < 4; ++i) {
        if (!outs[i]) return fail(PTDIT_ERR_NULL, "%s.%s is NULL", name, nm[i]);
        if ((uintptr_t)outs[i] % 16)
            return fail(PTDIT_ERR_ALIGN, "%s.%s is not 16-byte aligned", name, nm[i]);
        if (overlap(outs[i], gb, dz_in, zb) || overlap(outs[i], gb, z_in, zb) ||
            overlap(outs[i], gb, dz_out, zb) || (ws && overlap(outs[i], gb, ws, ws_bytes)))
            return fail(PTDIT_ERR_ALIAS, "%s.%s overlaps another argument or the workspace",
                        name, nm[i]);
        for (int j = 0; j < i; ++j)
            if (overlap(outs[i], gb, outs[j], gb))
                return fail(PTDIT_ERR_ALIAS, "%s.%s overlaps %s.%s", name, nm[i], name, nm[j]);
    }
    return PTDIT_OK;
}

int check_bwd_ws(const void *ws, size_t ws_bytes, size_t need) {
    if (fault("workspace"))
        return fail(PTDIT_ERR_WORKSPACE, "workspace refused (PTDIT_FAULT=workspace)");
    if (!ws) return fail(PTDIT_ERR_NULL, "workspace is NULL");
    if ((uintptr_t)ws % 256) return fail(PTDIT_ERR_ALIGN, "workspace is not 256-byte aligned");
    if (ws_bytes < need)
        return fail(PTDIT_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    return PTDIT_OK;
}

// ------------------------------------------------------------------ backward of GIIM
// Gc / Gq: dQ of each key tile as column blocks (only with more than one key tile),
// summed into dQc / the first block of Gp = [dQ | dK | dV] of the proxies.
struct WsGB {
    size_t Pa, Pq, Pk, Pvf, Pvb, Ap, Pp, Ck, Cvf, Cvb, dAp, dPp, dKVc, Gq, Gp, dPa;
    size_t dKc, dVc, dKp, dVp, lse_p, del_p, km_p;
    size_t Cq, Ac, dAc, Gc, dQc, lse_c, del_c, km_c;
    size_t WcoT, WcqT, WckvT, WpoT, WpT;
    int ktc, ktp;
    size_t total;
};

WsGB ws_layout_giim_bwd(const Dims &d, long M) {
    WsGB L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t e = d.elem, BM = (size_t)d.B * M, BN = (size_t)d.B * d.N, D = d.D;
    const size_t tp = thl_bytes(d, M, 0), tpv = thl_bytes(d, M, 1), tn = thl_bytes(d, d.N, 0);
    L.ktc = L.ktp = (int)((M + kThlRows - 1) / kThlRows);
    L.Pa = take(BM * D * e); L.Pq = take(tp); L.Pk = take(tp); L.Pvf = take(tpv); L.Pvb = take(tp);
    L.Ap = take(BM * D * e); L.Pp = take(BM * D * e);
    L.Ck = take(tp); L.Cvf = take(tpv); L.Cvb = take(tp);
    L.dAp = take(tp); L.dPp = take(BM * D * e); L.dKVc = take(BM * 2 * D * e);
    L.Gq = take(L.ktp > 1 ? BM * L.ktp * D * e : 0); L.Gp = take(BM * 3 * D * e);
    L.dPa = take(BM * D * e);
    L.dKc = take(BM * D * 4); L.dVc = take(BM * D * 4); L.dKp = take(BM * D * 4);
    L.dVp = take(BM * D * 4);
    L.lse_p = take(BM * d.heads * 4); L.del_p = take(BM * d.heads * 4);
    L.km_p = take((size_t)d.B * D * 4); L.km_c = take((size_t)d.B * D * 4);
    L.Cq = take(tn); L.Ac = take(BN * D * e); L.dAc = take(tn);
    L.Gc = take(L.ktc > 1 ? BN * L.ktc * D * e : 0); L.dQc = take(BN * D * e);
    L.lse_c = take(BN * d.heads * 4); L.del_c = take(BN * d.heads * 4);
    L.WcoT = take(D * D * e); L.WcqT = take(D * D * e); L.WckvT = take(D * 2 * D * e);
    L.WpoT = take(D * D * e); L.WpT = take(D * 3 * D * e);
    L.total = off;
    return L;
}

// dW[i] (+)= G^T X over `rows` rows for column blocks gcol[i] of G: launches of up to
// kWgradMax matrices (several blocks may add into one dW).
int wgrad_blocks(const Run &r, const void *G, int ldg, const int *gcol, float *const *dW, int n,
                 const void *X, long rows, const char *what) {
    for (int i0 = 0; i0 < n; i0 += kWgradMax) {
        WgradArgs g;
        memset(&g, 0, sizeof g);
        g.G[0] = G; g.ldg[0] = ldg; g.X[0] = X; g.ldx[0] = r.d.D;
        g.nmat = n - i0 < kWgradMax ? n - i0 : kWgradMax;
        for (int i = 0; i < g.nmat; ++i) {
            g.src[i] = 0;
            g.gcol[i] = gcol[i0 + i];
            g.dW[i] = dW[i0 + i];
        }
        g.M = g.N = r.d.D;
        g.rows = (int)rows;
        if (!wgrad_supported(g)) return cuda_fail(cudaErrorNotSupported, what);
        TRY(launch_fault(what));
        timing_begin(PTDIT_K_WGRAD, r.s);
        cudaError_t e = launch_wgrad(g, r.s);
        timing_end(r.s);
        count_launch();
        if (e != cudaSuccess) return cuda_fail(e, what);
    }
    return PTDIT_OK;
}

int rows_bwd(const Run &r, AttnArgs a, const void *dO, const float *lse, const float *del,
             void *dq, long ldq, float *dk, float *dv, const char *what) {
    a.dtype = r.d.dtype;
    a.heads = r.d.heads;
    a.d = r.d.d;
    a.B = r.d.B;
    a.scale = 1.0f / sqrtf((float)r.d.d);
    for (float *p : {dk, dv}) {
        cudaError_t em = cudaMemsetAsync(p, 0, (size_t)r.d.B * a.nk * r.d.D * sizeof(float), r.s);
        if (em != cudaSuccess) return cuda_fail(em, "zeroing the key and value gradients");
    }
    TRY(launch_fault(what));
    timing_begin(PTDIT_K_ATTN_ROWS_BWD, r.s);
    cudaError_t e = launch_attention_rows_bwd(a, dO, lse, del, dq, ldq, dk, dv, r.s);
    timing_end(r.s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, what);
}

int elementwise(const Run &r, cudaError_t e, const char *what) {
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, what);
}

// Keys in tiled head layout less their mean over each item's nk keys, in place (the
// attention's output is unchanged; its backward then keeps the keys' common
// component out of dQ).
int center_keys(const Run &r, void *K, int nk, float *mean) {
    const Dims &d = r.d;
    TRY(elementwise(r, launch_key_mean(K, d.B, nk, d.heads, d.d, mean, r.s), "backward: key mean"));
    return elementwise(r, launch_center_keys(K, d.B, nk, d.heads, d.d, mean, r.s),
                       "backward: keys less their mean");
}

// The attention arguments of GIIM's two cores over the backward's workspace.
AttnArgs giim_bwd_proxy_args(const Run &r, const WsGB &Lb, int M) {
    AttnArgs pa;
    memset(&pa, 0, sizeof pa);
    pa.mode = ATT_ROWS;
    pa.q = r.at(Lb.Pq); pa.k = r.at(Lb.Pk); pa.v = r.at(Lb.Pvf); pa.o = r.at(Lb.Ap);
    pa.q_bstride = pa.k_bstride = M;
    pa.nq = pa.nk = M;
    pa.tq = pa.tk = thl_identity(M, 0);
    pa.tv = thl_identity(M, 1, v_ones(r.d));
    pa.lse = reinterpret_cast<float *>(r.at(Lb.lse_p));
    return pa;
}

AttnArgs giim_bwd_cross_args(const Run &r, const WsGB &Lb, int M) {
    AttnArgs ca;
    memset(&ca, 0, sizeof ca);
    ca.mode = ATT_ROWS;
    ca.q = r.at(Lb.Cq); ca.k = r.at(Lb.Ck); ca.v = r.at(Lb.Cvf); ca.o = r.at(Lb.Ac);
    ca.q_bstride = r.d.N;
    ca.k_bstride = M;
    ca.nq = (int)r.d.N;
    ca.nk = M;
    ca.tq = thl_identity(r.d.N, 0);
    ca.tk = thl_identity(M, 0);
    ca.tv = thl_identity(M, 1, v_ones(r.d));
    ca.lse = reinterpret_cast<float *>(r.at(Lb.lse_c));
    return ca;
}

// GIIM's forward recomputed into the backward's workspace, keeping what the backward
// reads (proxies, projections with centred keys, both cores' outputs and log-sum-exp);
// with z1 set, also the module's output z1 = (z_in +) A_c Wo^T.
int giim_recompute(const Run &r, const WsGB &Lb, const ProxyGeom &pg, const ptdit_attn_w *psa,
                   const ptdit_attn_w *cross, unsigned flags, const void *z_in, void *z1) {
    const Dims &d = r.d;
    const int M = pg.M;
    const long BM = (long)d.B * M, BN = (long)d.B * d.N;
    auto P = [&](size_t o) { return r.at(o); };
    auto F = [&](size_t o) { return reinterpret_cast<float *>(r.at(o)); };
    const ThlDesc tp = thl_identity(M, 0), tpv = thl_identity(M, 1, v_ones(d));
    const ThlDesc tn = thl_identity(d.N, 0);
    TRY(extract_proxies(d, pg, PTDIT_PROXY_MEAN, nullptr, z_in, P(Lb.Pa), r.s));
    {
        const void *W[3] = {psa->wq, psa->wk, psa->wv};
        void *C[3] = {P(Lb.Pq), P(Lb.Pk), P(Lb.Pvf)};
        const ThlDesc *T[3] = {&tp, &tp, &tpv};
        TRY(gemm_thl(r, PTDIT_K_GEMM, P(Lb.Pa), BM, 3, W, C, T, "backward: proxy QKV"));
        const void *Wv[3] = {psa->wv, nullptr, nullptr};
        void *Cv[3] = {P(Lb.Pvb), nullptr, nullptr};
        const ThlDesc *Tv[3] = {&tp, nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, P(Lb.Pa), BM, 1, Wv, Cv, Tv, "backward: proxy V"));
    }
    TRY(center_keys(r, P(Lb.Pk), M, F(Lb.km_p)));
    TRY(attention(r, PTDIT_K_ATTN_PROXY, giim_bwd_proxy_args(r, Lb, M),
                  "backward: proxy self-attention"));
    {
        const void *W[3] = {psa->wo, nullptr, nullptr};
        void *C[3] = {P(Lb.Pp), nullptr, nullptr};
        const void *R[3] = {(flags & PTDIT_PROXY_RESIDUAL) ? P(Lb.Pa) : nullptr, nullptr, nullptr};
        TRY(gemm(r, PTDIT_K_GEMM, P(Lb.Ap), BM, 1, W, C, R, "backward: proxy output"));
    }
    {
        const void *W[3] = {cross->wk, cross->wv, cross->wv};
        void *C[3] = {P(Lb.Ck), P(Lb.Cvf), P(Lb.Cvb)};
        const ThlDesc *T[3] = {&tp, &tpv, &tp};
        TRY(gemm_thl(r, PTDIT_K_GEMM, P(Lb.Pp), BM, 3, W, C, T, "backward: proxy K/V"));
        const void *Wq[3] = {cross->wq, nullptr, nullptr};
        void *Cq[3] = {P(Lb.Cq), nullptr, nullptr};
        const ThlDesc *Tq[3] = {&tn, nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, z_in, BN, 1, Wq, Cq, Tq, "backward: latent Q"));
    }
    TRY(center_keys(r, P(Lb.Ck), M, F(Lb.km_c)));
    TRY(attention(r, PTDIT_K_ATTN_CROSS, giim_bwd_cross_args(r, Lb, M), "backward: cross-attention"));
    if (z1) {
        const void *W[3] = {cross->wo, nullptr, nullptr};
        void *C[3] = {z1, nullptr, nullptr};
        const void *R[3] = {(flags & PTDIT_NO_RESIDUAL) ? nullptr : z_in, nullptr, nullptr};
        TRY(gemm(r, PTDIT_K_GEMM, P(Lb.Ac), BN, 1, W, C, R, "backward: cross output projection"));
    }
    return PTDIT_OK;
}

// GIIM's backward once giim_recompute has filled the workspace.
int giim_backward(const Run &r, const WsGB &Lb, const ProxyGeom &pg, const ptdit_attn_w *psa,
                  const ptdit_attn_w *cross, unsigned flags, const void *z_in, const void *dz_out,
                  void *dz_in, const ptdit_attn_wgrad *dwp, const ptdit_attn_wgrad *dwc) {
    const Dims &d = r.d;
    const int M = pg.M, D = d.D, ktc = Lb.ktc, ktp = Lb.ktp;
    const long BM = (long)d.B * M, BN = (long)d.B * d.N;
    auto P = [&](size_t o) { return r.at(o); };
    auto F = [&](size_t o) { return reinterpret_cast<float *>(r.at(o)); };
    const ThlDesc tp = thl_identity(M, 0), tn = thl_identity(d.N, 0);
    const AttnArgs pa = giim_bwd_proxy_args(r, Lb, M), ca = giim_bwd_cross_args(r, Lb, M);
    // ---- transposed weights for the input gradients
    const long ldp = 3L * D;
    {
        const size_t blk = (size_t)D * d.elem;
        const void *src[8] = {cross->wo, cross->wq, cross->wk, cross->wv,
                              psa->wo, psa->wq, psa->wk, psa->wv};
        void *dst[8] = {P(Lb.WcoT), P(Lb.WcqT), P(Lb.WckvT), P(Lb.WckvT) + blk,
                        P(Lb.WpoT), P(Lb.WpT), P(Lb.WpT) + blk, P(Lb.WpT) + 2 * blk};
        const long ld[8] = {D, D, 2L * D, 2L * D, D, ldp, ldp, ldp};
        TRY(transposes(r, 8, src, dst, ld));
    }
    // ---- cross-attention backward
    {
        const void *W[3] = {P(Lb.WcoT), nullptr, nullptr};
        void *C[3] = {P(Lb.dAc), nullptr, nullptr};
        const ThlDesc *T[3] = {&tn, nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, dz_out, BN, 1, W, C, T, "backward: dA = dz_out Wo"));
    }
    TRY(elementwise(r, launch_row_delta(P(Lb.dAc), P(Lb.Ac), d.B, (int)d.N, d.heads, d.d, D,
                                        F(Lb.del_c), r.s), "backward: rowsum(dO O)"));
    AttnArgs cb = ca;
    cb.v = P(Lb.Cvb);
    cb.tv = tp;
    // dQ straight into dQc with one key tile, else per key tile, then summed
    TRY(rows_bwd(r, cb, P(Lb.dAc), F(Lb.lse_c), F(Lb.del_c), ktc > 1 ? P(Lb.Gc) : P(Lb.dQc), ktc > 1 ? (long)ktc * D : (long)D, F(Lb.dKc),
                 F(Lb.dVc), "cross-attention backward"));
    if (ktc > 1)
        TRY(elementwise(r, launch_sum_blocks_bf16(P(Lb.Gc), BN, ktc, D, (long)ktc * D, P(Lb.dQc), D,
                                                  r.s), "backward: dQ over the key tiles"));
    TRY(elementwise(r, launch_center_to_bf16(F(Lb.dKc), d.B, M, D, P(Lb.dKVc), 2L * D, r.s),
                    "backward: dK"));
    TRY(elementwise(r, launch_to_bf16(F(Lb.dVc), BM, D, P(Lb.dKVc) + (size_t)D * d.elem, 2L * D, r.s),
                    "backward: dV"));
    TRY(gemm_ex(r, PTDIT_K_GEMM, P(Lb.dKVc), BM, 2 * D, D, P(Lb.WckvT), P(Lb.dPp), nullptr, nullptr,
                ACT_NONE, "backward: dP' = dK Wk + dV Wv"));
    // ---- proxy self-attention backward
    {
        const void *W[3] = {P(Lb.WpoT), nullptr, nullptr};
        void *C[3] = {P(Lb.dAp), nullptr, nullptr};
        const ThlDesc *T[3] = {&tp, nullptr, nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, P(Lb.dPp), BM, 1, W, C, T, "backward: dAp = dP' Wo"));
    }
    TRY(elementwise(r, launch_row_delta(P(Lb.dAp), P(Lb.Ap), d.B, M, d.heads, d.d, D, F(Lb.del_p),
                                        r.s), "backward: proxy rowsum(dO O)"));
    AttnArgs pb = pa;
    pb.v = P(Lb.Pvb);
    pb.tv = tp;
    TRY(rows_bwd(r, pb, P(Lb.dAp), F(Lb.lse_p), F(Lb.del_p), ktp > 1 ? P(Lb.Gq) : P(Lb.Gp), ktp > 1 ? (long)ktp * D : ldp, F(Lb.dKp),
                 F(Lb.dVp), "proxy self-attention backward"));
    if (ktp > 1)
        TRY(elementwise(r, launch_sum_blocks_bf16(P(Lb.Gq), BM, ktp, D, (long)ktp * D, P(Lb.Gp), ldp,
                                                  r.s), "backward: proxy dQ over the key tiles"));
    TRY(elementwise(r, launch_center_to_bf16(F(Lb.dKp), d.B, M, D, P(Lb.Gp) + (size_t)D * d.elem,
                                             ldp, r.s), "backward: proxy dK"));
    TRY(elementwise(r, launch_to_bf16(F(Lb.dVp), BM, D, P(Lb.Gp) + (size_t)2 * D * d.elem, ldp, r.s),
                    "backward: proxy dV"));
    TRY(gemm_ex(r, PTDIT_K_GEMM, P(Lb.Gp), BM, (int)ldp, D, P(Lb.WpT), P(Lb.dPa),
                (flags & PTDIT_PROXY_RESIDUAL) ? P(Lb.dPp) : nullptr, nullptr, ACT_NONE,
                "backward: dP_a"));
    // ---- dz_in = (dz_out +) averaging^T(dP_a) + dQ Wq
    TRY(elementwise(r, launch_proxy_broadcast(pg, d.B, D, P(Lb.dPa),
                                              (flags & PTDIT_NO_RESIDUAL) ? nullptr : dz_out, dz_in, r.s),
                    "backward: averaging adjoint"));
    TRY(gemm_ex(r, PTDIT_K_GEMM, P(Lb.dQc), BN, D, D, P(Lb.WcqT), dz_in, dz_in, nullptr,
                ACT_NONE, "backward: input gradient"));
    // ---- weight gradients
    float *outs[8] = {dwp->dwq, dwp->dwk, dwp->dwv, dwp->dwo, dwc->dwq, dwc->dwk, dwc->dwv, dwc->dwo};
    for (float *o : outs) {
        cudaError_t em = cudaMemsetAsync(o, 0, (size_t)D * D * sizeof(float), r.s);
        if (em != cudaSuccess) return cuda_fail(em, "zeroing the weight gradients");
    }
    {
        const int c0[1] = {0};
        float *o1[1] = {dwc->dwo};
        TRY(wgrad_blocks(r, dz_out, D, c0, o1, 1, P(Lb.Ac), BN, "backward: dWo (cross)"));
        TRY(wgrad_blocks(r, P(Lb.dQc), D, c0, &outs[4], 1, z_in, BN, "backward: dWq (cross)"));
        const int ckv[2] = {0, D};
        float *okv[2] = {dwc->dwk, dwc->dwv};
        TRY(wgrad_blocks(r, P(Lb.dKVc), 2 * D, ckv, okv, 2, P(Lb.Pp), BM, "backward: dWk, dWv (cross)"));
        TRY(wgrad_blocks(r, P(Lb.dPp), D, c0, &outs[3], 1, P(Lb.Ap), BM, "backward: dWo (proxy)"));
        const int cp[3] = {0, D, 2 * D};
        TRY(wgrad_blocks(r, P(Lb.Gp), (int)ldp, cp, &outs[0], 3, P(Lb.Pa), BM,
                         "backward: dWq, dWk, dWv (proxy)"));
    }
    return PTDIT_OK;
}

int run_giim_bwd(const Run &r, const WsGB &Lb, const ProxyGeom &pg, const ptdit_attn_w *psa,
                 const ptdit_attn_w *cross, unsigned flags, const void *z_in, const void *dz_out,
                 void *dz_in, const ptdit_attn_wgrad *dwp, const ptdit_attn_wgrad *dwc) {
    TRY(giim_recompute(r, Lb, pg, psa, cross, flags, z_in, nullptr));
    return giim_backward(r, Lb, pg, psa, cross, flags, z_in, dz_out, dz_in, dwp, dwc);
}

// ------------------------------------------------------------------ backward of the path
// z1 and dL/dz1, GIIM's backward area (its recomputed forward stays there while TCM's
// backward runs), then TCM's backward area.
struct BlockBwd {
    size_t z1, dz1, giim, tcm, total;
};
BlockBwd block_bwd_layout(const Dims &d, long M) {
    BlockBwd L;
    const size_t tn = align256((size_t)d.B * d.N * d.D * d.elem);
    L.z1 = 0;
    L.dz1 = tn;
    L.giim = 2 * tn;
    L.tcm = L.giim + ws_layout_giim_bwd(d, M).total;
    L.total = L.tcm + tcm_bwd_layout(d).total;
    return L;
}

// The block path's geometry for the backward entry points: shape, proxies, both
// windows, the backward's restrictions.
int path_geometry(const ptdit_shape *shape, const int ratio[3], const int window[3],
                  const int shift[3], Dims *d, ProxyGeom *pg, WinGeom *wg0, WinGeom *wg1) {
    const int zero[3] = {0, 0, 0};
    TRY(check_shape(shape, d));
    TRY(make_proxy(*d, ratio, pg));
    TRY(make_window(*d, window, shift, wg1));
    TRY(make_window(*d, window, zero, wg0));
    TRY(check_bwd_shape(*d, *wg0));
    if ((pg->M + kThlRows - 1) / kThlRows > 64)
        return fail(PTDIT_ERR_SHAPE, "the backward takes at most 8192 proxies; M=%d", pg->M);
    return PTDIT_OK;
}

// The four modules' weights and weight gradients against each other and the I/O.
int check_path_grads(const Dims &d, const ptdit_attn_w *const *W, const ptdit_attn_wgrad *const *G,
                     const void *z_in, const void *dz_out, const void *dz_in, const void *ws,
                     size_t ws_bytes) {
    const char *wn[4] = {"psa", "cross", "wsa", "swsa"};
    const char *gn[4] = {"dw_psa", "dw_cross", "dw_wsa", "dw_swsa"};
    for (int m = 0; m < 4; ++m) {
        TRY(check_weights(W[m], wn[m]));
        TRY(check_bwd_io(d, W[m], z_in, dz_out, const_cast<void *>(dz_in), ws, ws_bytes));
    }
    for (int m = 0; m < 4; ++m) TRY(check_wgrad(d, G[m], gn[m], z_in, dz_out, dz_in, ws, ws_bytes));
    const size_t gb = (size_t)d.D * d.D * sizeof(float);
    for (int m = 0; m < 4; ++m)
        for (int n = 0; n < m; ++n) {
            const float *a[4] = {G[m]->dwq, G[m]->dwk, G[m]->dwv, G[m]->dwo};
            const float *b[4] = {G[n]->dwq, G[n]->dwk, G[n]->dwv, G[n]->dwo};
            for (int i = 0; i < 4; ++i)
                for (int j = 0; j < 4; ++j)
                    if (overlap(a[i], gb, b[j], gb))
                        return fail(PTDIT_ERR_ALIAS, "%s and %s overlap", gn[m], gn[n]);
        }
    return PTDIT_OK;
}

// The training pair's workspace: the whole-path backward's areas (z1, dL/dz1, GIIM's
// area, TCM's area with z^ and WSA's kept forward), then SWSA's kept Q, K, V window
// tiles and attention output.
struct TrainLayout {
    BlockBwd b;
    size_t sq, sk, sv, sa, total;
};
TrainLayout train_layout(const Dims &d, long M) {
    TrainLayout T;
    T.b = block_bwd_layout(d, M);
    const size_t tq = align256(thl_bytes(d, d.N, 0));
    T.sq = T.b.total;
    T.sk = T.sq + tq;
    T.sv = T.sk + tq;
    T.sa = T.sv + tq;
    T.total = T.sa + align256((size_t)d.B * d.N * d.D * d.elem);
    return T;
}

}  // namespace

namespace ptdit {
// Records a failure for ptdit_last_error() from another translation unit.
int report_error(int code, const char *text) { return fail(code, "%s", text); }
}  // namespace ptdit

// ------------------------------------------------------------------ exported API
extern "C" {

const char *ptdit_strerror(int status) {
    switch (status) {
        case PTDIT_OK: return "ok";
        case PTDIT_ERR_NULL: return "a required pointer is NULL";
        case PTDIT_ERR_SHAPE: return "invalid sizes, ratio, window or shift";
        case PTDIT_ERR_DTYPE: return "unknown dtype";
        case PTDIT_ERR_WORKSPACE: return "workspace too small";
        case PTDIT_ERR_CUDA: return "CUDA error";
        case PTDIT_ERR_TIMEOUT: return "a bounded device wait gave up";
        case PTDIT_ERR_ALIGN: return "pointer not aligned";
        case PTDIT_ERR_ALIAS: return "output overlaps an input";
        default: return "unknown status";
    }
}

const char *ptdit_last_error(void) { return g_err; }

long long ptdit_launch_count(void) { return g_launches; }

int ptdit_timing_enable(int max_launches) {
    TimingState &t = g_timing;
    for (auto e : t.ev0) cudaEventDestroy(e);
    for (auto e : t.ev1) cudaEventDestroy(e);
    t.ev0.clear(); t.ev1.clear(); t.kind.clear();
    t.max = t.count = 0;
    t.open_kind = -1;
    if (max_launches <= 0) return PTDIT_OK;
    t.ev0.resize(max_launches);
    t.ev1.resize(max_launches);
    t.kind.resize(max_launches);
    for (int i = 0; i < max_launches; ++i) {
        cudaError_t e = cudaEventCreate(&t.ev0[i]);
        if (e == cudaSuccess) e = cudaEventCreate(&t.ev1[i]);
        if (e != cudaSuccess) {
            t.ev0.resize(i); t.ev1.resize(i);
            ptdit_timing_enable(0);
            return cuda_fail(e, "cudaEventCreate");
        }
    }
    t.max = max_launches;
    return PTDIT_OK;
}

int ptdit_timing_read(int *kind, float *ms, int max) {
    TimingState &t = g_timing;
    const int n = t.count < max ? t.count : max;
    if (t.count > 0) {
        cudaError_t e = cudaEventSynchronize(t.ev1[t.count - 1]);
        if (e != cudaSuccess) {
            cuda_fail(e, "cudaEventSynchronize");
            return -1;
        }
    }
    for (int i = 0; i < n; ++i) {
        float v = 0.f;
        if (cudaEventElapsedTime(&v, t.ev0[i], t.ev1[i]) != cudaSuccess) {
            fail(PTDIT_ERR_CUDA, "cudaEventElapsedTime failed");
            return -1;
        }
        kind[i] = t.kind[i];
        ms[i] = v;
    }
    t.count = 0;
    return n;
}

size_t ptdit_workspace_bytes(const ptdit_shape *shape, const int ratio[3], const int window[3]) {
    Dims d;
    if (check_shape(shape, &d) != PTDIT_OK) return 0;
    long M = 0;
    if (ratio) {
        ProxyGeom pg;
        if (make_proxy(d, ratio, &pg) != PTDIT_OK) return 0;
        M = pg.M;
    }
    if (window) {
        const int zero[3] = {0, 0, 0};
        WinGeom wg;
        if (make_window(d, window, zero, &wg) != PTDIT_OK) return 0;
        if (wg.n == 128) return ws_layout(d, M).total_fused;
    }
    return ws_layout(d, M).total;
}

int ptdit_proxy_average(const ptdit_shape *shape, const int ratio[3], const void *z,
                        void *proxies, ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    TRY(check_shape(shape, &d, false));
    TRY(make_proxy(d, ratio, &pg));
    TRY(check_ptr(z, "z"));
    TRY(check_ptr(proxies, "proxies"));
    if (overlap(z, (size_t)d.B * d.N * d.D * d.elem, proxies, (size_t)d.B * pg.M * d.D * d.elem))
        return fail(PTDIT_ERR_ALIAS, "proxies overlap z");
    TRY(launch_fault("proxy average"));
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(PTDIT_K_AVERAGE, s);
    cudaError_t e = launch_proxy_average(d.dtype, pg, d.B, d.D, z, proxies, s);
    timing_end(s);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, "proxy average");
}

int ptdit_proxy_extract(const ptdit_shape *shape, const int ratio[3], int mode,
                        const int32_t *slots, const void *z, void *proxies,
                        ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    TRY(check_shape(shape, &d, false));
    TRY(make_proxy(d, ratio, &pg));
    TRY(check_proxy_mode(mode, slots));
    TRY(check_ptr(z, "z"));
    TRY(check_ptr(proxies, "proxies"));
    if (overlap(z, (size_t)d.B * d.N * d.D * d.elem, proxies, (size_t)d.B * pg.M * d.D * d.elem))
        return fail(PTDIT_ERR_ALIAS, "proxies overlap z");
    return extract_proxies(d, pg, mode, slots, z, proxies, (cudaStream_t)stream);
}

int ptdit_giim_ex(const ptdit_shape *shape, const int ratio[3], int mode, const int32_t *slots,
                  const ptdit_attn_w *psa, const ptdit_attn_w *cross, unsigned flags,
                  const void *z_in, void *z_out, void *ws, size_t ws_bytes,
                  ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    Ws L;
    TRY(check_shape(shape, &d));
    TRY(check_bf16_attention(d));
    TRY(make_proxy(d, ratio, &pg));
    TRY(check_proxy_mode(mode, slots));
    TRY(check_weights(psa, "psa"));
    TRY(check_weights(cross, "cross"));
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    TRY(check_w_alias(d, psa, z_out));
    TRY(check_w_alias(d, cross, z_out));
    TRY(check_ws(d, pg.M, ws, ws_bytes, &L));
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), L};
    r.cap = ws_bytes;
    return run_giim(r, pg, psa, cross, flags, z_in, z_out, mode, slots);
}

int ptdit_giim(const ptdit_shape *shape, const int ratio[3], const ptdit_attn_w *psa,
               const ptdit_attn_w *cross, unsigned flags, const void *z_in, void *z_out,
               void *ws, size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    Ws L;
    TRY(check_shape(shape, &d));
    TRY(check_bf16_attention(d));
    TRY(make_proxy(d, ratio, &pg));
    TRY(check_weights(psa, "psa"));
    TRY(check_weights(cross, "cross"));
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    TRY(check_w_alias(d, psa, z_out));
    TRY(check_w_alias(d, cross, z_out));
    TRY(check_ws(d, pg.M, ws, ws_bytes, &L));
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), L};
    r.cap = ws_bytes;
    return run_giim(r, pg, psa, cross, flags, z_in, z_out);
}

int ptdit_window_attn(const ptdit_shape *shape, const int window[3], const int shift[3],
                      const ptdit_attn_w *w, unsigned flags, const void *z_in, void *z_out,
                      void *ws, size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    WinGeom wg;
    Ws L;
    TRY(check_shape(shape, &d));
    TRY(make_window(d, window, shift, &wg));
    TRY(check_bf16_attention(d, &wg));
    TRY(check_weights(w, "w"));
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    TRY(check_w_alias(d, w, z_out));
    TRY(check_ws(d, 0, ws, ws_bytes, &L));
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), L};
    r.cap = ws_bytes;
    return run_window(r, wg, w, flags, z_in, z_out);
}

size_t ptdit_window_attn_bwd_workspace_bytes(const ptdit_shape *shape, const int window[3]) {
    Dims d;
    if (check_shape(shape, &d) != PTDIT_OK) return 0;
    const int zero[3] = {0, 0, 0};
    WinGeom wg;
    if (make_window(d, window, zero, &wg) != PTDIT_OK) return 0;
    return ws_layout_bwd(d).total;
}

int ptdit_window_attn_bwd(const ptdit_shape *shape, const int window[3], const int shift[3],
                          const ptdit_attn_w *w, unsigned flags, const void *z_in,
                          const void *dz_out, void *dz_in, const ptdit_attn_wgrad *dw, void *ws,
                          size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    WinGeom wg;
    TRY(check_shape(shape, &d));
    TRY(make_window(d, window, shift, &wg));
    TRY(check_bwd_shape(d, wg));
    TRY(check_weights(w, "w"));
    TRY(check_bwd_io(d, w, z_in, dz_out, dz_in, ws, ws_bytes));
    TRY(check_wgrad(d, dw, "dw", z_in, dz_out, dz_in, ws, ws_bytes));
    const WsBwd Lb = ws_layout_bwd(d);
    TRY(check_bwd_ws(ws, ws_bytes, Lb.total));
    const Ws none{};
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), none};
    return run_window_bwd(r, Lb, wg, w, flags, z_in, dz_out, dz_in, dw);
}

size_t ptdit_giim_bwd_workspace_bytes(const ptdit_shape *shape, const int ratio[3]) {
    Dims d;
    ProxyGeom pg;
    if (check_shape(shape, &d) != PTDIT_OK || make_proxy(d, ratio, &pg) != PTDIT_OK) return 0;
    return ws_layout_giim_bwd(d, pg.M).total;
}

int ptdit_giim_bwd(const ptdit_shape *shape, const int ratio[3], const ptdit_attn_w *psa,
                   const ptdit_attn_w *cross, unsigned flags, const void *z_in, const void *dz_out,
                   void *dz_in, const ptdit_attn_wgrad *dw_psa, const ptdit_attn_wgrad *dw_cross,
                   void *ws, size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    TRY(check_shape(shape, &d));
    TRY(make_proxy(d, ratio, &pg));
    if (d.dtype != PTDIT_BF16)
        return fail(PTDIT_ERR_DTYPE, "the backward runs in bf16 only (tensor cores)");
    TRY(check_bf16_attention(d));
    if (d.D % 128)
        return fail(PTDIT_ERR_SHAPE,
                    "the backward's weight-gradient kernel takes D a multiple of 128; D=%d", d.D);
    if ((pg.M + kThlRows - 1) / kThlRows > 64)
        return fail(PTDIT_ERR_SHAPE, "the backward takes at most 8192 proxies; M=%d", pg.M);
    TRY(check_weights(psa, "psa"));
    TRY(check_weights(cross, "cross"));
    TRY(check_bwd_io(d, psa, z_in, dz_out, dz_in, ws, ws_bytes));
    TRY(check_bwd_io(d, cross, z_in, dz_out, dz_in, ws, ws_bytes));
    TRY(check_wgrad(d, dw_psa, "dw_psa", z_in, dz_out, dz_in, ws, ws_bytes));
    TRY(check_wgrad(d, dw_cross, "dw_cross", z_in, dz_out, dz_in, ws, ws_bytes));
    {
        const size_t gb = (size_t)d.D * d.D * sizeof(float);
        const float *a[4] = {dw_psa->dwq, dw_psa->dwk, dw_psa->dwv, dw_psa->dwo};
        const float *b[4] = {dw_cross->dwq, dw_cross->dwk, dw_cross->dwv, dw_cross->dwo};
        for (int i = 0; i < 4; ++i)
            for (int j = 0; j < 4; ++j)
                if (overlap(a[i], gb, b[j], gb))
                    return fail(PTDIT_ERR_ALIAS, "dw_psa and dw_cross overlap");
    }
    const WsGB Lb = ws_layout_giim_bwd(d, pg.M);
    TRY(check_bwd_ws(ws, ws_bytes, Lb.total));
    const Ws none{};
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), none};
    return run_giim_bwd(r, Lb, pg, psa, cross, flags, z_in, dz_out, dz_in, dw_psa, dw_cross);
}

size_t ptdit_tcm_bwd_workspace_bytes(const ptdit_shape *shape, const int window[3]) {
    Dims d;
    if (check_shape(shape, &d) != PTDIT_OK) return 0;
    const int zero[3] = {0, 0, 0};
    WinGeom wg;
    if (make_window(d, window, zero, &wg) != PTDIT_OK) return 0;
    return tcm_bwd_layout(d).total;
}

int ptdit_tcm_bwd(const ptdit_shape *shape, const int window[3], const int shift[3],
                  const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
                  const void *z_in, const void *dz_out, void *dz_in,
                  const ptdit_attn_wgrad *dw_wsa, const ptdit_attn_wgrad *dw_swsa, void *ws,
                  size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    WinGeom wg0, wg1;
    const int zero[3] = {0, 0, 0};
    TRY(check_shape(shape, &d));
    TRY(make_window(d, window, shift, &wg1));
    TRY(make_window(d, window, zero, &wg0));
    TRY(check_bwd_shape(d, wg0));
    TRY(check_weights(wsa, "wsa"));
    TRY(check_weights(swsa, "swsa"));
    TRY(check_bwd_io(d, wsa, z_in, dz_out, dz_in, ws, ws_bytes));
    TRY(check_bwd_io(d, swsa, z_in, dz_out, dz_in, ws, ws_bytes));
    TRY(check_wgrad(d, dw_wsa, "dw_wsa", z_in, dz_out, dz_in, ws, ws_bytes));
    TRY(check_wgrad(d, dw_swsa, "dw_swsa", z_in, dz_out, dz_in, ws, ws_bytes));
    {
        const size_t gb = (size_t)d.D * d.D * sizeof(float);
        const float *a[4] = {dw_wsa->dwq, dw_wsa->dwk, dw_wsa->dwv, dw_wsa->dwo};
        const float *b[4] = {dw_swsa->dwq, dw_swsa->dwk, dw_swsa->dwv, dw_swsa->dwo};
        for (int i = 0; i < 4; ++i)
            for (int j = 0; j < 4; ++j)
                if (overlap(a[i], gb, b[j], gb))
                    return fail(PTDIT_ERR_ALIAS, "dw_wsa and dw_swsa overlap");
    }
    TRY(check_bwd_ws(ws, ws_bytes, tcm_bwd_layout(d).total));
    return run_tcm_bwd(d, (cudaStream_t)stream, static_cast<char *>(ws), wg0, wg1, wsa, swsa, flags,
                       z_in, dz_out, dz_in, dw_wsa, dw_swsa);
}

int ptdit_tcm(const ptdit_shape *shape, const int window[3], const int shift[3],
              const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
              const void *z_in, void *z_out, void *ws, size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    WinGeom wg0, wg1;
    Ws L;
    const int zero[3] = {0, 0, 0};
    TRY(check_shape(shape, &d));
    TRY(make_window(d, window, shift, &wg1));
    TRY(make_window(d, window, zero, &wg0));
    TRY(check_bf16_attention(d, &wg0));
    TRY(check_weights(wsa, "wsa"));
    TRY(check_weights(swsa, "swsa"));
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    TRY(check_w_alias(d, wsa, z_out));
    TRY(check_w_alias(d, swsa, z_out));
    TRY(check_ws(d, 0, ws, ws_bytes, &L));
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), L};
    r.cap = ws_bytes;
    TRY(run_window(r, wg0, wsa, flags, z_in, z_out));
    return run_window(r, wg1, swsa, flags, z_out, z_out);
}

int ptdit_block_attn(const ptdit_shape *shape, const int ratio[3], const int window[3],
                     const int shift[3], const ptdit_attn_w *psa, const ptdit_attn_w *cross,
                     const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
                     const void *z_in, void *z_out, void *ws, size_t ws_bytes,
                     ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    WinGeom wg0, wg1;
    Ws L;
    const int zero[3] = {0, 0, 0};
    TRY(check_shape(shape, &d));
    TRY(make_proxy(d, ratio, &pg));
    TRY(make_window(d, window, shift, &wg1));
    TRY(make_window(d, window, zero, &wg0));
    TRY(check_bf16_attention(d, &wg0));
    TRY(check_weights(psa, "psa"));
    TRY(check_weights(cross, "cross"));
    TRY(check_weights(wsa, "wsa"));
    TRY(check_weights(swsa, "swsa"));
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    TRY(check_w_alias(d, psa, z_out));
    TRY(check_w_alias(d, cross, z_out));
    TRY(check_w_alias(d, wsa, z_out));
    TRY(check_w_alias(d, swsa, z_out));
    TRY(check_ws(d, pg.M, ws, ws_bytes, &L));
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), L};
    r.cap = ws_bytes;
    TRY(run_giim(r, pg, psa, cross, flags, z_in, z_out));
    TRY(run_window(r, wg0, wsa, flags, z_out, z_out));
    return run_window(r, wg1, swsa, flags, z_out, z_out);
}

int ptdit_window_fused(int enable) {
    const int prev = g_window_fused ? 1 : 0;
    if (enable == 0 || enable == 1) g_window_fused = enable == 1;
    return prev;
}

size_t ptdit_block_attn_bwd_workspace_bytes(const ptdit_shape *shape, const int ratio[3],
                                            const int window[3]) {
    Dims d;
    ProxyGeom pg;
    WinGeom wg;
    const int zero[3] = {0, 0, 0};
    if (check_shape(shape, &d) != PTDIT_OK || make_proxy(d, ratio, &pg) != PTDIT_OK ||
        make_window(d, window, zero, &wg) != PTDIT_OK)
        return 0;
    return block_bwd_layout(d, pg.M).total;
}

int ptdit_block_attn_bwd(const ptdit_shape *shape, const int ratio[3], const int window[3],
                         const int shift[3], const ptdit_attn_w *psa, const ptdit_attn_w *cross,
                         const ptdit_attn_w *wsa, const ptdit_attn_w *swsa, unsigned flags,
                         const void *z_in, const void *dz_out, void *dz_in,
                         const ptdit_attn_wgrad *dw_psa, const ptdit_attn_wgrad *dw_cross,
                         const ptdit_attn_wgrad *dw_wsa, const ptdit_attn_wgrad *dw_swsa, void *ws,
                         size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    WinGeom wg0, wg1;
    TRY(path_geometry(shape, ratio, window, shift, &d, &pg, &wg0, &wg1));
    const ptdit_attn_w *W[4] = {psa, cross, wsa, swsa};
    const ptdit_attn_wgrad *G[4] = {dw_psa, dw_cross, dw_wsa, dw_swsa};
    TRY(check_path_grads(d, W, G, z_in, dz_out, dz_in, ws, ws_bytes));
    const BlockBwd L = block_bwd_layout(d, pg.M);
    TRY(check_bwd_ws(ws, ws_bytes, L.total));
    const cudaStream_t s = (cudaStream_t)stream;
    char *base = static_cast<char *>(ws);
    void *z1 = base + L.z1, *dz1 = base + L.dz1;
    const Ws none{};
    const WsGB Lg = ws_layout_giim_bwd(d, pg.M);
    Run rg{d, s, base + L.giim, none};
    TRY(giim_recompute(rg, Lg, pg, psa, cross, flags, z_in, z1));
    TRY(run_tcm_bwd(d, s, base + L.tcm, wg0, wg1, wsa, swsa, flags, z1, dz_out, dz1, dw_wsa,
                    dw_swsa));
    return giim_backward(rg, Lg, pg, psa, cross, flags, z_in, dz1, dz_in, dw_psa, dw_cross);
}

size_t ptdit_block_attn_train_workspace_bytes(const ptdit_shape *shape, const int ratio[3],
                                              const int window[3]) {
    Dims d;
    ProxyGeom pg;
    WinGeom wg;
    const int zero[3] = {0, 0, 0};
    if (check_shape(shape, &d) != PTDIT_OK || make_proxy(d, ratio, &pg) != PTDIT_OK ||
        make_window(d, window, zero, &wg) != PTDIT_OK)
        return 0;
    return train_layout(d, pg.M).total;
}

int ptdit_block_attn_fwd_train(const ptdit_shape *shape, const int ratio[3], const int window[3],
                               const int shift[3], const ptdit_attn_w *psa,
                               const ptdit_attn_w *cross, const ptdit_attn_w *wsa,
                               const ptdit_attn_w *swsa, unsigned flags, const void *z_in,
                               void *z_out, void *ws, size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    WinGeom wg0, wg1;
    TRY(path_geometry(shape, ratio, window, shift, &d, &pg, &wg0, &wg1));
    const ptdit_attn_w *W[4] = {psa, cross, wsa, swsa};
    const char *wn[4] = {"psa", "cross", "wsa", "swsa"};
    for (int m = 0; m < 4; ++m) TRY(check_weights(W[m], wn[m]));
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    for (int m = 0; m < 4; ++m) TRY(check_w_alias(d, W[m], z_out));
    const TrainLayout T = train_layout(d, pg.M);
    TRY(check_bwd_ws(ws, ws_bytes, T.total));
    const cudaStream_t s = (cudaStream_t)stream;
    char *base = static_cast<char *>(ws), *tcm = base + T.b.tcm;
    const Ws none{};
    const WsGB Lg = ws_layout_giim_bwd(d, pg.M);
    Run rg{d, s, base + T.b.giim, none};
    void *z1 = base + T.b.z1;
    TRY(giim_recompute(rg, Lg, pg, psa, cross, flags, z_in, z1));
    const TcmBwd Tc = tcm_bwd_layout(d);
    void *zh = tcm + Tc.zh;
    Ws Lw{};  // WSA's Q, K, V and attention output stay where its backward reads them
    Lw.Q = Tc.wq; Lw.K = Tc.wk; Lw.V = Tc.wv; Lw.O = Tc.wa;
    Run rw{d, s, tcm, Lw};
    TRY(run_window(rw, wg0, wsa, flags, z1, zh, nullptr, 0.f, false));
    Ws Ls{};  // and SWSA's
    Ls.Q = T.sq; Ls.K = T.sk; Ls.V = T.sv; Ls.O = T.sa;
    Run rs{d, s, base, Ls};
    return run_window(rs, wg1, swsa, flags, zh, z_out, nullptr, 0.f, false);
}

int ptdit_block_attn_bwd_saved(const ptdit_shape *shape, const int ratio[3], const int window[3],
                               const int shift[3], const ptdit_attn_w *psa,
                               const ptdit_attn_w *cross, const ptdit_attn_w *wsa,
                               const ptdit_attn_w *swsa, unsigned flags, const void *z_in,
                               const void *dz_out, void *dz_in, const ptdit_attn_wgrad *dw_psa,
                               const ptdit_attn_wgrad *dw_cross, const ptdit_attn_wgrad *dw_wsa,
                               const ptdit_attn_wgrad *dw_swsa, void *ws, size_t ws_bytes,
                               ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    WinGeom wg0, wg1;
    TRY(path_geometry(shape, ratio, window, shift, &d, &pg, &wg0, &wg1));
    const ptdit_attn_w *W[4] = {psa, cross, wsa, swsa};
    const ptdit_attn_wgrad *G[4] = {dw_psa, dw_cross, dw_wsa, dw_swsa};
    TRY(check_path_grads(d, W, G, z_in, dz_out, dz_in, ws, ws_bytes));
    const TrainLayout T = train_layout(d, pg.M);
    TRY(check_bwd_ws(ws, ws_bytes, T.total));
    const cudaStream_t s = (cudaStream_t)stream;
    char *base = static_cast<char *>(ws), *tcm = base + T.b.tcm;
    void *z1 = base + T.b.z1, *dz1 = base + T.b.dz1;
    const TcmBwd Tc = tcm_bwd_layout(d);
    void *zh = tcm + Tc.zh, *dzh = tcm + Tc.dzh;
    const Ws none{};
    Run r{d, s, tcm, none};
    WsBwd Ls = Tc.bwd;  // SWSA's kept forward, outside TCM's area
    Ls.Q = T.sq - T.b.tcm; Ls.K = T.sk - T.b.tcm; Ls.V = T.sv - T.b.tcm; Ls.A = T.sa - T.b.tcm;
    TRY(run_window_bwd(r, Ls, wg1, swsa, flags, zh, dz_out, dzh, dw_swsa, false));
    WsBwd Lw = Tc.bwd;
    Lw.Q = Tc.wq; Lw.K = Tc.wk; Lw.V = Tc.wv; Lw.A = Tc.wa;
    TRY(run_window_bwd(r, Lw, wg0, wsa, flags, z1, dzh, dz1, dw_wsa, false));
    const WsGB Lg = ws_layout_giim_bwd(d, pg.M);
    Run rg{d, s, base + T.b.giim, none};
    return giim_backward(rg, Lg, pg, psa, cross, flags, z_in, dz1, dz_in, dw_psa, dw_cross);
}

size_t ptdit_pt_block_workspace_bytes(const ptdit_shape *shape, const int ratio[3],
                                      int text_len, int mlp_hidden) {
    Dims d;
    ProxyGeom pg;
    if (check_shape(shape, &d) != PTDIT_OK || text_len < 1 || mlp_hidden < 1) return 0;
    if (make_proxy(d, ratio, &pg) != PTDIT_OK) return 0;
    return ws_layout(d, pg.M, text_len, mlp_hidden).total_fused;
}

int ptdit_pt_block(const ptdit_shape *shape, const int ratio[3], const int window[3],
                   const int shift[3], const ptdit_block_w *w, const void *text, int text_len,
                   int proxy_mode, const int32_t *slots, const void *z_in, void *z_out, void *ws,
                   size_t ws_bytes, ptdit_stream_t stream) {
    Dims d;
    ProxyGeom pg;
    WinGeom wg0, wg1;
    Ws L;
    const int zero[3] = {0, 0, 0};
    TRY(check_shape(shape, &d));
    TRY(make_proxy(d, ratio, &pg));
    TRY(make_window(d, window, shift, &wg1));
    TRY(make_window(d, window, zero, &wg0));
    TRY(check_bf16_attention(d, &wg0));
    TRY(check_proxy_mode(proxy_mode, slots));
    if (!w) return fail(PTDIT_ERR_NULL, "block weights are NULL");
    const ptdit_attn_w *mods[5] = {&w->psa, &w->cross, &w->wsa, &w->swsa, &w->text};
    const char *names[5] = {"psa", "cross", "wsa", "swsa", "text"};
    for (int i = 0; i < 5; ++i) {
        TRY(check_weights(mods[i], names[i]));
        TRY(check_w_alias(d, mods[i], z_out));
    }
    const ptdit_norm_w *norms[6] = {&w->norm_proxy, &w->norm_cross, &w->norm_wsa,
                                    &w->norm_swsa, &w->norm_text, &w->norm_mlp};
    const size_t zb = (size_t)d.B * d.N * d.D * d.elem, vb = (size_t)d.D * d.elem;
    for (int i = 0; i < 6; ++i) {
        TRY(check_ptr(norms[i]->gamma, "norm gamma"));
        TRY(check_ptr(norms[i]->beta, "norm beta"));
        if (overlap(norms[i]->gamma, vb, z_out, zb) || overlap(norms[i]->beta, vb, z_out, zb))
            return fail(PTDIT_ERR_ALIAS, "z_out overlaps a norm parameter");
    }
    if (w->mlp_hidden < 1) return fail(PTDIT_ERR_SHAPE, "mlp_hidden %d < 1", w->mlp_hidden);
    if (d.dtype == PTDIT_BF16 && w->mlp_hidden % 16)
        return fail(PTDIT_ERR_SHAPE, "bf16 MLP widths must be multiples of 16 (mlp_hidden=%d)",
                    w->mlp_hidden);
    if (!(w->eps > 0.f) || w->eps > 1.f)
        return fail(PTDIT_ERR_SHAPE, "eps must be in (0, 1]");
    const size_t hb = (size_t)w->mlp_hidden * d.D * d.elem, bh = (size_t)w->mlp_hidden * d.elem;
    TRY(check_ptr(w->w1, "w1"));
    TRY(check_ptr(w->b1, "b1"));
    TRY(check_ptr(w->w2, "w2"));
    TRY(check_ptr(w->b2, "b2"));
    if (overlap(w->w1, hb, z_out, zb) || overlap(w->w2, hb, z_out, zb) ||
        overlap(w->b1, bh, z_out, zb) || overlap(w->b2, vb, z_out, zb))
        return fail(PTDIT_ERR_ALIAS, "z_out overlaps an MLP weight");
    if (text_len < 1) return fail(PTDIT_ERR_SHAPE, "text_len %d < 1", text_len);
    TRY(check_ptr(text, "text"));
    if (overlap(text, (size_t)d.B * text_len * d.D * d.elem, z_out, zb))
        return fail(PTDIT_ERR_ALIAS, "z_out overlaps the text tokens");
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    TRY(check_ws(d, pg.M, ws, ws_bytes, &L, text_len, w->mlp_hidden));
    if (ws && overlap(ws, ws_bytes, text, (size_t)d.B * text_len * d.D * d.elem))
        return fail(PTDIT_ERR_ALIAS, "the text tokens overlap the workspace");
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), L};
    r.cap = ws_bytes;
    const NormSet nm{norms[0], norms[1], norms[2], norms[3], norms[4], norms[5], w->eps};
    TRY(run_giim(r, pg, &w->psa, &w->cross, 0, z_in, z_out, proxy_mode, slots, &nm));
    TRY(run_window(r, wg0, &w->wsa, 0, z_out, z_out, nm.wsa, nm.eps));
    TRY(run_window(r, wg1, &w->swsa, 0, z_out, z_out, nm.swsa, nm.eps));
    TRY(run_text(r, &w->text, nm.text, nm.eps, text, text_len, z_out));
    return run_mlp(r, w, nm.eps, z_out);
}

int ptdit_full_attn(const ptdit_shape *shape, const ptdit_attn_w *w, unsigned flags,
                    const void *z_in, void *z_out, void *ws, size_t ws_bytes,
                    ptdit_stream_t stream) {
    Dims d;
    Ws L;
    TRY(check_shape(shape, &d));
    TRY(check_bf16_attention(d));
    TRY(check_weights(w, "w"));
    TRY(check_io(d, z_in, z_out, ws, ws_bytes));
    TRY(check_w_alias(d, w, z_out));
    TRY(check_ws(d, 0, ws, ws_bytes, &L));
    Run r{d, (cudaStream_t)stream, static_cast<char *>(ws), L};
    r.cap = ws_bytes;
    const long BN = (long)d.B * d.N;
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.mode = ATT_ROWS;
    a.dtype = d.dtype;
    a.d = d.d;
    a.q = r.at(L.Q); a.k = r.at(L.K); a.v = r.at(L.V); a.o = r.at(L.O);
    a.q_bstride = a.k_bstride = d.N;
    a.nq = a.nk = (int)d.N;
    const bool tiled = attention_thl_supported(a);
    const ThlDesc tn = thl_identity(d.N, 0), tnv = thl_identity(d.N, 1, v_ones(d));
    if (tiled) {
        a.tq = a.tk = tn;
        a.tv = tnv;
    }
    {
        const void *W[3] = {w->wq, w->wk, w->wv};
        void *C[3] = {r.at(L.Q), r.at(L.K), r.at(L.V)};
        const ThlDesc *T[3] = {tiled ? &tn : nullptr, tiled ? &tn : nullptr, tiled ? &tnv : nullptr};
        TRY(gemm_thl(r, PTDIT_K_GEMM, z_in, BN, 3, W, C, T, "QKV projection"));
    }
    TRY(attention(r, PTDIT_K_ATTN_DENSE, a, "full self-attention"));
    {
        const void *W[3] = {w->wo, nullptr, nullptr};
        void *C[3] = {z_out, nullptr, nullptr};
        const void *R[3] = {(flags & PTDIT_NO_RESIDUAL) ? nullptr : z_in, nullptr, nullptr};
        TRY(gemm(r, PTDIT_K_GEMM, r.at(L.O), BN, 1, W, C, R, "output projection"));
    }
    return PTDIT_OK;
}

int ptdit_debug_proxy_map(const int grid[3], const int ratio[3], int32_t *proxy_of_token,
                          ptdit_stream_t stream) {
    if (!grid) return fail(PTDIT_ERR_NULL, "grid is NULL");
    ptdit_shape sh = {1, grid[0], grid[1], grid[2], 1, 1, PTDIT_F32};
    Dims d;
    ProxyGeom pg;
    TRY(check_shape(&sh, &d));
    TRY(make_proxy(d, ratio, &pg));
    if (!proxy_of_token) return fail(PTDIT_ERR_NULL, "proxy_of_token is NULL");
    cudaError_t e = launch_debug_proxy_map(pg, proxy_of_token, (cudaStream_t)stream);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, "proxy map");
}

int ptdit_debug_window_map(const int grid[3], const int window[3], const int shift[3],
                           int32_t *token_at_slot, uint8_t *allowed, ptdit_stream_t stream) {
    if (!grid) return fail(PTDIT_ERR_NULL, "grid is NULL");
    ptdit_shape sh = {1, grid[0], grid[1], grid[2], 1, 1, PTDIT_F32};
    Dims d;
    WinGeom wg;
    TRY(check_shape(&sh, &d));
    TRY(make_window(d, window, shift, &wg));
    if (!token_at_slot) return fail(PTDIT_ERR_NULL, "token_at_slot is NULL");
    cudaError_t e = launch_debug_window_map(wg, token_at_slot, allowed, (cudaStream_t)stream);
    count_launch();
    return e == cudaSuccess ? PTDIT_OK : cuda_fail(e, "window map");
}

int ptdit_debug_thl_map(const int grid[3], const int window[3], const int shift[3], int windowed,
                        int32_t *row_of_token, int32_t *token_of_row, int *tiles) {
    if (!grid) return fail(PTDIT_ERR_NULL, "grid is NULL");
    if (!tiles) return fail(PTDIT_ERR_NULL, "tiles is NULL");
    ptdit_shape sh = {1, grid[0], grid[1], grid[2], 1, 1, PTDIT_F32};
    Dims d;
    TRY(check_shape(&sh, &d));
    ThlDesc t;
    if (windowed) {
        WinGeom wg;
        TRY(make_window(d, window, shift, &wg));
        if (wg.n > kThlRows || kThlRows % wg.n)
            return fail(PTDIT_ERR_SHAPE, "windows of %d tokens do not pack into %d-row tiles", wg.n,
                        kThlRows);
        t = thl_window(wg, d.N, 0);
    } else {
        t = thl_identity(d.N, 0);
    }
    *tiles = t.tiles;
    if (row_of_token)
        for (long tok = 0; tok < d.N; ++tok) {
            int tile, r;
            thl_locate(t, tok, tile, r);
            row_of_token[tok] = tile * kThlRows + r;
        }
    if (token_of_row)
        for (int tile = 0; tile < t.tiles; ++tile)
            for (int r = 0; r < kThlRows; ++r)
                token_of_row[tile * kThlRows + r] = static_cast<int32_t>(thl_token(t, tile, r));
    return PTDIT_OK;
}

int ptdit_debug_thl_units(int d, int vpad, uint32_t *offset, int *units, int *block_bytes) {
    if (!units || !block_bytes) return fail(PTDIT_ERR_NULL, "units or block_bytes is NULL");
    if (d < 8 || d > 80 || d % 8)
        return fail(PTDIT_ERR_SHAPE, "head width %d: the tiled layout holds 8 .. 80, multiples of 8", d);
    const int vp = vpad && d > 64;
    *units = thl_units(d, vp);
    *block_bytes = static_cast<int>(thl_block_bytes(d, vp));
    if (offset)
        for (int r = 0; r < kThlRows; ++r)
            for (int p = 0; p < *units; ++p) offset[r * *units + p] = thl_unit(r, p, vp);
    return PTDIT_OK;
}

int ptdit_debug_gemm_schedule(long rows, int nseg, int nmat, int pairs, int32_t *first,
                              int32_t *tile, int *tiles, int *scheduled) {
    if (!tiles || !scheduled) return fail(PTDIT_ERR_NULL, "tiles or scheduled is NULL");
    if (gemm_tc2_schedule(rows, nseg, nmat, pairs, first, tile, tiles, scheduled) != 0)
        return fail(PTDIT_ERR_SHAPE, "no projection launch takes rows %ld, nseg %d, nmat %d, %d pairs",
                    rows, nseg, nmat, pairs);
    return PTDIT_OK;
}

}  // extern "C"
