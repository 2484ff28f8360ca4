// Attention core on the 5th-generation tensor cores for operands in plain
// row-major layout (head widths whose operands are not tiled, e.g. 56), and
// the dispatch: operands in tiled head layout go to the warp-specialised
// kernels of attn_rows_tc.cu (proxy SA, cross-attention, full SA) and
// attn_win_tc.cu (window and shifted-window SA).
//
// Qihoo-T2X reading note, §3 Method: Eq. GIIM (SA among the proxies, CS with
// every latent the query and the proxies keys/values) and Eq. TCM (WSA, and
// SWSA on the grid rolled by -s with the wrapped pairs masked).
//
// One CTA = one 128-row query tile x one head, 8 warps: thread t serves query
// row t % 128 (its TMEM lane) and half t / 128 of that row's keys and output
// columns.  Three CTAs fit on an SM, so one CTA's softmax overlaps another's
// loads and MMAs.
//   * Rows are gathered with 16-byte cp.async straight from the [rows, D]
//     projection outputs: head h is columns h*d .. h*d+d-1, and in window mode
//     the row of each slot comes from the roll/gather address function, so no
//     window or head copy is ever materialised.
//   * Q, K, V and P sit in shared memory in one layout, 16-byte chunks
//     major: byte (chunk c, row r) = c * 2048 + r * 16.  That is the
//     no-swizzle core-matrix layout of tcgen05: K-major for Q, K and P, and
//     MN-major for V, so P V needs no transpose.  d is zero-padded to a
//     multiple of 16 (72 -> 80).  P overwrites K once S is computed.
//   * S = Q K^T (128 x 128, fp32) accumulates in TMEM.  The key mask is built
//     once per tile with warp ballots (one 128-bit mask per mask key: window
//     in tile and wrap bits, or "key exists"); each thread then runs the
//     online softmax over its half of the row's own window in fp32 (row max
//     and sum combined across the two halves through shared memory) and
//     writes P as bf16; P V (128 x dpad) reuses S's TMEM columns and is added
//     to the thread's fp32 output columns in registers with the rescale.
//   * 2D windows of 64 tokens are packed two per tile (block-diagonal mask;
//     each row visits only its own window's keys); 3D windows of 128 tokens
//     are one tile; larger windows and long key sets stream key tiles.
// Every mbarrier wait is bounded (2 s) and reports PTDIT_ERR_TIMEOUT.
#include <math.h>

#include "tc_util.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128, BKV = 128, kThreads = 256;
constexpr uint32_t CHUNK = BQ * 16;  // bytes between 16-byte chunk columns (2048)
constexpr uint32_t kTmemCols = 128;
constexpr int kMaxKeys = 16;  // distinct mask keys per tile (2 windows x 8 wrap codes)

template <int DPAD>
struct AttnLayout {
    static constexpr int TILE = BQ * DPAD * 2;  // one Q, K or V tile
    static constexpr int P_BYTES = BQ * BKV * 2;
    static constexpr int KP = TILE > P_BYTES ? TILE : P_BYTES;  // K, then P over it
    static constexpr int OFF_Q = 0, OFF_K = TILE, OFF_V = TILE + KP;
    static constexpr int OFF_KMASK = OFF_V + TILE;            // uint32[kMaxKeys][4]
    static constexpr int OFF_RED = OFF_KMASK + kMaxKeys * 16; // float[2][2][128]
    static constexpr int OFF_BAR = OFF_RED + 4 * BQ * 4;
    static constexpr int BYTES = OFF_BAR + 64;  // bar_s, bar_o, drain, tmem slot, abort
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct Slot {
    long row;  // row index into q/k/v/o, or -1 for an empty slot
    int info;  // mask key: window-in-tile * 8 + wrap bits (window mode), 0 (rows), -1 empty
};

// Slot `r` (0..127) of a query tile, or of key tile `kt` of that query tile.
__device__ __forceinline__ Slot slot_of(const AttnArgs &a, int b, int tile, int r, int kt,
                                        bool key) {
    Slot s{-1, -1};
    if (a.mode == ATT_WINDOW) {
        const WinGeom &g = a.geom;
        int win, slot, wit;
        if (g.n <= BQ) {
            const int pack = BQ / g.n;
            wit = fdiv(g.f_n, r);
            win = tile * pack + wit;
            slot = r - wit * g.n;
            if (win >= g.nwin) return s;
        } else {
            const int per = g.n / BQ;
            win = tile / per;
            wit = 0;
            slot = (key ? kt : tile % per) * BQ + r;
        }
        int wrap;
        const int tok = window_token(g, win, slot, &wrap);
        s.row = (long)b * (key ? a.k_bstride : a.q_bstride) + tok;
        s.info = wit * 8 + wrap;
    } else {
        const int j = (key ? kt : tile) * BQ + r;
        if (j < (key ? a.nk : a.nq)) {
            s.row = (long)b * (key ? a.k_bstride : a.q_bstride) + j;
            s.info = 0;
        }
    }
    return s;
}

__device__ __forceinline__ bool wait_and_fence(uint64_t *bar, uint32_t parity,
                                               volatile int *abort, int *status) {
    const bool ok = mbar_wait(bar, parity, abort, status);
    fence_before_sync();
    return ok;
}

// 16-byte chunks [c0, c1) of one row into a chunk-major tile (zero-fill for an empty slot).
__device__ __forceinline__ void load_row(uint8_t *tile, const __nv_bfloat16 *base, long ld,
                                         long row, int c0, int c1, int r) {
    const __nv_bfloat16 *src = base + (row >= 0 ? row : 0) * ld;
    const uint32_t bytes = row >= 0 ? 16 : 0;
    for (int c = c0; c < c1; ++c) cp_async16(tile + c * CHUNK + r * 16, src + c * 8, bytes);
}

template <int DPAD>
__global__ void __launch_bounds__(kThreads, 3) attn_tc_kernel(AttnArgs a, int n_ktiles, int nkeys,
                                                                int *status) {
    using L = AttnLayout<DPAD>;
    constexpr int NCH = DPAD / 8, HALF = DPAD / 2;
    extern __shared__ __align__(16) uint8_t sm[];
    uint8_t *sQ = sm + L::OFF_Q, *sK = sm + L::OFF_K, *sV = sm + L::OFF_V, *sP = sm + L::OFF_K;
    uint32_t *kmask = reinterpret_cast<uint32_t *>(sm + L::OFF_KMASK);
    float *red_max = reinterpret_cast<float *>(sm + L::OFF_RED);  // [2][128]
    float *red_sum = red_max + 2 * BQ;                             // [2][128]
    uint64_t *bar_s = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *bar_o = bar_s + 1;
    uint64_t *drain = bar_s + 2;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_s + 3);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int t = threadIdx.x, warp = t / 32, lane = t % 32;
    const int r = t % BQ, hf = t / BQ;  // query row (= TMEM lane) and half
    const int h = blockIdx.x, tile = blockIdx.y, b = blockIdx.z;
    const int d = a.d, nch = d / 8;
    const int lc0 = hf ? (nch + 1) / 2 : 0, lc1 = hf ? nch : (nch + 1) / 2;  // chunks I load
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q) + (long)h * d;
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k) + (long)h * d;
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(a.v) + (long)h * d;
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o) + (long)h * d;

    if (t == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    // zero the padded chunks of Q and V once (K's may later hold P: Q's zeros
    // cancel whatever finite values sit there)
    if (hf == 0)
        for (int c = nch; c < NCH; ++c) {
            *reinterpret_cast<uint4 *>(sQ + c * CHUNK + r * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sK + c * CHUNK + r * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sV + c * CHUNK + r * 16) = make_uint4(0, 0, 0, 0);
        }

    const Slot q = slot_of(a, b, tile, r, 0, false);
    const int qi = q.info;
    load_row(sQ, qg, a.ldq, q.row, lc0, lc1, r);
    // the row's own key columns, split between the two halves
    int c_lo = 0, c_hi = BKV;
    if (a.mode == ATT_WINDOW && a.geom.n < BQ) {
        c_lo = (r / a.geom.n) * a.geom.n;
        c_hi = c_lo + a.geom.n;
    }
    const int a0 = c_lo + hf * ((c_hi - c_lo) / 2), a1 = a0 + (c_hi - c_lo) / 2;

    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t t_row = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const float sl2 = a.scale * 1.4426950408889634f;  // scores in the log2 domain

    float m_i = -INFINITY, l_i = 0.f;
    float o[HALF];
#pragma unroll
    for (int i = 0; i < HALF; ++i) o[i] = 0.f;
    uint32_t phase = 0;
    bool ok = true;

    for (int kt = 0; kt < n_ktiles && ok; ++kt) {
        // ---- K and V rows of this key tile
        const Slot k = slot_of(a, b, tile, r, kt, true);
        load_row(sK, kg, a.ldk, k.row, lc0, lc1, r);
        load_row(sV, vg, a.ldv, k.row, lc0, lc1, r);
        cp_async_commit();
        cp_async_wait_all();
        fence_async_smem();
        __syncthreads();

        // ---- S = Q K^T (tensor core) while warps 0-3 build the key masks
        if (t == 0) {
            fence_after_sync();
            constexpr uint32_t idesc = idesc_bf16(BQ, BKV);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
#pragma unroll
            for (int ks = 0; ks < DPAD / 16; ++ks)
                mma_bf16(tmem, sdesc_interleave(aQ + ks * 2 * CHUNK, CHUNK, 128),
                         sdesc_interleave(aK + ks * 2 * CHUNK, CHUNK, 128), idesc, ks > 0);
            mma_commit(bar_s);
        }
        if (hf == 0)
            for (int v = 0; v < nkeys; ++v) {
                const uint32_t bits = __ballot_sync(0xffffffffu, k.info == v);
                if (lane == 0) kmask[v * 4 + warp] = bits;
            }
        // one thread waits; the barrier hands its verdict (and the tcgen05
        // completion it observed) to the whole CTA
        ok = __syncthreads_and(t == 0 ? wait_and_fence(bar_s, phase, abort, status) : true);
        if (!ok) break;
        fence_after_sync();

        uint32_t allow[4] = {0u, 0u, 0u, 0u};
        if (qi >= 0) {
            const uint4 w4 = *reinterpret_cast<const uint4 *>(kmask + qi * 4);
            allow[0] = w4.x;
            allow[1] = w4.y;
            allow[2] = w4.z;
            allow[3] = w4.w;
        }

        // ---- pass 1: this half's row max
        float tmax = -INFINITY;
#pragma unroll 1
        for (int c0 = a0; c0 < a1; c0 += 16) {
            uint32_t sc[16];
            tmem_ld16(t_row + c0, sc);
            tmem_ld_wait();
            const uint32_t w = allow[c0 >> 5] >> (c0 & 16);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if ((w >> j) & 1u) tmax = fmaxf(tmax, __uint_as_float(sc[j]));
        }
        red_max[hf * BQ + r] = tmax;
        __syncthreads();
        const float m_tile = fmaxf(red_max[r], red_max[BQ + r]) * sl2;
        const float m_new = fmaxf(m_i, m_tile);
        const float ref = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = m_i == -INFINITY ? 0.f : ex2_approx(m_i - ref);

        // ---- pass 2: P = exp2(S * scale * log2 e - max), bf16, over K's buffer
        float psum = 0.f;
#pragma unroll 1
        for (int c0 = a0; c0 < a1; c0 += 16) {
            uint32_t sc[16];
            tmem_ld16(t_row + c0, sc);
            tmem_ld_wait();
            const uint32_t w = allow[c0 >> 5] >> (c0 & 16);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float pv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = 8 * g + e;
                    pv[e] = ((w >> j) & 1u) ? ex2_approx(fmaf(__uint_as_float(sc[j]), sl2, -ref))
                                            : 0.f;
                }
                uint4 v;
                v.x = pack_bf16(pv[0], pv[1]);
                v.y = pack_bf16(pv[2], pv[3]);
                v.z = pack_bf16(pv[4], pv[5]);
                v.w = pack_bf16(pv[6], pv[7]);
                // the row sum uses the bf16 values the MMA will see
                const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(hv[e]);
                    psum += f.x + f.y;
                }
                *reinterpret_cast<uint4 *>(sP + ((c0 >> 3) + g) * CHUNK + r * 16) = v;
            }
        }
        // zeros for this half's P columns that lie outside the row's window
        for (int c = hf * 8; c < hf * 8 + 8; ++c)
            if (c * 8 < c_lo || c * 8 >= c_hi)
                *reinterpret_cast<uint4 *>(sP + c * CHUNK + r * 16) = make_uint4(0, 0, 0, 0);
        red_sum[hf * BQ + r] = psum;
        fence_before_sync();
        fence_async_smem();
        __syncthreads();
        l_i = l_i * alpha + red_sum[r] + red_sum[BQ + r];
        m_i = m_new;

        // ---- PV = P V into S's TMEM columns
        if (t == 0) {
            fence_after_sync();
            constexpr uint32_t idesc = idesc_bf16(BQ, DPAD, true);
            const uint32_t aP = smem_u32(sP), aV = smem_u32(sV);
#pragma unroll
            for (int ks = 0; ks < BKV / 16; ++ks)
                mma_bf16(tmem, sdesc_interleave(aP + ks * 2 * CHUNK, CHUNK, 128),
                         sdesc_interleave(aV + ks * 256, 128, CHUNK), idesc, ks > 0);
            mma_commit(bar_o);
        }
        ok = __syncthreads_and(t == 0 ? wait_and_fence(bar_o, phase, abort, status) : true);
        if (!ok) break;
        fence_after_sync();
        {
            const uint32_t base = t_row + hf * HALF;
            if constexpr (HALF >= 32) {
                uint32_t v32[32];
                tmem_ld32(base, v32);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = o[j] * alpha + __uint_as_float(v32[j]);
            }
            if constexpr (HALF % 32 == 8) {
                uint32_t v8[8];
                tmem_ld8(base + (HALF / 32) * 32, v8);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    o[(HALF / 32) * 32 + j] = o[(HALF / 32) * 32 + j] * alpha + __uint_as_float(v8[j]);
            }
        }
        fence_before_sync();
        __syncthreads();  // TMEM, K/P and V are free for the next key tile
        phase ^= 1;
    }

    if (ok && q.row >= 0) {
        const float inv = 1.f / l_i;
        __nv_bfloat16 *dst = og + q.row * a.ldo + hf * HALF;
#pragma unroll
        for (int c = 0; c < HALF / 8; ++c) {
            if (hf * (HALF / 8) + c < nch) {
                uint4 v;
                v.x = pack_bf16(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
                v.y = pack_bf16(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
                v.z = pack_bf16(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
                v.w = pack_bf16(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
                *reinterpret_cast<uint4 *>(dst + c * 8) = v;
            }
        }
    }
    cp_async_wait_all();
    // a CTA that gave up waits (bounded) for its MMAs before releasing TMEM
    if (!ok && t == 0) {
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, status);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int DPAD>
cudaError_t launch_dpad(const AttnArgs &a, cudaStream_t s) {
    using L = AttnLayout<DPAD>;
    int *status = device_status_ptr();
    if (!status) return cudaErrorInvalidValue;
    int tiles, n_ktiles, nkeys;
    if (a.mode == ATT_WINDOW) {
        const WinGeom &g = a.geom;
        tiles = g.n <= BQ ? (g.nwin + BQ / g.n - 1) / (BQ / g.n) : g.nwin * (g.n / BQ);
        n_ktiles = g.n <= BQ ? 1 : g.n / BQ;
        nkeys = (g.n < BQ ? BQ / g.n : 1) * 8;
    } else {
        tiles = (a.nq + BQ - 1) / BQ;
        n_ktiles = (a.nk + BKV - 1) / BKV;
        nkeys = 1;
    }
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DPAD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(a.heads, tiles, a.B);
    attn_tc_kernel<DPAD><<<grid, kThreads, L::BYTES, s>>>(a, n_ktiles, nkeys, status);
    return cudaGetLastError();
}

int dpad_of(int d) { return (d + 15) / 16 * 16; }

}  // namespace

bool attention_tc_supported(const AttnArgs &a) {
    if (a.dtype != DT_BF16 || a.d % 8) return false;
    const int dp = dpad_of(a.d);
    if (dp != 64 && dp != 80) return false;
    if (a.ldq % 8 || a.ldk % 8 || a.ldv % 8 || a.ldo % 8) return false;
    if ((uintptr_t)a.q % 16 || (uintptr_t)a.k % 16 || (uintptr_t)a.v % 16 || (uintptr_t)a.o % 16)
        return false;
    if (a.mode == ATT_WINDOW) {  // windows of 64, 128 or a multiple of 128 tokens
        const int n = a.geom.n;
        return n == 64 || n % BQ == 0;
    }
    return a.nq >= 1 && a.nk >= 1;
}

// Operands in tiled head layout (head width 64..80): the warp-specialised
// row kernel (proxy SA, cross-attention, full SA) and window kernel.
bool attention_thl_supported(const AttnArgs &a) {
    if (a.dtype != DT_BF16 || a.d < 64 || a.d > 80 || a.d % 8) return false;
    if (a.mode == ATT_WINDOW)
        return (a.geom.n == 64 || a.geom.n == 128) && a.q_bstride == a.k_bstride;
    return a.nq >= 1 && a.nk >= 1;
}

cudaError_t launch_attention_rows_tc(const AttnArgs &a, cudaStream_t s);
cudaError_t launch_attention_win_tc(const AttnArgs &a, cudaStream_t s);

cudaError_t launch_attention_tc(const AttnArgs &a, cudaStream_t s) {
    if (a.tq.mode != 0)
        return a.mode == ATT_ROWS ? launch_attention_rows_tc(a, s) : launch_attention_win_tc(a, s);
    switch (dpad_of(a.d)) {  // row-major operands: the per-tile kernel above
        case 64: return launch_dpad<64>(a, s);
        case 80: return launch_dpad<80>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ptdit
