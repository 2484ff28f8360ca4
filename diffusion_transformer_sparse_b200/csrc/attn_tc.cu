// Attention core on the 5th-generation tensor cores: window / shifted-window
// self-attention (TCM), proxy self-attention and latent -> proxy
// cross-attention (GIIM), and full self-attention (the dense comparator).
//
// Qihoo-T2X reading note, §3 Method: Eq. GIIM (SA among the proxies, CS with
// every latent the query and the proxies keys/values) and Eq. TCM (WSA, and
// SWSA on the grid rolled by -s with the wrapped pairs masked).
//
// One CTA = one 128-row query tile x one head (4 warps, thread r owns row r).
//   * Rows are gathered with 16-byte cp.async straight from the [rows, D]
//     projection outputs: head h is columns h*d .. h*d+d-1, and in window mode
//     the row of each slot comes from the roll/gather address function, so no
//     window or head copy is ever materialised.
//   * Q, K, V and P sit in shared memory in one layout, 16-byte chunks
//     major: byte (chunk c, row r) = c * 2048 + r * 16.  That is the
//     no-swizzle core-matrix layout of tcgen05: K-major for Q, K and P, and
//     MN-major for V, so P V needs no transpose.  d is zero-padded to a
//     multiple of 16 (72 -> 80).
//   * S = Q K^T (128 x 128, fp32) accumulates in TMEM; each thread reads its
//     row with tcgen05.ld, applies the mask (window membership and equal wrap
//     bits, or the ragged key tail), runs the online softmax in fp32 and
//     writes P as bf16; P V (128 x dpad) accumulates in TMEM and is added to
//     the thread's fp32 output row in registers with the softmax rescale.
//   * 2D windows of 64 tokens are packed two per tile (block-diagonal mask);
//     3D windows of 128 tokens are one tile.
// Every mbarrier wait is bounded (2 s) and reports PTDIT_ERR_TIMEOUT.
#include <math.h>

#include "tc_util.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128, BKV = 128, kThreads = 128;
constexpr uint32_t CHUNK = BQ * 16;  // bytes between 16-byte chunk columns (2048)
constexpr uint32_t kTmemCols = 256;

template <int DPAD>
struct AttnLayout {
    static constexpr int TILE = BQ * DPAD * 2;  // Q, K or V tile bytes
    static constexpr int P_BYTES = BQ * BKV * 2;
    static constexpr int OFF_Q = 0, OFF_K = TILE, OFF_V = 2 * TILE, OFF_P = 3 * TILE;
    static constexpr int OFF_QROW = OFF_P + P_BYTES;
    static constexpr int OFF_KROW = OFF_QROW + BQ * 8;
    static constexpr int OFF_QINFO = OFF_KROW + BKV * 8;
    static constexpr int OFF_KINFO = OFF_QINFO + BQ * 4;
    static constexpr int OFF_BAR = OFF_KINFO + BKV * 4;
    static constexpr int BYTES = OFF_BAR + 4 * 8 + 16;  // bar_s, bar_o, drain, tmem slot, abort
    static constexpr int ALLOC = BYTES + 128;
};

// Row index (or -1) and mask key of slot `slot` of the query / key set.
// info: window-in-tile * 8 + wrap bits (window mode), 0 (row mode), -1 empty.
struct Slot {
    long row;
    int info;
};

__device__ __forceinline__ Slot window_slot(const AttnArgs &a, int b, int tile, int slot_in_tile,
                                            int key_tile) {
    const WinGeom &g = a.geom;
    Slot s{-1, -1};
    int win, slot, wit;
    if (g.n <= BQ) {
        const int pack = BQ / g.n;
        wit = slot_in_tile / g.n;
        win = tile * pack + wit;
        slot = slot_in_tile % g.n;
        if (win >= g.nwin) return s;
    } else {
        const int per = g.n / BQ;
        win = tile / per;
        wit = 0;
        slot = (key_tile >= 0 ? key_tile : tile % per) * BQ + slot_in_tile;
    }
    int wrap;
    const int tok = window_token(g, win, slot, &wrap);
    s.row = (long)b * a.k_bstride + tok;
    s.info = wit * 8 + wrap;
    return s;
}

template <int DPAD>
__global__ void __launch_bounds__(kThreads) attn_tc_kernel(AttnArgs a, int *status) {
    using L = AttnLayout<DPAD>;
    constexpr int NCH = DPAD / 8;
    extern __shared__ uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 127) &
                                              ~static_cast<uintptr_t>(127));
    uint8_t *sQ = sm + L::OFF_Q, *sK = sm + L::OFF_K, *sV = sm + L::OFF_V, *sP = sm + L::OFF_P;
    long *krow = reinterpret_cast<long *>(sm + L::OFF_KROW);
    int *qinfo = reinterpret_cast<int *>(sm + L::OFF_QINFO);
    int *kinfo = reinterpret_cast<int *>(sm + L::OFF_KINFO);
    uint64_t *bar_s = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *bar_o = bar_s + 1;
    uint64_t *drain = bar_s + 2;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar_s + 3);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int tid = threadIdx.x, warp = tid / 32;
    const int h = blockIdx.x, tile = blockIdx.y, b = blockIdx.z;
    const int d = a.d, nch = d / 8;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q) + (long)h * d;
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k) + (long)h * d;
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(a.v) + (long)h * d;
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o) + (long)h * d;

    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);

    // zero the padded chunks of Q, K and V once; loads never touch them
    for (int c = nch; c < NCH; ++c) {
        *reinterpret_cast<uint4 *>(sQ + c * CHUNK + tid * 16) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sK + c * CHUNK + tid * 16) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sV + c * CHUNK + tid * 16) = make_uint4(0, 0, 0, 0);
    }

    // this thread's query row
    long qrow;
    int qi;
    int n_ktiles;
    if (a.mode == ATT_WINDOW) {
        Slot s = window_slot(a, b, tile, tid, -1);
        qrow = s.row >= 0 ? s.row - (long)b * a.k_bstride + (long)b * a.q_bstride : -1;
        qi = s.info;
        n_ktiles = a.geom.n <= BQ ? 1 : a.geom.n / BQ;
    } else {
        const int r = tile * BQ + tid;
        qrow = r < a.nq ? (long)b * a.q_bstride + r : -1;
        qi = r < a.nq ? 0 : -1;
        n_ktiles = (a.nk + BKV - 1) / BKV;
    }
    qinfo[tid] = qi;
    {
        const __nv_bfloat16 *src = qg + (qrow >= 0 ? qrow : 0) * a.ldq;
        const uint32_t bytes = qrow >= 0 ? 16 : 0;
        for (int c = 0; c < nch; ++c) cp_async16(sQ + c * CHUNK + tid * 16, src + c * 8, bytes);
    }

    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t t_s = tmem + (static_cast<uint32_t>(warp * 32) << 16);  // S: columns 0..127
    const uint32_t t_o = t_s + BKV;                                        // PV: columns 128..
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
    const float sl2 = a.scale * 1.4426950408889634f;  // scores in the log2 domain

    float m_i = -INFINITY, l_i = 0.f;
    float o[DPAD];
#pragma unroll
    for (int i = 0; i < DPAD; ++i) o[i] = 0.f;
    uint32_t phase = 0;
    bool ok = true;

    for (int kt = 0; kt < n_ktiles && ok; ++kt) {
        // ---- K and V rows of this key tile
        long kr;
        int ki;
        if (a.mode == ATT_WINDOW) {
            Slot s = window_slot(a, b, tile, tid, a.geom.n <= BQ ? -1 : kt);
            kr = s.row;
            ki = s.info;
        } else {
            const int j = kt * BKV + tid;
            kr = j < a.nk ? (long)b * a.k_bstride + j : -1;
            ki = j < a.nk ? 0 : -1;
        }
        kinfo[tid] = ki;
        {
            const long r = kr >= 0 ? kr : 0;
            const uint32_t bytes = kr >= 0 ? 16 : 0;
            for (int c = 0; c < nch; ++c) {
                cp_async16(sK + c * CHUNK + tid * 16, kg + r * a.ldk + c * 8, bytes);
                cp_async16(sV + c * CHUNK + tid * 16, vg + r * a.ldv + c * 8, bytes);
            }
        }
        cp_async_commit();
        cp_async_wait_all();
        fence_async_smem();
        __syncthreads();

        // ---- S = Q K^T
        if (tid == 0) {
            fence_after_sync();
            constexpr uint32_t idesc = idesc_bf16(BQ, BKV);
#pragma unroll
            for (int ks = 0; ks < DPAD / 16; ++ks)
                mma_bf16(tmem, sdesc_interleave(aQ + ks * 2 * CHUNK, CHUNK, 128),
                         sdesc_interleave(aK + ks * 2 * CHUNK, CHUNK, 128), idesc, ks > 0);
            mma_commit(bar_s);
        }
        // the decision to go on is the same for every thread of the CTA
        ok = __syncthreads_and(mbar_wait(bar_s, phase, abort, status));
        if (!ok) break;
        fence_after_sync();

        // ---- masked online softmax of row tid (two passes over TMEM)
        float tmax = -INFINITY;
#pragma unroll 1
        for (int c0 = 0; c0 < BKV; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(t_s + c0, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int kj = kinfo[c0 + j];
                if (kj >= 0 && kj == qi) tmax = fmaxf(tmax, __uint_as_float(r[j]) * sl2);
            }
        }
        const float m_new = fmaxf(m_i, tmax);
        const float ref = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = m_i == -INFINITY ? 0.f : exp2f(m_i - ref);
        float psum = 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < BKV; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(t_s + c0, r);
            tmem_ld_wait();
            float pv[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int kj = kinfo[c0 + j];
                const float p = (kj >= 0 && kj == qi) ? exp2f(__uint_as_float(r[j]) * sl2 - ref) : 0.f;
                pv[j] = p;
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint4 v;
                v.x = pack_bf16(pv[8 * g + 0], pv[8 * g + 1]);
                v.y = pack_bf16(pv[8 * g + 2], pv[8 * g + 3]);
                v.z = pack_bf16(pv[8 * g + 4], pv[8 * g + 5]);
                v.w = pack_bf16(pv[8 * g + 6], pv[8 * g + 7]);
                // the row sum uses the bf16 values the MMA will see
                const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(hv[e]);
                    psum += f.x + f.y;
                }
                *reinterpret_cast<uint4 *>(sP + ((c0 >> 3) + g) * CHUNK + tid * 16) = v;
            }
        }
        l_i = l_i * alpha + psum;
        m_i = m_new;
        fence_before_sync();
        fence_async_smem();
        __syncthreads();

        // ---- PV = P V
        if (tid == 0) {
            fence_after_sync();
            constexpr uint32_t idesc = idesc_bf16(BQ, DPAD, true);
#pragma unroll
            for (int ks = 0; ks < BKV / 16; ++ks)
                mma_bf16(tmem + BKV, sdesc_interleave(aP + ks * 2 * CHUNK, CHUNK, 128),
                         sdesc_interleave(aV + ks * 256, 128, CHUNK), idesc, ks > 0);
            mma_commit(bar_o);
        }
        ok = __syncthreads_and(mbar_wait(bar_o, phase, abort, status));
        if (!ok) break;
        fence_after_sync();
#pragma unroll
        for (int c0 = 0; c0 < DPAD; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(t_o + c0, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) o[c0 + j] = o[c0 + j] * alpha + __uint_as_float(r[j]);
        }
        fence_before_sync();
        __syncthreads();  // S, P, K and V are free for the next key tile
        phase ^= 1;
    }

    if (ok && qrow >= 0) {
        const float inv = 1.f / l_i;
        __nv_bfloat16 *dst = og + qrow * a.ldo;
#pragma unroll
        for (int c = 0; c < DPAD / 8; ++c) {
            if (c < nch) {
                uint4 v;
                v.x = pack_bf16(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
                v.y = pack_bf16(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
                v.z = pack_bf16(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
                v.w = pack_bf16(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
                *reinterpret_cast<uint4 *>(dst + c * 8) = v;
            }
        }
    }
    // a CTA that gave up waits (bounded) for its MMAs before releasing TMEM
    if (!ok && tid == 0) {
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
    int tiles;
    if (a.mode == ATT_WINDOW) {
        const WinGeom &g = a.geom;
        tiles = g.n <= BQ ? (g.nwin + BQ / g.n - 1) / (BQ / g.n) : g.nwin * (g.n / BQ);
    } else {
        tiles = (a.nq + BQ - 1) / BQ;
    }
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DPAD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    dim3 grid(a.heads, tiles, a.B);
    attn_tc_kernel<DPAD><<<grid, kThreads, L::ALLOC, s>>>(a, status);
    return cudaGetLastError();
}

int dpad_of(int d) { return (d + 15) / 16 * 16; }

}  // namespace

bool attention_tc_supported(const AttnArgs &a) {
    if (a.dtype != DT_BF16 || a.d % 8) return false;
    const int dp = dpad_of(a.d);
    if (dp != 64 && dp != 80 && dp != 128) return false;
    if (a.ldq % 8 || a.ldk % 8 || a.ldv % 8 || a.ldo % 8) return false;
    if ((uintptr_t)a.q % 16 || (uintptr_t)a.k % 16 || (uintptr_t)a.v % 16 || (uintptr_t)a.o % 16)
        return false;
    if (a.mode == ATT_WINDOW) {
        const int n = a.geom.n;
        return (n <= BQ && BQ % n == 0) || n % BQ == 0;
    }
    return a.nq >= 1 && a.nk >= 1;
}

cudaError_t launch_attention_tc(const AttnArgs &a, cudaStream_t s) {
    switch (dpad_of(a.d)) {
        case 64: return launch_dpad<64>(a, s);
        case 80: return launch_dpad<80>(a, s);
        case 128: return launch_dpad<128>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ptdit
