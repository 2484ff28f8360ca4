// Row-mode attention core on the tensor cores: proxy self-attention and
// latent -> proxy cross-attention of GIIM (Qihoo-T2X reading note, §3
// Method, Eq. GIIM), and full self-attention (the dense comparator of the
// complexity paragraph).  Queries are rows [0, nq) and keys rows [0, nk) of
// each batch item; head h is columns h*d .. h*d+d-1.
//
// FlashAttention-style warp specialisation, one persistent CTA per SM:
//   warp 0       loader: one TMA load per 128-row tile -- two query tiles
//                per unit, K and V tiles into a two-stage ring.  A 4-D tensor
//                map (8 elements, rows, 16-byte chunks, heads) writes each tile
//                straight into the chunk-major layout below and zero-fills the
//                padded chunk.
//   warp 1       MMA issuer: S0 = Q0 K^T and S1 = Q1 K^T into TMEM, then
//                P0 V and P1 V into TMEM once each softmax has written P.
//   warps 4-7 and 8-11   two softmax warpgroups, one per query tile: thread r
//                owns row r (its TMEM lane), reads S with tcgen05.ld, runs the
//                fp32 online softmax and writes P (bf16) to shared memory; the
//                P V products accumulate in TMEM, rescaled in place only when
//                a row's reference max has to rise.
// Both query tiles share every K/V tile, and while one warpgroup runs its
// softmax the tensor core works for the other.  Shared memory layout: 16-byte
// chunks major, byte (chunk c, row r) = c * 2048 + r * 16 (the no-swizzle
// core-matrix layout: K-major for Q, K and P, MN-major for V); d is padded
// with zeros to a multiple of 16.  Every wait is bounded (2 s).
#include <math.h>

#include "tc_util.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128, BKV = 128;
constexpr uint32_t CHUNK = BQ * 16;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;  // S0, S1, O0, O1: 128 columns each

template <int DPAD>
struct RowsLayout {
    static constexpr int TILE = BQ * DPAD * 2;
    static constexpr int P_BYTES = BQ * BKV * 2;
    static constexpr int OFF_Q = 0;             // Q0, Q1
    static constexpr int OFF_K = 2 * TILE;      // K0, K1 (stages)
    static constexpr int OFF_V = 4 * TILE;      // V0, V1
    static constexpr int OFF_P = 6 * TILE;      // P0, P1
    static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
    // kv_full[2], kv_empty[2], q_full, q_empty, s_full[2], p_full[2], o_full[2], drain
    static constexpr int NBARS = 14;
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16 + 1024;  // + base alignment slack
    static_assert(TILE % 1024 == 0 && P_BYTES % 1024 == 0, "tiles stay 1 KB aligned");
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct RowsSched {
    int qp;     // query-tile pairs (256 rows) per batch item and head
    int kt;     // key tiles per unit
    int units;  // batch items x heads x qp
};

__device__ __forceinline__ void decode(const AttnArgs &a, const RowsSched &sc, int u, int &b,
                                       int &h, int &qp) {
    qp = u % sc.qp;
    const int r = u / sc.qp;
    h = r % a.heads;
    b = r / a.heads;
}

template <int DPAD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_rows_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                     const __grid_constant__ CUtensorMap mv, AttnArgs a, RowsSched sc,
                     int *status) {
    using L = RowsLayout<DPAD>;
    constexpr int NCH = DPAD / 8;
    extern __shared__ uint8_t sm_raw[];
    // TMA destinations: align the base to 1 KB (tile offsets are multiples of 1 KB)
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *kv_full = bars, *kv_empty = bars + 2, *q_full = bars + 4, *q_empty = bars + 5;
    uint64_t *s_full = bars + 6, *p_full = bars + 8, *o_full = bars + 10, *drain = bars + 12;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, nch = d / 8;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], BQ);
            mbar_init(&o_full[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;

    const int u0 = (int)((long)blockIdx.x * sc.units / gridDim.x);
    const int u1 = (int)((long)(blockIdx.x + 1) * sc.units / gridDim.x);

    if (warp == 0) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            prefetch_tensormap(&mq);
            prefetch_tensormap(&mk);
            prefetch_tensormap(&mv);
            int item = 0, last_q_unit = -1;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                int b, h, qp;
                decode(a, sc, u, b, h, qp);
                for (int j = 0; j < sc.kt; ++j, ++item) {
                    const int st = item & 1;
                    if (j == 0) {
                        if (!mbar_wait(q_empty, ((u - u0) & 1) ^ 1, abort, status)) { ok = false; break; }
                        const int row0 = (int)((long)b * a.q_bstride + qp * 2 * BQ);
                        mbar_expect_tx(q_full, 2 * L::TILE);
                        tma_load_4d(sm + L::OFF_Q, &mq, q_full, 0, row0, 0, h);
                        tma_load_4d(sm + L::OFF_Q + L::TILE, &mq, q_full, 0, row0 + BQ, 0, h);
                        last_q_unit = u - u0;
                    }
                    if (!mbar_wait(&kv_empty[st], ((item >> 1) & 1) ^ 1, abort, status)) { ok = false; break; }
                    const int krow = (int)((long)b * a.k_bstride + j * BKV);
                    mbar_expect_tx(&kv_full[st], 2 * L::TILE);
                    tma_load_4d(sm + L::OFF_K + st * L::TILE, &mk, &kv_full[st], 0, krow, 0, h);
                    tma_load_4d(sm + L::OFF_V + st * L::TILE, &mv, &kv_full[st], 0, krow, 0, h);
                }
            }
            if (!ok) {  // let copies still in flight land before the CTA exits
                volatile int never = 0;
                for (int i = item - 2; i < item; ++i)
                    if (i >= 0) mbar_wait(&kv_full[i & 1], (i >> 1) & 1, &never, status);
                if (last_q_unit >= 0) mbar_wait(q_full, last_q_unit & 1, &never, status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(BQ, BKV);
            constexpr uint32_t idesc_o = idesc_bf16(BQ, DPAD, true);
            int item = 0;
            bool ok = true, any = false;
            for (int u = u0; u < u1 && ok; ++u) {
                for (int j = 0; j < sc.kt; ++j, ++item) {
                    const int st = item & 1;
                    const uint32_t ph = item & 1;
                    if (!mbar_wait(&kv_full[st], (item >> 1) & 1, abort, status)) { ok = false; break; }
                    if (j == 0 && !mbar_wait(q_full, (u - u0) & 1, abort, status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t aK = smem_u32(sm + L::OFF_K + st * L::TILE);
                    const uint32_t aV = smem_u32(sm + L::OFF_V + st * L::TILE);
                    for (int g = 0; g < 2; ++g) {
                        const uint32_t aQ = smem_u32(sm + L::OFF_Q + g * L::TILE);
#pragma unroll
                        for (int ks = 0; ks < DPAD / 16; ++ks)
                            mma_bf16(tmem + g * BKV, sdesc_interleave(aQ + ks * 2 * CHUNK, CHUNK, 128),
                                     sdesc_interleave(aK + ks * 2 * CHUNK, CHUNK, 128), idesc_s,
                                     ks > 0);
                        mma_commit(&s_full[g]);
                    }
                    any = true;
                    if (j == sc.kt - 1) mma_commit(q_empty);
                    for (int g = 0; g < 2; ++g) {
                        if (!mbar_wait(&p_full[g], ph, abort, status)) { ok = false; break; }
                        fence_after_sync();
                        const uint32_t aP = smem_u32(sm + L::OFF_P + g * L::P_BYTES);
#pragma unroll
                        for (int ks = 0; ks < BKV / 16; ++ks)
                            mma_bf16(tmem + 256 + g * 128,
                                     sdesc_interleave(aP + ks * 2 * CHUNK, CHUNK, 128),
                                     sdesc_interleave(aV + ks * 256, 128, CHUNK), idesc_o,
                                     (j | ks) > 0);
                        mma_commit(&o_full[g]);
                    }
                    if (!ok) break;
                    mma_commit(&kv_empty[st]);
                }
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                mma_commit(drain);
                volatile int never = 0;
                mbar_wait(drain, 0, &never, status);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax warpgroups
        // The output accumulates in TMEM (each P V adds onto it).  Scores are
        // exponentiated against a per-row reference max that is only raised
        // when a tile's max exceeds it by more than 2^8 (weights then stay
        // below 256, harmless in fp32); raising it rescales the row of O in
        // TMEM, after the previous P V has landed.
        const int g = (warp - 4) / 4;
        const int r = (warp % 4) * 32 + lane;  // query row of the tile = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + g * BKV;
        const uint32_t t_o = tmem + lane_base + 256 + g * 128;
        uint8_t *sP = sm + L::OFF_P + g * L::P_BYTES;
        const float sl2 = a.scale * 1.4426950408889634f;
        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);
        int item = 0;
        bool ok = true;
        for (int u = u0; u < u1 && ok; ++u) {
            int b, h, qp;
            decode(a, sc, u, b, h, qp);
            const int iq = qp * 2 * BQ + g * BQ + r;
            float m_ref = -INFINITY, l_i = 0.f;
            for (int j = 0; j < sc.kt; ++j, ++item) {
                const uint32_t ph = item & 1;
                const int nvalid = min(BKV, a.nk - j * BKV);
                if (!mbar_wait(&s_full[g], ph, abort, status)) { ok = false; break; }
                fence_after_sync();
                float tmax = -INFINITY;
#pragma unroll 1
                for (int c0 = 0; c0 < nvalid; c0 += 32) {
                    uint32_t s[32];
                    tmem_ld32(t_s + c0, s);
                    tmem_ld_wait();
                    if (c0 + 32 <= nvalid) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) tmax = fmaxf(tmax, __uint_as_float(s[e]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (c0 + e < nvalid) tmax = fmaxf(tmax, __uint_as_float(s[e]));
                    }
                }
                tmax *= sl2;
                if (tmax > m_ref + 8.f) {  // raise the reference; O so far shrinks by alpha
                    const float alpha = m_ref == -INFINITY ? 0.f : ex2_approx(m_ref - tmax);
                    if (j > 0) {
                        // O holds P V up to tile j-1 once that MMA has landed
                        if (!mbar_wait(&o_full[g], ph ^ 1, abort, status)) { ok = false; break; }
                        fence_after_sync();
#pragma unroll
                        for (int c0 = 0; c0 < DPAD; c0 += 16) {
                            uint32_t ov[16];
                            tmem_ld16(t_o + c0, ov);
                            tmem_ld_wait();
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                            tmem_st16(t_o + c0, ov);
                        }
                        tmem_st_wait();
                    }
                    l_i *= alpha;
                    m_ref = tmax;
                }
                const float ref = m_ref == -INFINITY ? 0.f : m_ref;
                float psum = 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < BKV; c0 += 32) {
                    uint4 v[4];
                    if (c0 + 32 <= nvalid) {
                        uint32_t s[32];
                        tmem_ld32(t_s + c0, s);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            float pv[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                pv[e] = ex2_approx(fmaf(__uint_as_float(s[8 * q + e]), sl2, -ref));
                                psum += pv[e];
                            }
                            v[q].x = pack_bf16(pv[0], pv[1]);
                            v[q].y = pack_bf16(pv[2], pv[3]);
                            v[q].z = pack_bf16(pv[4], pv[5]);
                            v[q].w = pack_bf16(pv[6], pv[7]);
                        }
                    } else if (c0 < nvalid) {
                        uint32_t s[32];
                        tmem_ld32(t_s + c0, s);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            float pv[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int jj = 8 * q + e;
                                pv[e] = c0 + jj < nvalid
                                            ? ex2_approx(fmaf(__uint_as_float(s[jj]), sl2, -ref))
                                            : 0.f;
                                psum += pv[e];
                            }
                            v[q].x = pack_bf16(pv[0], pv[1]);
                            v[q].y = pack_bf16(pv[2], pv[3]);
                            v[q].z = pack_bf16(pv[4], pv[5]);
                            v[q].w = pack_bf16(pv[6], pv[7]);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) v[q] = make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(sP + ((c0 >> 3) + q) * CHUNK + r * 16) = v[q];
                }
                l_i += psum;
                fence_before_sync();
                fence_async_smem();
                mbar_arrive(&p_full[g]);
            }
            if (!ok) break;
            // the unit's last P V, then O / l to global memory
            if (!mbar_wait(&o_full[g], (item - 1) & 1, abort, status)) { ok = false; break; }
            fence_after_sync();
            const float inv = 1.f / l_i;
            __nv_bfloat16 *dst = og + ((long)b * a.q_bstride + iq) * a.ldo + (long)h * d;
#pragma unroll
            for (int c0 = 0; c0 < DPAD; c0 += 16) {
                uint32_t ov[16];
                tmem_ld16(t_o + c0, ov);
                tmem_ld_wait();
                if (iq < a.nq) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        if ((c0 >> 3) + c < nch) {
                            uint4 v;
                            v.x = pack_bf16(__uint_as_float(ov[8 * c + 0]) * inv, __uint_as_float(ov[8 * c + 1]) * inv);
                            v.y = pack_bf16(__uint_as_float(ov[8 * c + 2]) * inv, __uint_as_float(ov[8 * c + 3]) * inv);
                            v.z = pack_bf16(__uint_as_float(ov[8 * c + 4]) * inv, __uint_as_float(ov[8 * c + 5]) * inv);
                            v.w = pack_bf16(__uint_as_float(ov[8 * c + 6]) * inv, __uint_as_float(ov[8 * c + 7]) * inv);
                            *reinterpret_cast<uint4 *>(dst + c0 + 8 * c) = v;
                        }
                    }
                }
            }
            fence_before_sync();  // O is read before the next unit's first P V overwrites it
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int DPAD>
cudaError_t launch_rows(const AttnArgs &a, cudaStream_t s) {
    using L = RowsLayout<DPAD>;
    int *status = device_status_ptr();
    if (!status) return cudaErrorInvalidValue;
    const int nch = a.d / 8;
    CUtensorMap mq, mk, mv;
    if (!encode_map_rows_heads_bf16(&mq, a.q, (uint64_t)a.B * a.q_bstride, a.ldq * 2, nch, a.heads,
                                    a.d, BQ, DPAD / 8) ||
        !encode_map_rows_heads_bf16(&mk, a.k, (uint64_t)a.B * a.k_bstride, a.ldk * 2, nch, a.heads,
                                    a.d, BKV, DPAD / 8) ||
        !encode_map_rows_heads_bf16(&mv, a.v, (uint64_t)a.B * a.k_bstride, a.ldv * 2, nch, a.heads,
                                    a.d, BKV, DPAD / 8))
        return cudaErrorNotSupported;  // the caller falls back to the gather kernel
    RowsSched sc;
    sc.qp = (a.nq + 2 * BQ - 1) / (2 * BQ);
    sc.kt = (a.nk + BKV - 1) / BKV;
    sc.units = a.B * a.heads * sc.qp;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int grid = sc.units < sms ? sc.units : sms;
    cudaError_t e = cudaFuncSetAttribute(attn_rows_kernel<DPAD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    attn_rows_kernel<DPAD><<<grid, kThreads, L::BYTES, s>>>(mq, mk, mv, a, sc, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_rows_tc(const AttnArgs &a, cudaStream_t s) {
    const int dp = (a.d + 15) / 16 * 16;
    if (dp == 64) return launch_rows<64>(a, s);
    if (dp == 80) return launch_rows<80>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace ptdit
