// Window and shifted-window self-attention of TCM on the tensor cores
// (Qihoo-T2X reading note, §3 Method, Eq. TCM): windows of 64 tokens (2D,
// packed two per 128-row tile) or 128 tokens (3D, one per tile) of the grid
// rolled by -shift, pairs that the roll wrapped masked out.
//
// One persistent CTA per SM with two independent slots; a unit is one tile
// (128 query rows = its own 128 key rows) of one head:
//   warps 2, 3   gather loaders, one per slot: each lane computes the token
//                row of its slots with the roll/wrap address function (no
//                permuted copy exists anywhere), cp.asyncs the Q, K and V rows
//                of the head into shared memory (16-byte chunks major: the
//                no-swizzle core-matrix layout, K-major for Q and K, MN-major
//                for V), builds one 128-bit key mask per mask key (window in
//                tile, wrap bits) with ballots, waits for its copies, fences
//                them to the async proxy and arrives on the slot's barrier.
//   warp 1       MMA issuer: S = Q K^T into TMEM, then P V with P read from
//                TMEM (written over S by the softmax) and V from shared memory.
//   warps 4-7, 8-11   softmax of slot 0 / slot 1: thread r owns query row r
//                (its TMEM lane), reads only its own window's scores, applies
//                the key mask, runs the softmax in fp32, writes P as bf16
//                pairs into TMEM, then scales its output row by 1/l and stores
//                it to global memory.
// While one slot computes, the other slot's rows stream in, so HBM stays busy.
// Every wait is bounded (2 s).
#include <math.h>

#include "tc_util.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128;
constexpr uint32_t CHUNK = BQ * 16;  // bytes between 16-byte chunk columns
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;  // per slot: S/P 128 columns, O 128 columns
constexpr int kKeys = 16;            // mask keys per tile: 2 windows x 8 wrap codes

template <int DPAD>
struct WinLayout {
    static constexpr int TILE = BQ * DPAD * 2;
    static constexpr int OFF_TILES = 0;                    // [slot][Q, K, V]
    static constexpr int OFF_INFO = 6 * TILE;              // int info[2][128]
    static constexpr int OFF_ROW = OFF_INFO + 2 * BQ * 4;  // long row[2][128]
    static constexpr int OFF_MASK = OFF_ROW + 2 * BQ * 8;  // uint32 kmask[2][kKeys][4]
    static constexpr int OFF_BAR = OFF_MASK + 2 * kKeys * 16;
    // load_full[2], slot_free[2], s_full[2], p_full[2], o_full[2], o_free[2], drain
    static constexpr int NBARS = 13;
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16;
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct WinSched {
    int tiles;  // tiles per batch item
    int units;  // B x tiles x heads
};

template <int DPAD>
__global__ void __launch_bounds__(kThreads, 1) attn_win_kernel(AttnArgs a, WinSched sc, int *status) {
    using L = WinLayout<DPAD>;
    constexpr int NCH = DPAD / 8;
    extern __shared__ __align__(128) uint8_t sm[];
    int *info = reinterpret_cast<int *>(sm + L::OFF_INFO);
    long *rowsm = reinterpret_cast<long *>(sm + L::OFF_ROW);
    uint32_t *kmask = reinterpret_cast<uint32_t *>(sm + L::OFF_MASK);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *load_full = bars, *slot_free = bars + 2, *s_full = bars + 4, *p_full = bars + 6;
    uint64_t *o_full = bars + 8, *o_free = bars + 10, *drain = bars + 12;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, nch = d / 8, n = a.geom.n;

    if (threadIdx.x == 0) {
        for (int g = 0; g < 2; ++g) {
            mbar_init(&load_full[g], 32);
            mbar_init(&slot_free[g], 1);
            mbar_init(&s_full[g], 1);
            mbar_init(&p_full[g], BQ);
            mbar_init(&o_full[g], 1);
            mbar_init(&o_free[g], BQ);
        }
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    // zero the padded chunks of the six tiles once; the loaders never touch them
    for (int i = threadIdx.x; i < 6 * BQ * (NCH - nch); i += kThreads) {
        const int t = i / (BQ * (NCH - nch)), rest = i % (BQ * (NCH - nch));
        const int c = nch + rest / BQ, r = rest % BQ;
        *reinterpret_cast<uint4 *>(sm + t * L::TILE + c * CHUNK + r * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;

    const int u0 = (int)((long)blockIdx.x * sc.units / gridDim.x);
    const int u1 = (int)((long)(blockIdx.x + 1) * sc.units / gridDim.x);
    // slot g takes units u0 + g, u0 + g + 2, ...: k-th unit of slot g
    auto unit_of = [&](int g, int k) { return u0 + g + 2 * k; };

    if (warp == 2 || warp == 3) {
        // ------------------------------------------------------------ gather loader of slot g
        const int g = warp - 2;
        uint8_t *sQ = sm + (3 * g + 0) * L::TILE, *sK = sm + (3 * g + 1) * L::TILE,
                *sV = sm + (3 * g + 2) * L::TILE;
        const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(a.q);
        const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(a.k);
        const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(a.v);
        const WinGeom &geo = a.geom;
        const int pack = BQ / n;
        for (int k = 0; unit_of(g, k) < u1; ++k) {
            const int u = unit_of(g, k);
            const int h = u % a.heads, rest = u / a.heads, tile = rest % sc.tiles,
                      b = rest / sc.tiles;
            if (!mbar_wait(&slot_free[g], (k & 1) ^ 1, abort, status)) break;
            int inf[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = q * 32 + lane;
                const int wit = r / n, win = tile * pack + wit, slot = r - wit * n;
                long row = -1;
                int in = -1;
                if (win < geo.nwin) {
                    int wrap;
                    row = (long)b * a.k_bstride + window_token(geo, win, slot, &wrap);
                    in = wit * 8 + wrap;
                }
                inf[q] = in;
                info[g * BQ + r] = in;
                rowsm[g * BQ + r] = row;
                const long rr = row >= 0 ? row : 0;
                const uint32_t bytes = row >= 0 ? 16 : 0;
                const __nv_bfloat16 *pq = qb + rr * a.ldq + (long)h * d;
                const __nv_bfloat16 *pk = kb + rr * a.ldk + (long)h * d;
                const __nv_bfloat16 *pv = vb + rr * a.ldv + (long)h * d;
                for (int c = 0; c < nch; ++c) {
                    cp_async16(sQ + c * CHUNK + r * 16, pq + c * 8, bytes);
                    cp_async16(sK + c * CHUNK + r * 16, pk + c * 8, bytes);
                    cp_async16(sV + c * CHUNK + r * 16, pv + c * 8, bytes);
                }
            }
            // one 128-bit key mask per mask key: keys of the same window and wrap code
            for (int v = 0; v < kKeys; ++v)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t bits = __ballot_sync(0xffffffffu, inf[q] == v);
                    if (lane == 0) kmask[(g * kKeys + v) * 4 + q] = bits;
                }
            cp_async_commit();  // wait_group only covers committed copies
            cp_async_wait_all();
            fence_async_smem();
            mbar_arrive(&load_full[g]);
        }
        cp_async_commit();
        cp_async_wait_all();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(BQ, BQ);
            constexpr uint32_t idesc_o = idesc_bf16(BQ, DPAD, true);
            bool ok = true, any = false;
            for (int k = 0; ok && unit_of(0, k) < u1; ++k) {
                for (int g = 0; g < 2 && ok; ++g) {
                    if (unit_of(g, k) >= u1) continue;
                    if (!mbar_wait(&load_full[g], k & 1, abort, status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t aQ = smem_u32(sm + (3 * g + 0) * L::TILE);
                    const uint32_t aK = smem_u32(sm + (3 * g + 1) * L::TILE);
#pragma unroll
                    for (int ks = 0; ks < DPAD / 16; ++ks)
                        mma_bf16(tmem + g * 256, sdesc_interleave(aQ + ks * 2 * CHUNK, CHUNK, 128),
                                 sdesc_interleave(aK + ks * 2 * CHUNK, CHUNK, 128), idesc_s, ks > 0);
                    mma_commit(&s_full[g]);
                    any = true;
                }
                for (int g = 0; g < 2 && ok; ++g) {
                    if (unit_of(g, k) >= u1) continue;
                    if (!mbar_wait(&p_full[g], k & 1, abort, status)) { ok = false; break; }
                    if (!mbar_wait(&o_free[g], (k & 1) ^ 1, abort, status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t aV = smem_u32(sm + (3 * g + 2) * L::TILE);
#pragma unroll
                    for (int ks = 0; ks < BQ / 16; ++ks)
                        mma_bf16_ts(tmem + g * 256 + 128, tmem + g * 256 + ks * 8,
                                    sdesc_interleave(aV + ks * 256, 128, CHUNK), idesc_o, ks > 0);
                    mma_commit(&o_full[g]);
                    mma_commit(&slot_free[g]);  // Q, K and V of this slot are read
                }
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                mma_commit(drain);
                volatile int never = 0;
                mbar_wait(drain, 0, &never, status);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax of slot g
        const int g = (warp - 4) / 4;
        const int r = (warp % 4) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + g * 256, t_o = t_s + 128;
        const float sl2 = a.scale * 1.4426950408889634f;
        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);
        // the row's own keys: its window inside the tile
        const int c_lo = n < BQ ? (r / n) * n : 0;
        for (int k = 0; unit_of(g, k) < u1; ++k) {
            const int u = unit_of(g, k);
            const int h = u % a.heads;
            if (!mbar_wait(&load_full[g], k & 1, abort, status)) break;  // masks and rows
            const int qi = info[g * BQ + r];
            const long qrow = rowsm[g * BQ + r];  // queries and keys share rows in window mode
            const bool live = rowsm[g * BQ + r] >= 0;
            uint32_t allow[4] = {0u, 0u, 0u, 0u};
            if (qi >= 0) {
                const uint4 w4 = *reinterpret_cast<const uint4 *>(kmask + (g * kKeys + qi) * 4);
                allow[0] = w4.x;
                allow[1] = w4.y;
                allow[2] = w4.z;
                allow[3] = w4.w;
            }
            if (!mbar_wait(&s_full[g], k & 1, abort, status)) break;
            fence_after_sync();
            float l = 0.f;
            uint32_t pk[64];
            if (n < BQ) {  // 64 keys: one half of the tile (the same half for the whole warp)
                uint32_t sv[64];
                tmem_ld32(t_s + c_lo, *reinterpret_cast<uint32_t(*)[32]>(sv));
                tmem_ld32(t_s + c_lo + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                tmem_ld_wait();
                const uint32_t w0 = c_lo == 0 ? allow[0] : allow[2];
                const uint32_t w1 = c_lo == 0 ? allow[1] : allow[3];
                float mx = -INFINITY;
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const bool ok = ((e < 32 ? w0 : w1) >> (e & 31)) & 1u;
                    if (!ok) sv[e] = __float_as_uint(-INFINITY);
                    mx = fmaxf(mx, __uint_as_float(sv[e]));
                }
                const float ref = mx * sl2;
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pp[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), sl2, -ref));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -ref));
                    ps[c & 3] += p0 + p1;
                    pp[c] = pack_bf16(p0, p1);
                }
                l = (ps[0] + ps[1]) + (ps[2] + ps[3]);
                // P columns hold key pairs: this window's 64 keys, zeros for the other window
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    pk[c] = c_lo == 0 ? pp[c] : 0u;
                    pk[32 + c] = c_lo == 0 ? 0u : pp[c];
                }
            } else {  // 128 keys
                uint32_t sv[128];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld32(t_s + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(sv + 32 * q));
                tmem_ld_wait();
                float mx = -INFINITY;
#pragma unroll
                for (int e = 0; e < 128; ++e) {
                    if (!((allow[e >> 5] >> (e & 31)) & 1u)) sv[e] = __float_as_uint(-INFINITY);
                    mx = fmaxf(mx, __uint_as_float(sv[e]));
                }
                const float ref = mx * sl2;
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), sl2, -ref));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -ref));
                    ps[c & 3] += p0 + p1;
                    pk[c] = pack_bf16(p0, p1);
                }
                l = (ps[0] + ps[1]) + (ps[2] + ps[3]);
            }
            tmem_st32(t_s, *reinterpret_cast<uint32_t(*)[32]>(pk));
            tmem_st32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
            tmem_st_wait();
            fence_before_sync();
            mbar_arrive(&p_full[g]);
            if (!mbar_wait(&o_full[g], k & 1, abort, status)) break;
            fence_after_sync();
            const float inv = 1.f / l;
            __nv_bfloat16 *dst = og + (live ? qrow : 0) * a.ldo + (long)h * d;
#pragma unroll
            for (int c0 = 0; c0 < DPAD; c0 += 16) {
                uint32_t ov[16];
                tmem_ld16(t_o + c0, ov);
                tmem_ld_wait();
                if (live) {
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
            fence_before_sync();
            mbar_arrive(&o_free[g]);
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
cudaError_t launch_win(const AttnArgs &a, cudaStream_t s) {
    using L = WinLayout<DPAD>;
    int *status = device_status_ptr();
    if (!status) return cudaErrorInvalidValue;
    WinSched sc;
    const int pack = BQ / a.geom.n;
    sc.tiles = (a.geom.nwin + pack - 1) / pack;
    sc.units = a.B * sc.tiles * a.heads;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int grid = (sc.units + 1) / 2 < sms ? (sc.units + 1) / 2 : sms;
    cudaError_t e = cudaFuncSetAttribute(attn_win_kernel<DPAD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    attn_win_kernel<DPAD><<<grid, kThreads, L::BYTES, s>>>(a, sc, status);
    return cudaGetLastError();
}

}  // namespace

bool attention_win_tc_supported(const AttnArgs &a) {
    return a.mode == ATT_WINDOW && (a.geom.n == 64 || a.geom.n == 128) && a.q_bstride == a.k_bstride;
}

cudaError_t launch_attention_win_tc(const AttnArgs &a, cudaStream_t s) {
    const int dp = (a.d + 15) / 16 * 16;
    if (dp == 64) return launch_win<64>(a, s);
    if (dp == 80) return launch_win<80>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace ptdit
