// Window and shifted-window self-attention of TCM on the tensor cores
// (Qihoo-T2X reading note, §3 Method, Eq. TCM): windows of 64 tokens (2D,
// packed two per 128-row tile) or 128 tokens (3D, one per tile) of the grid
// rolled by -shift, pairs that the roll wrapped masked out.
//
// One persistent CTA per SM with two independent slots; a unit is one tile
// (128 query rows = its own 128 key rows) of one head:
//   warps 2, 3   loaders, one per slot: each lane computes the token row of
//                its slots with the roll/wrap address function (no permuted
//                copy exists anywhere), then the warp copies the head's Q, K
//                and V rows with 16-byte cp.async into the 128-byte-swizzled
//                K-major layout (columns 64.. in a 32-byte-swizzled block for
//                Q and K, a second 128-byte atom for V).  Eight lanes cover
//                one row's 128 contiguous bytes, so an instruction touches
//                four rows instead of 32; Q and K complete on their own
//                barrier so S = Q K^T starts while V is still arriving.  Key
//                masks (window in tile x wrap bits) are built with ballots.
//                (Tile loads by TMA are not used here: a box walks the head's
//                rows one by one, and at 144 bytes a row that rate, not HBM,
//                bounded the loads.)
//   warp 1       MMA issuer: S = Q K^T into TMEM, then O = P V with P read
//                from TMEM (the softmax writes it over S) and V from shared
//                memory, padded to 128 columns so one MMA per K step covers
//                the head.
//   warps 4-7, 8-11   softmax of slot 0 / slot 1: thread r owns query row r,
//                reads only its own window's scores, masks, exponentiates in
//                fp32, writes P as bf16 pairs into TMEM, then scales its
//                output row by 1/l and stores it.
// Every wait is bounded (2 s).
#include <math.h>

#include "tc_util.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;  // per slot: S/P 128 columns, O 128 columns
constexpr int kKeys = 16;            // mask keys per tile: 2 windows x 8 wrap codes

template <int DPAD>
struct WinLayout {
    static constexpr bool HAS_B = DPAD > 64;                   // head columns 64..79
    static constexpr int TILE_A = BQ * 128;                    // columns 0..63, 128-byte swizzle
    static constexpr int TILE_B = HAS_B ? BQ * 32 : 0;         // columns 64..79, 32-byte swizzle
    static constexpr int TILE = TILE_A + TILE_B;               // a Q or K tile (K-major)
    static constexpr int VTILE = HAS_B ? 2 * TILE_A : TILE_A;  // V, MN-major, padded to 128
    static constexpr int NPV = HAS_B ? 128 : 64;
    static constexpr int SLOT = 2 * TILE + VTILE;              // Q, K, V of one slot
    static constexpr int OFF_INFO = 2 * SLOT;                  // int info[2][128]
    static constexpr int OFF_ROW = OFF_INFO + 2 * BQ * 4;      // long row[2][128]
    static constexpr int OFF_MASK = OFF_ROW + 2 * BQ * 8;      // uint32 kmask[2][kKeys][4]
    static constexpr int OFF_BAR = OFF_MASK + 2 * kKeys * 16;
    // qk_full[2], v_full[2], slot_free[2], s_full[2], p_full[2], o_full[2], o_free[2], drain
    static constexpr int NBARS = 15;
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16 + 1024;  // + base alignment slack
    static_assert(TILE_A % 1024 == 0 && TILE % 1024 == 0 && SLOT % 1024 == 0,
                  "swizzled tiles stay 1 KB aligned");
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct WinSched {
    int tiles;  // tiles per batch item
    int units;  // B x tiles x heads
};

// Byte offset of 16-byte unit c of row r (0..7) inside one 128-byte-swizzled atom.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return r * 128 + ((c ^ r) << 4); }
// Same for a 32-byte-swizzled atom (8 rows x 2 units).
__device__ __forceinline__ uint32_t sw32(int r, int u) { return r * 32 + ((u ^ ((r >> 2) & 1)) << 4); }

template <int DPAD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_win_kernel(const __grid_constant__ AttnArgs a, WinSched sc, int *status) {
    using L = WinLayout<DPAD>;
    extern __shared__ uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    int *info = reinterpret_cast<int *>(sm + L::OFF_INFO);
    long *rowsm = reinterpret_cast<long *>(sm + L::OFF_ROW);
    uint32_t *kmask = reinterpret_cast<uint32_t *>(sm + L::OFF_MASK);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *qk_full = bars, *v_full = bars + 2, *slot_free = bars + 4, *s_full = bars + 6;
    uint64_t *p_full = bars + 8, *o_full = bars + 10, *o_free = bars + 12, *drain = bars + 14;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, n = a.geom.n, nch = d / 8;

    if (threadIdx.x == 0) {
        for (int g = 0; g < 2; ++g) {
            mbar_init(&qk_full[g], 32);
            mbar_init(&v_full[g], 32);
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
    // zero, once, the padding columns no copy writes: Q and K columns d..79,
    // V columns d..127 (their products with P and Q are then exactly 0)
    if (L::HAS_B) {
        for (int i = threadIdx.x; i < 2 * BQ * 8; i += kThreads) {
            const int g = i / (BQ * 8), r = (i / 8) % BQ, c = i % 8;
            uint8_t *slot = sm + g * L::SLOT;
            const uint4 z = make_uint4(0, 0, 0, 0);
            if (8 + c >= nch) {
                if (c < 2) {
                    const uint32_t o = L::TILE_A + (r >> 3) * 256 + sw32(r & 7, c);
                    *reinterpret_cast<uint4 *>(slot + o) = z;
                    *reinterpret_cast<uint4 *>(slot + L::TILE + o) = z;
                }
                *reinterpret_cast<uint4 *>(slot + 2 * L::TILE + L::TILE_A + (r >> 3) * 1024 +
                                           sw128(r & 7, c)) = z;
            }
        }
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
        // ------------------------------------------------------------ loader of slot g
        const int g = warp - 2;
        uint8_t *sQ = sm + g * L::SLOT, *sK = sQ + L::TILE, *sV = sK + L::TILE;
        const char *gq = static_cast<const char *>(a.q);
        const char *gk = static_cast<const char *>(a.k);
        const char *gv = static_cast<const char *>(a.v);
        const long ldq = a.ldq * 2, ldk = a.ldk * 2, ldv = a.ldv * 2;  // row pitches in bytes
        const WinGeom &geo = a.geom;
        const int pack = BQ / n;
        const int c8 = lane & 7;  // 16-byte chunk (columns 8 c8 .. 8 c8 + 7) of the main copies
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
            }
            __syncwarp();
            const long hoff = (long)h * d * 2;
            // columns 0..63: eight lanes per row, four rows per instruction; Q and K first
#pragma unroll 4
            for (int it = 0; it < BQ / 4; ++it) {
                const int r = 4 * it + (lane >> 3);
                const long row = rowsm[g * BQ + r];
                const uint32_t bytes = row >= 0 ? 16u : 0u;
                const long rr = row >= 0 ? row : 0;
                const uint32_t o = (r >> 3) * 1024 + sw128(r & 7, c8);
                cp_async16(sQ + o, gq + rr * ldq + hoff + c8 * 16, bytes);
                cp_async16(sK + o, gk + rr * ldk + hoff + c8 * 16, bytes);
            }
            if (L::HAS_B) {  // columns 64 .. d-1: one row per lane
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int r = q * 32 + lane;
                    const long row = rowsm[g * BQ + r];
                    const uint32_t bytes = row >= 0 ? 16u : 0u;
                    const long rr = row >= 0 ? row : 0;
                    for (int c = 8; c < nch; ++c) {
                        const uint32_t o = L::TILE_A + (r >> 3) * 256 + sw32(r & 7, c - 8);
                        cp_async16(sQ + o, gq + rr * ldq + hoff + c * 16, bytes);
                        cp_async16(sK + o, gk + rr * ldk + hoff + c * 16, bytes);
                    }
                }
            }
            cp_async_commit();
#pragma unroll 4
            for (int it = 0; it < BQ / 4; ++it) {
                const int r = 4 * it + (lane >> 3);
                const long row = rowsm[g * BQ + r];
                const uint32_t bytes = row >= 0 ? 16u : 0u;
                const long rr = row >= 0 ? row : 0;
                cp_async16(sV + (r >> 3) * 1024 + sw128(r & 7, c8), gv + rr * ldv + hoff + c8 * 16,
                           bytes);
            }
            if (L::HAS_B) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int r = q * 32 + lane;
                    const long row = rowsm[g * BQ + r];
                    const uint32_t bytes = row >= 0 ? 16u : 0u;
                    const long rr = row >= 0 ? row : 0;
                    for (int c = 8; c < nch; ++c)
                        cp_async16(sV + L::TILE_A + (r >> 3) * 1024 + sw128(r & 7, c - 8),
                                   gv + rr * ldv + hoff + c * 16, bytes);
                }
            }
            cp_async_commit();
            // one 128-bit key mask per mask key: keys of the same window and wrap code
            for (int v = 0; v < kKeys; ++v)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t bits = __ballot_sync(0xffffffffu, inf[q] == v);
                    if (lane == 0) kmask[(g * kKeys + v) * 4 + q] = bits;
                }
            cp_async_wait_group1();  // Q and K have landed (V may still be in flight)
            fence_async_smem();
            mbar_arrive(&qk_full[g]);
            cp_async_wait_all();
            fence_async_smem();
            mbar_arrive(&v_full[g]);
        }
        cp_async_commit();
        cp_async_wait_all();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(BQ, BQ);
            constexpr uint32_t idesc_o = idesc_bf16(BQ, L::NPV, true);
            bool ok = true, any = false;
            for (int k = 0; ok && unit_of(0, k) < u1; ++k) {
                for (int g = 0; g < 2 && ok; ++g) {
                    if (unit_of(g, k) >= u1) continue;
                    if (!mbar_wait(&qk_full[g], k & 1, abort, status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t aQ = smem_u32(sm + g * L::SLOT);
                    const uint32_t aK = aQ + L::TILE;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + g * 256, sdesc_sw128(aQ + kk * 32), sdesc_sw128(aK + kk * 32),
                                 idesc_s, kk > 0);
                    if (L::HAS_B)
                        mma_bf16(tmem + g * 256, sdesc_sw32(aQ + L::TILE_A), sdesc_sw32(aK + L::TILE_A),
                                 idesc_s, 1);
                    mma_commit(&s_full[g]);
                    any = true;
                }
                for (int g = 0; g < 2 && ok; ++g) {
                    if (unit_of(g, k) >= u1) continue;
                    if (!mbar_wait(&v_full[g], k & 1, abort, status)) { ok = false; break; }
                    if (!mbar_wait(&p_full[g], k & 1, abort, status)) { ok = false; break; }
                    if (!mbar_wait(&o_free[g], (k & 1) ^ 1, abort, status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t aV = smem_u32(sm + g * L::SLOT + 2 * L::TILE);
#pragma unroll
                    for (int ks = 0; ks < BQ / 16; ++ks)
                        mma_bf16_ts(tmem + g * 256 + 128, tmem + g * 256 + ks * 8,
                                    sdesc_sw128_mn(aV + ks * 2048, L::TILE_A), idesc_o, ks > 0);
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
        const int nch = d / 8;
        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);
        // the row's own keys: its window inside the tile
        const int c_lo = n < BQ ? (r / n) * n : 0;
        for (int k = 0; unit_of(g, k) < u1; ++k) {
            const int u = unit_of(g, k);
            const int h = u % a.heads;
            if (!mbar_wait(&qk_full[g], k & 1, abort, status)) break;  // masks and rows
            const int qi = info[g * BQ + r];
            const long qrow = rowsm[g * BQ + r];  // queries and keys share rows in window mode
            const bool live = qrow >= 0;
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
    if (*abort) {
        // give box loads still in flight into this CTA a moment to land
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 100000) {
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

// Windows of 64 or 128 tokens (any shape and shift), head width 64..80.
bool attention_win_tc_supported(const AttnArgs &a) {
    if (a.dtype != DT_BF16 || a.mode != ATT_WINDOW) return false;
    if (!(a.geom.n == 64 || a.geom.n == 128) || a.q_bstride != a.k_bstride) return false;
    if (a.d % 8 || a.d < 64 || a.d > 80) return false;
    if (a.ldq % 8 || a.ldk % 8 || a.ldv % 8 || a.ldo % 8) return false;
    return true;
}

cudaError_t launch_attention_win_tc(const AttnArgs &a, cudaStream_t s) {
    if (a.d <= 64) return launch_win<64>(a, s);
    return launch_win<80>(a, s);
}

}  // namespace ptdit
