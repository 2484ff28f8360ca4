// Row-mode attention core on the tensor cores: proxy self-attention and
// latent -> proxy cross-attention of GIIM (Qihoo-T2X reading note, §3
// Method, Eq. GIIM), and full self-attention (the dense comparator of the
// complexity paragraph).  Queries are rows [0, nq) and keys rows [0, nk) of
// each batch item; head h is columns h*d .. h*d+d-1.
//
// FlashAttention-style warp specialisation, one persistent CTA per SM:
//   warp 0       loader: two 128-row query tiles per unit (double buffered
//                across units), K tiles and V tiles into two-stage rings of
//                their own (a K stage is released after both score MMAs, a V
//                stage after both P V MMAs), each one contiguous bulk copy:
//                the projections wrote Q, K and V in tiled head layout
//                (thl.cuh), so a (tile, head) block already
//                is the swizzled shared-memory tile (columns 0..63 with the
//                128-byte swizzle, 64..79 with the 32-byte swizzle, zeros past
//                the head; V padded to 128 columns).
//   warp 1       MMA issuer (the whole warp runs the loop, lane 0 issues):
//                S_g = Q_g K^T (K-major operands) into TMEM, and
//                once softmax g has written P_g, P_g V with P_g read straight
//                from TMEM and V as an MN-major operand (no transpose),
//                accumulating into O_g in TMEM.
//   warp 2       output stores: one tensor store per staged 128-row output tile.
//   warps 4-7 and 8-11   two softmax warpgroups, one per query tile: thread r
//                owns row r (its TMEM lane), reads its 128 scores with one
//                wait, runs the fp32 online softmax and writes P (bf16, two per
//                column) back over the first 64 columns of its scores; O is
//                rescaled in TMEM only when a row's reference max has to rise
//                by more than 2^8.  P never touches shared memory (a version
//                with P in shared memory, which lets the next S be issued as
//                soon as the softmax has read the current one, was slower: the
//                P writes and reads crowd shared-memory bandwidth, and the
//                unpadded V it needed costs a second, N = 16, MMA per K step).
// Both query tiles share every K/V tile; the MMA warp issues PV_0, S_0(next),
// PV_1, S_1(next), so each softmax gets its next scores while the other one
// works.  Splitting each tile's scores into two 64-key slots (so that the next
// half's scores are ready when the softmax of a half ends) was slower: it
// doubles the softmax -> P V -> S round trips, each about as long as before.
// Every wait is bounded (2 s).
#include <math.h>

#include "tc_util.cuh"
#include "thl.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128, BKV = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;  // S0, S1, O0, O1: 128 columns each

constexpr int NSTAGE = 2;  // depth of the K ring and of the V ring

template <int DPAD>
struct RowsLayout {
    static constexpr bool HAS_B = DPAD > 64;            // head columns 64..79
    static constexpr int TILE_A = BQ * 64 * 2;          // 128 rows x 128 B, 128-byte swizzle
    static constexpr int TILE_B = HAS_B ? BQ * 16 * 2 : 0;  // 128 rows x 32 B, 32-byte swizzle
    static constexpr int TILE = TILE_A + TILE_B;        // a Q or K tile (K-major)
    // V is the MN-major operand of P V: one MMA per K step costs the same for
    // N = 64 or 128, so its head columns are padded to 128 with a second
    // 64-wide 128-byte-swizzled atom (zeros past the head) instead of being
    // split into an N = 64 and an N = 16 MMA.
    static constexpr int VTILE = HAS_B ? 2 * TILE_A : TILE_A;
    static constexpr int NPV = HAS_B ? 128 : 64;        // N of the P V MMA
    static constexpr int OFF_Q = 0;                     // [unit parity][query tile]
    static constexpr int OFF_K = 4 * TILE;              // [stage]
    static constexpr int OFF_V = OFF_K + NSTAGE * TILE; // [stage]
    // output staging of each softmax warpgroup: 128 rows, pitch <= 160 B
    static constexpr int STG = BQ * 160;
    static constexpr int OFF_STG = OFF_V + NSTAGE * VTILE;
    static constexpr int OFF_BAR = OFF_STG + 2 * STG;
    // k_full[NSTAGE], k_empty[NSTAGE], v_full[NSTAGE], v_empty[NSTAGE], q_full[2], q_empty[2],
    // s_full[2], p_full[2], o_full[2],
    // drain, stage_full[2], stage_free[2]
    static constexpr int NBARS = 4 * NSTAGE + 15;
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16 + 1024;  // + base alignment slack
    static_assert(TILE % 1024 == 0 && TILE_A % 1024 == 0, "swizzled tiles stay 1 KB aligned");
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

template <int DPAD, bool SUMV>
__global__ void __launch_bounds__(kThreads, 1)
    attn_rows_kernel(const __grid_constant__ AttnArgs a, RowsSched sc,
                     const __grid_constant__ CUtensorMap omap, int *status) {
    using L = RowsLayout<DPAD>;
    extern __shared__ uint8_t sm_raw[];
    // TMA destinations: align the base to 1 KB (tile offsets are multiples of 1 KB)
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *k_full = bars, *k_empty = bars + NSTAGE;
    uint64_t *v_full = bars + 2 * NSTAGE, *v_empty = bars + 3 * NSTAGE;
    uint64_t *q_full = bars + 4 * NSTAGE, *q_empty = q_full + 2, *s_full = q_full + 4;
    uint64_t *p_full = q_full + 6, *o_full = q_full + 8, *drain = q_full + 10;
    uint64_t *stage_full = q_full + 11, *stage_free = q_full + 13;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, nch = d / 8;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], BQ);
            mbar_init(&o_full[s], 1);
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        mbar_init(drain, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&stage_full[s], BQ);
            mbar_init(&stage_free[s], 1);
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    pdl_wait();  // the projections that wrote Q, K and V have completed
    pdl_trigger();

    const int u0 = (int)((long)blockIdx.x * sc.units / gridDim.x);
    const int u1 = (int)((long)(blockIdx.x + 1) * sc.units / gridDim.x);

    if (warp == 0) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            const uint8_t *qg = static_cast<const uint8_t *>(a.q);
            const uint8_t *kg = static_cast<const uint8_t *>(a.k);
            const uint8_t *vg = static_cast<const uint8_t *>(a.v);
            // the (tile, head) block of batch item b
            auto block = [&](const uint8_t *base, const ThlDesc &t, int b, int tile, int h,
                             uint32_t bytes) {
                return base + (((long)b * t.tiles + tile) * a.heads + h) * (long)bytes;
            };
            int item = 0, k_issued = 0, v_issued = 0, last_q_unit = -1;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                int b, h, qp;
                decode(a, sc, u, b, h, qp);
                const int un = u - u0;
                for (int j = 0; j < sc.kt; ++j, ++item) {
                    const int st = item % NSTAGE;
                    if (j == 0) {
                        const int qb = un & 1;
                        if (!mbar_wait(&q_empty[qb], ((un >> 1) & 1) ^ 1, abort, status)) { ok = false; break; }
                        // the unit's second query tile may lie past the last one: the
                        // last tile is loaded twice then (its second results are
                        // not stored), so no row scores uninitialised memory
                        mbar_expect_tx(&q_full[qb], 2 * L::TILE);
                        for (int g = 0; g < 2; ++g)
                            bulk_load(sm + L::OFF_Q + (qb * 2 + g) * L::TILE,
                                      block(qg, a.tq, b, min(2 * qp + g, a.tq.tiles - 1), h, L::TILE),
                                      L::TILE, &q_full[qb]);
                        last_q_unit = un;
                    }
                    // K and V have rings of their own: a K stage is free once both
                    // score MMAs of its item have read it, a V stage only after both
                    // P V MMAs, so the next K tile is on its way a P V earlier
                    const uint32_t par = ((item / NSTAGE) & 1) ^ 1;
                    if (!mbar_wait(&k_empty[st], par, abort, status)) { ok = false; break; }
                    mbar_expect_tx(&k_full[st], L::TILE);
                    bulk_load(sm + L::OFF_K + st * L::TILE, block(kg, a.tk, b, j, h, L::TILE), L::TILE,
                              &k_full[st]);
                    ++k_issued;
                    if (!mbar_wait(&v_empty[st], par, abort, status)) { ok = false; break; }
                    mbar_expect_tx(&v_full[st], L::VTILE);
                    bulk_load(sm + L::OFF_V + st * L::VTILE, block(vg, a.tv, b, j, h, L::VTILE),
                              L::VTILE, &v_full[st]);
                    ++v_issued;
                }
            }
            if (!ok) {  // let copies still in flight land before the CTA exits
                volatile int never = 0;
                for (int i = k_issued - NSTAGE; i < k_issued; ++i)
                    if (i >= 0) mbar_wait(&k_full[i % NSTAGE], (i / NSTAGE) & 1, &never, status);
                for (int i = v_issued - NSTAGE; i < v_issued; ++i)
                    if (i >= 0) mbar_wait(&v_full[i % NSTAGE], (i / NSTAGE) & 1, &never, status);
                if (last_q_unit >= 0)
                    mbar_wait(&q_full[last_q_unit & 1], (last_q_unit >> 1) & 1, &never, status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Order per item i: PV0(i), S0(i+1), PV1(i), S1(i+1), so each softmax
        // warpgroup gets its next S right after handing over its P, while the
        // other warpgroup is still busy.  The whole warp runs this loop (its
        // operands stay warp-uniform) and lane 0 issues each MMA and commit; the
        // waits are taken by the whole warp.
        {
            constexpr uint32_t idesc_s = idesc_bf16(BQ, BKV);
            constexpr uint32_t idesc_o = idesc_bf16(BQ, L::NPV, true);
            const int n_items = (u1 - u0) * sc.kt;
            bool ok = true, any = false;
            // the operands of S(i): the K tile and, at a unit's first tile, the
            // unit's Q tiles
            auto wait_s_operands = [&](int i) {
                const int st = i % NSTAGE, j = i % sc.kt, un = i / sc.kt, qb = un & 1;
                if (!mbar_wait_warp(&k_full[st], (i / NSTAGE) & 1, abort, status)) return false;
                if (j == 0 && !mbar_wait_warp(&q_full[qb], (un >> 1) & 1, abort, status)) return false;
                return true;
            };
            // S_g(i) = Q_g K(i)^T (its operands waited for)
            auto issue_s = [&](int i, int g) {
                const int st = i % NSTAGE, j = i % sc.kt, un = i / sc.kt, qb = un & 1;
                const uint32_t aK = smem_u32(sm + L::OFF_K + st * L::TILE);
                const uint32_t aQ = smem_u32(sm + L::OFF_Q + (qb * 2 + g) * L::TILE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    warp_mma_bf16(tmem + g * BKV, sdesc_sw128(aQ + kk * 32), sdesc_sw128(aK + kk * 32),
                                  idesc_s, kk > 0);
                if (L::HAS_B)
                    warp_mma_bf16(tmem + g * BKV, sdesc_sw32(aQ + L::TILE_A), sdesc_sw32(aK + L::TILE_A),
                                  idesc_s, 1);
                warp_mma_commit(&s_full[g]);
                if (g == 1) {
                    warp_mma_commit(&k_empty[st]);  // both S of item i have read K(i)
                    if (j == sc.kt - 1) warp_mma_commit(&q_empty[qb]);  // the unit's Q tiles are read
                }
                any = true;
            };
            if (n_items > 0) {
                ok = wait_s_operands(0);
                fence_after_sync();
                if (ok) {
                    issue_s(0, 0);
                    issue_s(0, 1);
                }
            }
            for (int i = 0; i < n_items && ok; ++i) {
                const int st = i % NSTAGE, j = i % sc.kt;
                const uint32_t aV = smem_u32(sm + L::OFF_V + st * L::VTILE);
                // V(i) and the operands of S(i+1) are waited for here, while the
                // softmax still works on S(i): both landed long ago (their stages
                // were released an item earlier), and no wait then sits between
                // P_g(i) and the MMAs that follow it.  A wait issued right behind
                // a burst of MMAs only answers once they have run.
                if (!mbar_wait_warp(&v_full[st], (i / NSTAGE) & 1, abort, status) ||
                    (i + 1 < n_items && !wait_s_operands(i + 1))) { ok = false; break; }
                for (int g = 0; g < 2 && ok; ++g) {
                    if (!mbar_wait_warp(&p_full[g], i & 1, abort, status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t tP = tmem + g * BKV;  // P_g over the first 64 columns of S_g
                    const uint32_t tO = tmem + 256 + g * 128;
#pragma unroll
                    for (int ks = 0; ks < BKV / 16; ++ks)
                        warp_mma_bf16_ts(tO, tP + ks * 8, sdesc_sw128_mn(aV + ks * 2048, L::TILE_A),
                                         idesc_o, (j | ks) > 0);
                    warp_mma_commit(&o_full[g]);
                    if (g == 1) warp_mma_commit(&v_empty[st]);  // both P V of item i have read V(i)
                    if (i + 1 < n_items) issue_s(i + 1, g);
                }
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                warp_mma_commit(drain);
                volatile int never = 0;
                mbar_wait_warp(drain, 0, &never, status);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ output stores
        // Each softmax warpgroup stages its unit's 128 normalised output rows
        // in shared memory and moves on; lane 0 here writes them out with one
        // tensor store per query tile (rows past nq are not written).
        if (lane == 0) {
            prefetch_tensormap(&omap);
            int un_count = 0;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u, ++un_count) {
                int b, h, qp;
                decode(a, sc, u, b, h, qp);
                for (int g = 0; g < 2; ++g) {
                    if (!mbar_wait(&stage_full[g], un_count & 1, abort, status)) { ok = false; break; }
                    const int q0 = qp * 2 * BQ + g * BQ;  // query index of staging row 0
                    if (q0 < a.nq) {
                        tma_store_3d(&omap, sm + L::OFF_STG + g * L::STG, h * d, q0, b);
                        bulk_commit();
                    }
                    bulk_wait_read_all();  // the staging rows have been read
                    mbar_arrive(&stage_free[g]);
                }
            }
            bulk_wait_all();  // the output is in global memory before the CTA exits
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax warpgroups
        // The output accumulates in TMEM (each P V adds onto it).  Scores are
        // exponentiated against a per-row reference max that is only raised
        // when a tile's max exceeds it by more than 2^8 (weights then stay
        // below 256, harmless in fp32); raising it rescales the row of O in
        // TMEM, after the previous P V has landed.  TMEM loads and stores are
        // warp-collective, so every decision in front of one is taken by the
        // whole warp: wait results are combined over the warp, and a rescale
        // runs when any row of the warp needs it (the others scale by 1).
        const int g = (warp - 4) / 4;
        auto wait_all = [&](uint64_t *bar, uint32_t par) {
            return __all_sync(0xffffffffu, mbar_wait(bar, par, abort, status));
        };
        const int r = (warp % 4) * 32 + lane;  // query row of the tile = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + g * BKV;
        const uint32_t t_o = tmem + lane_base + 256 + g * 128;
        const float sl2 = a.scale * 1.4426950408889634f;
        // staging rows as the tensor store reads them: packed at nch * 16 bytes,
        // or, for nch == 8, 128 bytes with the 128-byte swizzle (16-byte piece u
        // of row r at (u ^ (r & 7)) * 16), so that no two lanes of a store
        // phase hit the same banks
        const bool sw128 = nch == 8;
        int item = 0, un_count = 0;
        bool ok = true;
        for (int u = u0; u < u1 && ok; ++u) {
            int b, h, qp;
            decode(a, sc, u, b, h, qp);
            float m_ref = -INFINITY, l_i = 0.f;
            for (int j = 0; j < sc.kt; ++j, ++item) {
                const uint32_t ph = item & 1;
                const int nvalid = min(BKV, a.nk - j * BKV);
                if (!wait_all(&s_full[g], ph)) { ok = false; break; }
                fence_after_sync();
                // the whole row of S: four loads, one wait
                uint32_t sv[BKV];
                tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
                tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(sv + 64));
                tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(sv + 96));
                tmem_ld_wait();
                if (nvalid < BKV) {  // ragged last key tile: masked keys score -inf
#pragma unroll
                    for (int e = 0; e < BKV; ++e)
                        if (e >= nvalid) sv[e] = __float_as_uint(-INFINITY);
                }
                // row max over 8 independent chains of three-input maxima
                float mx[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) mx[c] = __uint_as_float(sv[c]);
#pragma unroll
                for (int e = 8; e < BKV; e += 16)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        mx[c] = e + 8 + c < BKV
                                    ? fmax3(mx[c], __uint_as_float(sv[e + c]), __uint_as_float(sv[e + 8 + c]))
                                    : fmaxf(mx[c], __uint_as_float(sv[e + c]));
                float tmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
                tmax *= sl2;
                const bool raise = tmax > m_ref + 8.f;  // raise the reference; O so far shrinks by alpha
                if (__any_sync(0xffffffffu, raise)) {
                    const float alpha = !raise ? 1.f : (m_ref == -INFINITY ? 0.f : ex2_approx(m_ref - tmax));
                    if (j > 0) {
                        // O holds P V up to tile j-1 once that MMA has landed
                        if (!wait_all(&o_full[g], ph ^ 1)) { ok = false; break; }
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
                    if (raise) m_ref = tmax;
                }
                const float ref = m_ref;
                float ps[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) ps[c] = 0.f;
                // P as bf16 pairs, written over the first 64 columns of S.  With
                // SUMV the row sum comes out of P V (V's ones column) instead of
                // being added up here.
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float x0 = fmaf(__uint_as_float(sv[64 * half + 2 * c]), sl2, -ref);
                        const float x1 = fmaf(__uint_as_float(sv[64 * half + 2 * c + 1]), sl2, -ref);
                        const float p0 = ex2_approx(x0);
                        const float p1 = ex2_approx(x1);
                        if (!SUMV) {
                            ps[(2 * c) & 7] += p0;
                            ps[(2 * c + 1) & 7] += p1;
                        }
                        pk[c] = pack_bf16(p0, p1);
                    }
                    tmem_st32(t_s + 32 * half, pk);
                }
                tmem_st_wait();
                if (!SUMV)
                    l_i += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                fence_before_sync();
                mbar_arrive(&p_full[g]);
            }
            if (!ok) break;
            // the unit's last P V, then O / l into the staging rows (once the
            // store warp has read the previous unit's); warp 2 writes them out
            if (!wait_all(&o_full[g], (item - 1) & 1)) { ok = false; break; }
            if (!wait_all(&stage_free[g], (un_count & 1) ^ 1)) { ok = false; break; }
            fence_after_sync();
            uint8_t *stg = sm + L::OFF_STG + g * L::STG;
            {
                uint32_t ov[DPAD];
                tmem_ld32(t_o, *reinterpret_cast<uint32_t(*)[32]>(ov));
                tmem_ld32(t_o + 32, *reinterpret_cast<uint32_t(*)[32]>(ov + 32));
                if (DPAD > 64) tmem_ld16(t_o + 64, *reinterpret_cast<uint32_t(*)[16]>(ov + 64));
                tmem_ld_wait();
                // SUMV: column d = DPAD - 8 of O holds the row sum of P
                const float lrow = SUMV ? __uint_as_float(ov[DPAD - 8]) : l_i;
                const float inv = 1.f / lrow;
                // the row's log-sum-exp of the scaled scores, base 2 (for a backward pass)
                if (a.lse) {
                    const int q = qp * 2 * BQ + g * BQ + r;
                    if (q < a.nq) a.lse[((long)b * a.heads + h) * a.nq + q] = m_ref + __log2f(lrow);
                }
#pragma unroll
                for (int u = 0; u < DPAD / 8; ++u)
                    if (u < nch) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(ov[8 * u + 0]) * inv, __uint_as_float(ov[8 * u + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(ov[8 * u + 2]) * inv, __uint_as_float(ov[8 * u + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(ov[8 * u + 4]) * inv, __uint_as_float(ov[8 * u + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(ov[8 * u + 6]) * inv, __uint_as_float(ov[8 * u + 7]) * inv);
                        const int piece = sw128 ? (u ^ (r & 7)) : u;
                        *reinterpret_cast<uint4 *>(stg + r * nch * 16 + piece * 16) = v;
                    }
            }
            fence_before_sync();  // O is read before the next unit's first P V overwrites it
            fence_async_smem();   // the staging rows are visible to the tensor store
            mbar_arrive(&stage_full[g]);
            ++un_count;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int DPAD, bool SUMV>
cudaError_t launch_rows(const AttnArgs &a, cudaStream_t s) {
    using L = RowsLayout<DPAD>;
    int *status = device_status_ptr();
    if (!status) return cudaErrorInvalidValue;
    // the tiles are the tiled-head-layout blocks the projections wrote
    if (a.tq.mode != THL_IDENTITY || a.tk.mode != THL_IDENTITY || a.tv.mode != THL_IDENTITY ||
        a.tq.vpad || a.tk.vpad || !a.tv.vpad || L::TILE != (int)thl_block_bytes(a.d, 0) ||
        L::VTILE != (int)thl_block_bytes(a.d, 1))
        return cudaErrorInvalidValue;
    // the output tiles go out as tensor stores of (d columns, 128 rows) boxes
    CUtensorMap omap;
    if (reinterpret_cast<uintptr_t>(a.o) % 16 || a.ldo % 8 ||
        !encode_map_out_rows_bf16(&omap, a.o, (uint64_t)a.heads * a.d, (uint64_t)a.nq,
                                  (uint64_t)a.B, (uint64_t)a.ldo * 2,
                                  (uint64_t)a.q_bstride * a.ldo * 2, (uint32_t)a.d, BQ, a.d == 64))
        return cudaErrorInvalidValue;
    RowsSched sc;
    sc.qp = (a.nq + 2 * BQ - 1) / (2 * BQ);
    sc.kt = (a.nk + BKV - 1) / BKV;
    sc.units = a.B * a.heads * sc.qp;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int grid = sc.units < sms ? sc.units : sms;
    cudaError_t e = cudaFuncSetAttribute(attn_rows_kernel<DPAD, SUMV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_rows_kernel<DPAD, SUMV>, dim3(grid), dim3(kThreads), L::BYTES, s, a, sc,
                      omap, status);
}

}  // namespace

cudaError_t launch_attention_rows_tc(const AttnArgs &a, cudaStream_t s) {
    // d = 72: the row sums come out of P V through V's ones column (column 72);
    // other widths (8 .. 80, multiples of 8) sum P in the softmax
    if (a.d < 8 || a.d > 80 || a.d % 8) return cudaErrorInvalidValue;
    if (a.d == 72 && a.tv.ones) return launch_rows<80, true>(a, s);
    return a.d <= 64 ? launch_rows<64, false>(a, s) : launch_rows<80, false>(a, s);
}

}  // namespace ptdit
