// Row-mode attention core on the tensor cores: proxy self-attention and
// latent -> proxy cross-attention of GIIM (Qihoo-T2X reading note, §3
// Method, Eq. GIIM), the text cross-attention of the complete PT-Block, and
// full self-attention (the dense comparator of the complexity paragraph).
// Queries are rows [0, nq) and keys rows [0, nk) of each batch item; head h
// is columns h*d .. h*d+d-1.
//
// One persistent CTA per SM; a unit is two 128-row query tiles (A, B) of one
// (batch item, head).  The unit's work is a sequence of items, one per
// (key tile j, query tile t) in the order (0,A), (0,B), (1,A), (1,B), ...,
// so both query tiles use each K/V tile while it is in shared memory.
//   warp 0       loader: the unit's two Q tiles (double buffered across
//                units) and each key tile's K and V into a two-stage ring,
//                each one contiguous bulk copy: the projections wrote Q, K and
//                V in tiled head layout (thl.cuh), so a (tile, head) block is
//                already the swizzled shared-memory tile (V padded to 128
//                columns for d > 64: one P V MMA per K step).
//   warp 1       MMA issuer: S(i) = Q_t K_j^T into score buffer i % 2 of TMEM,
//                and, once the softmax has written P(i) over it, O_t += P(i) V_j
//                with P read from TMEM; then S(i + 2).  The scores of the next
//                item are computed while the softmax of this one runs, and a
//                P V never waits for the next item's scores.
//   warps 4-7, 8-11   softmax: both warpgroups work on every item, thread r of
//                warpgroup g owning keys 64 g .. 64 g + 63 of query row r (its
//                TMEM lane).  The two threads of a row exchange their maxima
//                through shared memory (an mbarrier per warp pair and item
//                parity), keep one reference max per query tile that only rises
//                by more than 2^8 (rescaling that tile's O in TMEM after its
//                previous P V has landed), exponentiate 64 scores each with
//                ex2.approx and write their half of P as bf16 pairs.  After a
//                unit's last item they read O_A and O_B, divide by the row sum
//                (V's ones column when d = 72, else the two halves' sums) and
//                store each warp's 32 rows through its own staging rows, with
//                consecutive lanes on consecutive 16-byte pieces of a row.
// TMEM: score buffers at columns 0 and 128, O_A at 256, O_B at 384.
// Every wait is bounded (2 s); the softmax warps decide per warp.
#include <math.h>

#include "tc_util.cuh"
#include "thl.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128, BKV = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr int NSTAGE = 2;  // K/V ring depth

template <int DPAD>
struct RowsLayout {
    static constexpr bool HAS_B = DPAD > 64;             // head columns 64..79
    static constexpr int TILE_A = BQ * 64 * 2;           // 128 rows x 128 B, 128-byte swizzle
    static constexpr int TILE_B = HAS_B ? BQ * 16 * 2 : 0;  // 128 rows x 32 B, 32-byte swizzle
    static constexpr int TILE = TILE_A + TILE_B;         // a Q or K tile (K-major)
    // V is the MN-major operand of P V, padded to 128 columns for d > 64 (one
    // N = 128 MMA per K step costs what an N = 64 one does)
    static constexpr int VTILE = HAS_B ? 2 * TILE_A : TILE_A;
    static constexpr int NPV = HAS_B ? 128 : 64;         // N of the P V MMA
    static constexpr int OFF_Q = 0;                      // [unit parity][query tile]
    static constexpr int OFF_K = 4 * TILE;               // [stage]
    static constexpr int OFF_V = OFF_K + NSTAGE * TILE;  // [stage]
    static constexpr int OFF_XM = OFF_V + NSTAGE * VTILE;  // float [item parity][half][128]
    static constexpr int OFF_XL = OFF_XM + 2 * 2 * BQ * 4;  // float [query tile][half][128]
    // output staging: 32 rows of at most 6 16-byte units per softmax warp
    static constexpr int WSTG = 32 * 96;
    static constexpr int OFF_STG = OFF_XL + 2 * 2 * BQ * 4;
    static constexpr int OFF_BAR = OFF_STG + 8 * WSTG;
    // q_full[2], q_empty[2], kv_full[2], kv_empty[2], s_full[2], p_full[2],
    // pv_done[2], o_full[2], xbar[4][2], lbar[4], drain
    static constexpr int NBARS = 16 + 8 + 4 + 1;
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
    attn_rows_kernel(const __grid_constant__ AttnArgs a, RowsSched sc, int *status) {
    using L = RowsLayout<DPAD>;
    extern __shared__ uint8_t sm_raw[];
    // TMA destinations: align the base to 1 KB (tile offsets are multiples of 1 KB)
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *q_full = bars, *q_empty = bars + 2, *kv_full = bars + 4, *kv_empty = bars + 6;
    uint64_t *s_full = bars + 8, *p_full = bars + 10, *pv_done = bars + 12, *o_full = bars + 14;
    uint64_t *xbar = bars + 16;  // [warp pair][item parity]
    uint64_t *lbar = bars + 24;  // [warp pair]
    uint64_t *drain = bars + 28;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, nch = d / 8;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 2 * BQ);  // both threads of every row
            mbar_init(&pv_done[s], 1);
            mbar_init(&o_full[s], 1);
        }
        for (int w = 0; w < 4; ++w) {
            mbar_init(&xbar[2 * w], 64);
            mbar_init(&xbar[2 * w + 1], 64);
            mbar_init(&lbar[w], 64);
        }
        mbar_init(drain, 1);
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
    const int kt = sc.kt;

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
            int kc = 0, last_q_unit = -1;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                int b, h, qp;
                decode(a, sc, u, b, h, qp);
                const int un = u - u0, qb = un & 1;
                if (!mbar_wait(&q_empty[qb], ((un >> 1) & 1) ^ 1, abort, status)) { ok = false; break; }
                // the unit's second query tile may lie past the last one: the last
                // tile is loaded twice then (its second results are not stored)
                mbar_expect_tx(&q_full[qb], 2 * L::TILE);
                for (int g = 0; g < 2; ++g)
                    bulk_load(sm + L::OFF_Q + (qb * 2 + g) * L::TILE,
                              block(qg, a.tq, b, min(2 * qp + g, a.tq.tiles - 1), h, L::TILE),
                              L::TILE, &q_full[qb]);
                last_q_unit = un;
                for (int j = 0; j < kt; ++j, ++kc) {
                    const int st = kc % NSTAGE;
                    if (!mbar_wait(&kv_empty[st], ((kc / NSTAGE) & 1) ^ 1, abort, status)) { ok = false; break; }
                    mbar_expect_tx(&kv_full[st], L::TILE + L::VTILE);
                    bulk_load(sm + L::OFF_K + st * L::TILE, block(kg, a.tk, b, j, h, L::TILE), L::TILE,
                              &kv_full[st]);
                    bulk_load(sm + L::OFF_V + st * L::VTILE, block(vg, a.tv, b, j, h, L::VTILE),
                              L::VTILE, &kv_full[st]);
                }
            }
            if (!ok) {  // let copies still in flight land before the CTA exits
                volatile int never = 0;
                for (int i = kc - NSTAGE; i < kc; ++i)
                    if (i >= 0) mbar_wait(&kv_full[i % NSTAGE], (i / NSTAGE) & 1, &never, status);
                if (last_q_unit >= 0)
                    mbar_wait(&q_full[last_q_unit & 1], (last_q_unit >> 1) & 1, &never, status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(BQ, BKV);
            constexpr uint32_t idesc_o = idesc_bf16(BQ, L::NPV, true);
            const int per_unit = 2 * kt;
            const int n_items = (u1 - u0) * per_unit;
            bool ok = true, any = false;
            // S(i) = Q_t K_j^T into score buffer i % 2 (after P V(i - 2), issued
            // before it, has read P(i - 2) out of that buffer: tcgen05.mma
            // instructions of one thread run in issue order)
            auto issue_s = [&](int i) {
                const int un = i / per_unit, il = i % per_unit, j = il >> 1, t = il & 1;
                const int kc = un * kt + j, st = kc % NSTAGE, qb = un & 1;
                if (t == 0) {
                    if (!mbar_wait(&kv_full[st], (kc / NSTAGE) & 1, abort, status)) return false;
                    if (j == 0 && !mbar_wait(&q_full[qb], (un >> 1) & 1, abort, status)) return false;
                    fence_after_sync();
                }
                const uint32_t aK = smem_u32(sm + L::OFF_K + st * L::TILE);
                const uint32_t aQ = smem_u32(sm + L::OFF_Q + (qb * 2 + t) * L::TILE);
                const uint32_t tS = tmem + (i & 1) * BKV;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tS, sdesc_sw128(aQ + kk * 32), sdesc_sw128(aK + kk * 32), idesc_s,
                             kk > 0);
                if (L::HAS_B)
                    mma_bf16(tS, sdesc_sw32(aQ + L::TILE_A), sdesc_sw32(aK + L::TILE_A), idesc_s, 1);
                mma_commit(&s_full[i & 1]);
                if (t == 1 && j == kt - 1) mma_commit(&q_empty[qb]);  // the unit's Q tiles are read
                any = true;
                return true;
            };
            if (n_items > 0) ok = issue_s(0);
            if (ok && n_items > 1) ok = issue_s(1);
            for (int i = 0; i < n_items && ok; ++i) {
                const int un = i / per_unit, il = i % per_unit, j = il >> 1, t = il & 1;
                const int kc = un * kt + j, st = kc % NSTAGE;
                if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, abort, status)) { ok = false; break; }
                fence_after_sync();
                const uint32_t aV = smem_u32(sm + L::OFF_V + st * L::VTILE);
                const uint32_t tP = tmem + (i & 1) * BKV;  // P over the first 64 columns
                const uint32_t tO = tmem + 256 + t * 128;
#pragma unroll
                for (int ks = 0; ks < BKV / 16; ++ks)
                    mma_bf16_ts(tO, tP + ks * 8, sdesc_sw128_mn(aV + ks * 2048, L::TILE_A), idesc_o,
                                (j | ks) > 0);
                mma_commit(&pv_done[t]);
                if (t == 1) mma_commit(&kv_empty[st]);  // both S and both P V of key tile j
                if (j == kt - 1) mma_commit(&o_full[t]);
                if (i + 2 < n_items) ok = issue_s(i + 2);
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                mma_commit(drain);
                volatile int never = 0;
                mbar_wait(drain, 0, &never, status);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax
        // TMEM loads and stores are warp-collective: every decision in front of
        // one is taken by the whole warp (bounded waits per warp; a rescale runs
        // when any row of the warp needs it, the others scale by 1).
        const int hf = (warp - 4) / 4, w = warp % 4;
        const int r = w * 32 + lane;  // query row of the tile = TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(w * 32) << 16;
        float *xm = reinterpret_cast<float *>(sm + L::OFF_XM);  // [item parity][half][row]
        float *xl = reinterpret_cast<float *>(sm + L::OFF_XL);  // [query tile][half][row]
        const float sl2 = a.scale * 1.4426950408889634f;
        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);
        // output units (8 columns) of this thread: half 0 the first ceil(nch / 2)
        const int nu0 = (nch + 1) / 2, ub = hf ? nu0 : 0, nu = hf ? nch - nu0 : nu0;
        const int pitch = nu * 16 + (nu % 2 == 0 ? 16 : 0);  // an odd number of 16-byte units
        uint8_t *stg = sm + L::OFF_STG + (warp - 4) * L::WSTG;
        // O columns this thread rescales: half 0 [0, 64), half 1 [64, DPAD)
        const int oc0 = hf ? 64 : 0, oc1 = hf ? DPAD : (DPAD < 64 ? DPAD : 64);
        int it = 0, un_count = 0;
        bool ok = true;
        for (int u = u0; u < u1 && ok; ++u, ++un_count) {
            int b, h, qp;
            decode(a, sc, u, b, h, qp);
            float m_ref[2] = {-INFINITY, -INFINITY}, l_i[2] = {0.f, 0.f};
            for (int j = 0; j < kt && ok; ++j) {
                const int nvalid = min(BKV, a.nk - j * BKV);
#pragma unroll
                for (int t = 0; t < 2; ++t, ++it) {
                    if (!mbar_wait_warp(&s_full[it & 1], (it >> 1) & 1, abort, status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t t_s = tmem + lane_base + (it & 1) * BKV;
                    uint32_t sv[64];
                    tmem_ld32(t_s + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(sv));
                    tmem_ld32(t_s + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                    tmem_ld_wait();
                    if (nvalid < BKV) {  // ragged last key tile: absent keys score -inf
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            if (64 * hf + e >= nvalid) sv[e] = __float_as_uint(-INFINITY);
                    }
                    float mx[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) mx[c] = __uint_as_float(sv[c]);
#pragma unroll
                    for (int e = 4; e < 64; e += 8)
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            mx[c] = e + 4 + c < 64
                                        ? fmax3(mx[c], __uint_as_float(sv[e + c]), __uint_as_float(sv[e + 4 + c]))
                                        : fmaxf(mx[c], __uint_as_float(sv[e + c]));
                    const float mine = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                    // the row's other half, through shared memory: both threads of the
                    // row arrive on the warp pair's barrier of this item parity (and
                    // have both read their scores before either writes P over them)
                    float *xs = xm + (it & 1) * 2 * BQ;
                    xs[hf * BQ + r] = mine;
                    mbar_arrive(&xbar[2 * w + (it & 1)]);
                    if (!mbar_wait_warp(&xbar[2 * w + (it & 1)], (it >> 1) & 1, abort, status)) { ok = false; break; }
                    const float tmax = fmaxf(mine, xs[(1 - hf) * BQ + r]) * sl2;
                    const bool raise = tmax > m_ref[t] + 8.f;  // O so far shrinks by alpha
                    if (__any_sync(0xffffffffu, raise)) {
                        const float alpha =
                            !raise ? 1.f : (m_ref[t] == -INFINITY ? 0.f : ex2_approx(m_ref[t] - tmax));
                        if (j > 0 && oc0 < oc1) {
                            // O_t holds P V up to key tile j - 1 once that MMA has landed
                            // (pv_done[t] completes once per P V of query tile t)
                            const int pvc = un_count * kt + j - 1;
                            if (!mbar_wait_warp(&pv_done[t], pvc & 1, abort, status)) { ok = false; break; }
                            fence_after_sync();
                            const uint32_t t_o = tmem + lane_base + 256 + t * 128;
#pragma unroll
                            for (int c0 = 0; c0 < 64; c0 += 16) {
                                if (oc0 + c0 >= oc1) break;
                                uint32_t ov[16];
                                tmem_ld16(t_o + oc0 + c0, ov);
                                tmem_ld_wait();
#pragma unroll
                                for (int e = 0; e < 16; ++e)
                                    ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                                tmem_st16(t_o + oc0 + c0, ov);
                            }
                            tmem_st_wait();
                        }
                        l_i[t] *= alpha;
                        if (raise) m_ref[t] = tmax;
                    }
                    const float ref = m_ref[t];
                    float ps[4] = {0.f, 0.f, 0.f, 0.f};
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), sl2, -ref));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -ref));
                        if (!SUMV) ps[c & 3] += p0 + p1;
                        pk[c] = pack_bf16(p0, p1);
                    }
                    // keys 64 hf .. 64 hf + 63 as bf16 pairs: columns 32 hf .. 32 hf + 31
                    tmem_st32(t_s + 32 * hf, pk);
                    tmem_st_wait();
                    if (!SUMV) l_i[t] += (ps[0] + ps[1]) + (ps[2] + ps[3]);
                    fence_before_sync();
                    mbar_arrive(&p_full[it & 1]);
                }
            }
            if (!ok) break;
            // ---- the unit's outputs: O_A, then O_B
#pragma unroll 1
            for (int t = 0; t < 2; ++t) {
                float lsum = 0.f;
                if (!SUMV) {  // the row sum of P: both halves (lbar completes once per tile)
                    float *xt = xl + t * 2 * BQ;
                    xt[hf * BQ + r] = l_i[t];
                    mbar_arrive(&lbar[w]);
                    if (!mbar_wait_warp(&lbar[w], t, abort, status)) { ok = false; break; }
                    lsum = l_i[t] + xt[(1 - hf) * BQ + r];
                }
                if (!mbar_wait_warp(&o_full[t], un_count & 1, abort, status)) { ok = false; break; }
                fence_after_sync();
                const uint32_t t_o = tmem + lane_base + 256 + t * 128;
                uint32_t ov[40];
#pragma unroll
                for (int v = 0; v < 5; ++v)
                    if (v < nu) tmem_ld8(t_o + 8 * (ub + v), *reinterpret_cast<uint32_t(*)[8]>(ov + 8 * v));
                uint32_t sv8[8];
                if (SUMV) tmem_ld8(t_o + d, sv8);  // V's ones column: the row sum of P
                tmem_ld_wait();
                // O is in registers: the next unit's first P V may overwrite it after
                // this thread's next arrival on p_full
                fence_before_sync();
                const float inv = 1.f / (SUMV ? __uint_as_float(sv8[0]) : lsum);
#pragma unroll
                for (int v = 0; v < 5; ++v)
                    if (v < nu) {
                        uint4 o;
                        o.x = pack_bf16(__uint_as_float(ov[8 * v + 0]) * inv, __uint_as_float(ov[8 * v + 1]) * inv);
                        o.y = pack_bf16(__uint_as_float(ov[8 * v + 2]) * inv, __uint_as_float(ov[8 * v + 3]) * inv);
                        o.z = pack_bf16(__uint_as_float(ov[8 * v + 4]) * inv, __uint_as_float(ov[8 * v + 5]) * inv);
                        o.w = pack_bf16(__uint_as_float(ov[8 * v + 6]) * inv, __uint_as_float(ov[8 * v + 7]) * inv);
                        *reinterpret_cast<uint4 *>(stg + lane * pitch + v * 16) = o;
                    }
                __syncwarp();
                // the warp's 32 rows x nu units: consecutive lanes on consecutive units
                const long q0 = (long)(2 * qp + t) * BQ + w * 32;  // query index of staging row 0
                __nv_bfloat16 *obase = og + (long)b * a.q_bstride * a.ldo + (long)h * d + 8 * ub;
                for (int i = lane; i < 32 * nu; i += 32) {
                    const int row = i / nu, v = i - row * nu;
                    if (q0 + row < a.nq)
                        *reinterpret_cast<uint4 *>(obase + (q0 + row) * a.ldo + v * 8) =
                            *reinterpret_cast<const uint4 *>(stg + row * pitch + v * 16);
                }
                __syncwarp();  // the staging rows are free again
            }
        }
    }
    if (*abort) {
        // a wait gave up: let bulk copies still in flight into this CTA land
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
                      status);
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
