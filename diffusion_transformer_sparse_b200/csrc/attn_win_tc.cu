// Window and shifted-window self-attention of TCM on the tensor cores
// (Qihoo-T2X reading note, §3 Method, Eq. TCM): windows of 64 tokens (2D,
// packed two per 128-row tile) or 128 tokens (3D, one per tile) of the grid
// rolled by -shift, pairs that the roll wrapped masked out.
//
// One persistent CTA per SM; a unit is one tile (128 query rows = its own 128
// key rows) of one head.  Three load buffers keep up to three units' operands
// in flight while two TMEM slots (S/P and O) alternate between the units:
//   warp 2       loader: the window projection wrote Q, K and V in tiled head
//                layout (thl.cuh) with window tiles, so a unit's Q, K and V
//                are three contiguous 20 KB blocks, each already the swizzled
//                shared-memory tile (columns 0..63 with the 128-byte swizzle,
//                64..79 with the 32-byte swizzle, zeros past the head and in
//                rows without a window, V's column d = 1 when d = 72): three
//                bulk copies into the unit's buffer, Q and K on one barrier and
//                V on another.  It also computes the token of each tile row
//                with the roll/wrap address function (for the key masks and the
//                output rows) and builds the key masks (window in tile x wrap
//                bits) with ballots, once per (batch item, tile) and buffer:
//                the heads of one tile follow each other.
//   warp 1       MMA issuer: S = Q K^T into the unit's TMEM slot, then O = P V
//                with P read from TMEM (the softmax writes it over S) and V
//                from shared memory as the MN-major operand: columns 0..63 in
//                one N = 64 MMA per K step (128-byte swizzle), 64..79 in one
//                N = 16 MMA (32-byte swizzle).  Order: S(0), S(1), then per
//                unit k: P V(k), S(k + 2).
//   warps 4-7, 8-11   softmax of TMEM slot 0 / 1 (units k = 0, 2, ... /
//                1, 3, ...): thread r owns query row r, reads only its own
//                window's scores, masks, exponentiates in fp32 and writes P as
//                bf16 pairs into TMEM.  Then each warp reads its 32 output rows
//                from TMEM, scales them by 1/l, stages them in the unit's Q/K
//                area (the tensor cores are done with it) and stores them with
//                consecutive lanes on consecutive 16-byte pieces of a token
//                row; when its four warps are done the buffer goes back to the
//                loader.
// With SUMV the row sums of P come out of P V through V's ones column.
// Every wait is bounded (2 s, or the limit ptdit_debug_wait_limit sets); the
// loader and softmax warps decide to give up per warp, never per lane.
#include <math.h>

#include "tc_util.cuh"
#include "thl.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;  // per slot: S/P 128 columns, O 128 columns
// Key masks of a tile: one per (window in tile, wrap code).  Windows of 16, 32
// or 64 tokens (8, 4 or 2 per tile, each inside one 64-key half of the tile)
// keep 64 bits per mask, the bits of their half: up to 64 masks.  A window of
// 128 tokens keeps 128 bits per mask: 8 masks.  512 bytes per buffer either way.
constexpr int kMaskWords = 128;
constexpr int NBUF = 3;              // load buffers: units whose operands are in flight

template <int DPAD>
struct WinLayout {
    static constexpr bool HAS_B = DPAD > 64;                   // head columns 64..79
    static constexpr int TILE_A = BQ * 128;                    // columns 0..63, 128-byte swizzle
    static constexpr int TILE_B = HAS_B ? BQ * 32 : 0;         // columns 64..79, 32-byte swizzle
    static constexpr int TILE = TILE_A + TILE_B;               // a Q or K tile (K-major)
    static constexpr int BUF = 3 * TILE;                       // Q, K, V of one unit
    static constexpr int OFF_INFO = NBUF * BUF;                // int info[NBUF][128]
    static constexpr int OFF_ROW = OFF_INFO + NBUF * BQ * 4;   // int row[NBUF][128] (token rows)
    static constexpr int OFF_MASK = OFF_ROW + NBUF * BQ * 4;   // uint32 kmask[NBUF][kMaskWords]
    // output staging: 32 rows (pitch <= 160 B) per softmax warp
    static constexpr int WSTG = 32 * 160;
    static constexpr int OFF_STG = OFF_MASK + NBUF * kMaskWords * 4;
    static constexpr int OFF_OROW = OFF_STG + 8 * WSTG;       // int orow[8][32]: rows being stored
    static constexpr int OFF_BAR = OFF_OROW + 8 * 32 * 4;
    // qk_full[NBUF], v_full[NBUF], buf_free[NBUF], s_full[2], p_full[2], o_full[2], o_free[2], drain
    static constexpr int NBARS = 3 * NBUF + 9;
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16 + 1024;  // + base alignment slack
    static_assert(TILE_A % 1024 == 0 && TILE % 1024 == 0 && BUF % 1024 == 0,
                  "swizzled tiles stay 1 KB aligned");
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct WinSched {
    int tiles;  // tiles per batch item
    int units;  // B x tiles x heads
    unsigned long long wait_ns;  // limit of every wait for work (the final drain keeps 2 s)
};

template <int DPAD, bool SUMV>
__global__ void __launch_bounds__(kThreads, 1)
    attn_win_kernel(const __grid_constant__ AttnArgs a, WinSched sc, int *status) {
    using L = WinLayout<DPAD>;
    extern __shared__ uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    int *info = reinterpret_cast<int *>(sm + L::OFF_INFO);
    int *rowsm = reinterpret_cast<int *>(sm + L::OFF_ROW);  // B * N < 2^31 (checked by the API)
    uint32_t *kmask = reinterpret_cast<uint32_t *>(sm + L::OFF_MASK);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *qk_full = bars, *v_full = bars + NBUF, *buf_free = bars + 2 * NBUF;
    uint64_t *s_full = bars + 3 * NBUF, *p_full = s_full + 2, *o_full = s_full + 4;
    uint64_t *o_free = s_full + 6, *drain = s_full + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, n = a.geom.n;

    if (threadIdx.x == 0) {
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&qk_full[b], 32);  // the loader's 32 lanes (rows and masks) + Q, K bytes
            mbar_init(&v_full[b], 1);
            mbar_init(&buf_free[b], 1);  // the unit's P V has read its operands
        }
        for (int g = 0; g < 2; ++g) {
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
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    pdl_wait();  // the projection that wrote Q, K and V has completed
    pdl_trigger();

    const int u0 = (int)((long)blockIdx.x * sc.units / gridDim.x);
    const int u1 = (int)((long)(blockIdx.x + 1) * sc.units / gridDim.x);
    const int nunits = u1 - u0;  // local unit k: buffer k % NBUF, TMEM slot k % 2

    if (warp == 2) {
        // ------------------------------------------------------------ loader
        const uint8_t *qg = static_cast<const uint8_t *>(a.q);
        const uint8_t *kg = static_cast<const uint8_t *>(a.k);
        const uint8_t *vg = static_cast<const uint8_t *>(a.v);
        const WinGeom &geo = a.geom;
        const int pack = BQ / n;
        int held0 = -1, held1 = -1, held2 = -1;  // (batch item, tile) whose rows each buffer holds
        for (int k = 0; k < nunits; ++k) {
            const int u = u0 + k, bf = k % NBUF;
            const int h = u % a.heads, rest = u / a.heads, tile = rest % sc.tiles,
                      b = rest / sc.tiles;
            if (!mbar_wait_warp(&buf_free[bf], ((k / NBUF) & 1) ^ 1, abort, status, sc.wait_ns))
                break;
            uint8_t *sQ = sm + bf * L::BUF, *sK = sQ + L::TILE, *sV = sK + L::TILE;
            if (lane == 0) {
                const long blk = ((long)b * sc.tiles + tile) * a.heads + h;
                mbar_expect_tx_only(&qk_full[bf], 2 * L::TILE);
                bulk_load(sQ, qg + blk * L::TILE, L::TILE, &qk_full[bf]);
                bulk_load(sK, kg + blk * L::TILE, L::TILE, &qk_full[bf]);
                mbar_expect_tx(&v_full[bf], L::TILE);
                bulk_load(sV, vg + blk * L::TILE, L::TILE, &v_full[bf]);
            }
            // rows and masks depend on (batch item, tile) only: the heads of one tile
            // follow each other, so most units find them in their buffer already
            int &held = bf == 0 ? held0 : (bf == 1 ? held1 : held2);
            if (rest != held) {
                held = rest;
                int inf[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int r = q * 32 + lane;
                    const int wit = r / n, win = tile * pack + wit, slot = r - wit * n;
                    int row = -1, in = -1;
                    if (win < geo.nwin) {
                        int wrap;
                        row = static_cast<int>(b * a.k_bstride) + window_token(geo, win, slot, &wrap);
                        in = wit * 8 + wrap;
                    }
                    inf[q] = in;
                    info[bf * BQ + r] = in;
                    rowsm[bf * BQ + r] = row;
                }
                // one key mask per mask key (window in tile, wrap code): the keys of
                // the same window and wrap code, over the window's 64-key half of
                // the tile (windows of up to 64 tokens) or over all 128 keys
                const int nkeys = n < BQ ? (BQ / n) * 8 : 8;
                for (int v = 0; v < nkeys; ++v) {
                    const int half = n < BQ ? ((v >> 3) * n) >> 6 : 0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t bits = __ballot_sync(0xffffffffu, inf[q] == v);
                        if (lane == 0) {
                            if (n >= BQ)
                                kmask[bf * kMaskWords + v * 4 + q] = bits;
                            else if ((q >> 1) == half)
                                kmask[bf * kMaskWords + v * 2 + (q & 1)] = bits;
                        }
                    }
                }
            }
            __syncwarp();
            mbar_arrive(&qk_full[bf]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs the loop with warp-uniform operands; lane 0 issues)
        {
            constexpr uint32_t idesc_s = idesc_bf16(BQ, BQ);
            constexpr uint32_t idesc_o = idesc_bf16(BQ, 64, true);   // V columns 0..63
            constexpr uint32_t idesc_ob = idesc_bf16(BQ, 16, true);  // V columns 64..79
            bool ok = true, any = false;
            // S(k) into TMEM slot k % 2 (after P V(k - 2), issued earlier, has read P(k - 2))
            auto issue_s = [&](int k) {
                const int bf = k % NBUF, g = k & 1;
                if (!mbar_wait_warp(&qk_full[bf], (k / NBUF) & 1, abort, status, sc.wait_ns)) return false;
                fence_after_sync();
                const uint32_t aQ = smem_u32(sm + bf * L::BUF);
                const uint32_t aK = aQ + L::TILE;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    warp_mma_bf16(tmem + g * 256, sdesc_sw128(aQ + kk * 32), sdesc_sw128(aK + kk * 32),
                             idesc_s, kk > 0);
                if (L::HAS_B)
                    warp_mma_bf16(tmem + g * 256, sdesc_sw32(aQ + L::TILE_A), sdesc_sw32(aK + L::TILE_A),
                             idesc_s, 1);
                warp_mma_commit(&s_full[g]);
                any = true;
                return true;
            };
            // O(k) = P(k) V(k), once the softmax has written P(k) and the output of
            // unit k - 2 has been read out of the slot's O columns
            auto issue_pv = [&](int k) {
                const int bf = k % NBUF, g = k & 1;
                if (!mbar_wait_warp(&p_full[g], (k >> 1) & 1, abort, status, sc.wait_ns)) return false;
                if (!mbar_wait_warp(&o_free[g], ((k >> 1) & 1) ^ 1, abort, status, sc.wait_ns))
                    return false;
                if (!mbar_wait_warp(&v_full[bf], (k / NBUF) & 1, abort, status, sc.wait_ns)) return false;
                fence_after_sync();
                const uint32_t aV = smem_u32(sm + bf * L::BUF + 2 * L::TILE);
                const uint32_t tO = tmem + g * 256 + 128;
#pragma unroll
                for (int ks = 0; ks < BQ / 16; ++ks) {
                    warp_mma_bf16_ts(tO, tmem + g * 256 + ks * 8, sdesc_sw128_mn(aV + ks * 2048, L::TILE_A),
                                idesc_o, ks > 0);
                    if (L::HAS_B)
                        warp_mma_bf16_ts(tO + 64, tmem + g * 256 + ks * 8,
                                    sdesc_sw32_mn(aV + L::TILE_A + ks * 512), idesc_ob, ks > 0);
                }
                warp_mma_commit(&o_full[g]);
                warp_mma_commit(&buf_free[bf]);  // S and P V have read the unit's Q, K and V
                return true;
            };
            if (nunits > 0) ok = issue_s(0);
            if (ok && nunits > 1) ok = issue_s(1);
            for (int k = 0; k < nunits && ok; ++k) {
                ok = issue_pv(k);
                if (ok && k + 2 < nunits) ok = issue_s(k + 2);
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                warp_mma_commit(drain);
                volatile int never = 0;
                mbar_wait_warp(drain, 0, &never, status);
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
        // staging row pitch: an odd number of 16-byte units where that fits
        const int pitch = nch * 16 + (nch % 8 == 0 ? 16 : 0);
        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);
        // the row's own keys: its window inside the tile
        // (windows of up to 64 tokens lie inside one 64-key half of the tile)
        const int c_lo = n < BQ ? (r >> 6) << 6 : 0;
        for (int k = g; k < nunits; k += 2) {
            const int u = u0 + k, bf = k % NBUF;
            const uint32_t ph = (k >> 1) & 1;  // phase of this slot's barriers
            const int h = u % a.heads;
            // every wait of these warps is decided by the whole warp (a TMEM load or
            // store, which all 32 lanes must reach, follows each of them)
            if (!mbar_wait_warp(&qk_full[bf], (k / NBUF) & 1, abort, status, sc.wait_ns))
                break;  // masks and rows
            const int qi = info[bf * BQ + r];
            // this row's token: the buffer's rows may be rewritten once P V has read it
            const int qrow = rowsm[bf * BQ + r];
            uint32_t allow[4] = {0u, 0u, 0u, 0u};
            if (qi >= 0) {
                if (n < BQ) {  // the 64 bits of the row's half
                    const uint2 w2 =
                        *reinterpret_cast<const uint2 *>(kmask + bf * kMaskWords + qi * 2);
                    allow[0] = w2.x;
                    allow[1] = w2.y;
                } else {
                    const uint4 w4 =
                        *reinterpret_cast<const uint4 *>(kmask + bf * kMaskWords + qi * 4);
                    allow[0] = w4.x;
                    allow[1] = w4.y;
                    allow[2] = w4.z;
                    allow[3] = w4.w;
                }
            }
            if (!mbar_wait_warp(&s_full[g], ph, abort, status, sc.wait_ns)) break;
            fence_after_sync();
            float l = 0.f;
            uint32_t pk[64];
            if (n < BQ) {  // 64 keys: one half of the tile (the same half for the whole warp)
                uint32_t sv[64];
                tmem_ld32(t_s + c_lo, *reinterpret_cast<uint32_t(*)[32]>(sv));
                tmem_ld32(t_s + c_lo + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                tmem_ld_wait();
                const uint32_t w0 = allow[0], w1 = allow[1];
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if ((w0 & w1) != 0xffffffffu) {  // some key masked (a window the roll wrapped)
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const bool ok = ((e < 32 ? w0 : w1) >> (e & 31)) & 1u;
                        if (!ok) sv[e] = __float_as_uint(-INFINITY);
                    }
                }
#pragma unroll
                for (int e = 0; e < 64; e += 8)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        mx[c] = fmax3(mx[c], __uint_as_float(sv[e + c]), __uint_as_float(sv[e + 4 + c]));
                const float ref = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sl2;
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pp[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float x0 = fmaf(__uint_as_float(sv[2 * c]), sl2, -ref);
                    const float x1 = fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -ref);
                    const float p0 = ex2_approx(x0);
                    const float p1 = ex2_approx(x1);
                    if (!SUMV) ps[c & 3] += p0 + p1;
                    pp[c] = pack_bf16(p0, p1);
                }
                if (!SUMV) l = (ps[0] + ps[1]) + (ps[2] + ps[3]);
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
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if ((allow[0] & allow[1] & allow[2] & allow[3]) != 0xffffffffu) {  // some key masked
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        if (!((allow[e >> 5] >> (e & 31)) & 1u)) sv[e] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int e = 0; e < 128; e += 8)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        mx[c] = fmax3(mx[c], __uint_as_float(sv[e + c]), __uint_as_float(sv[e + 4 + c]));
                const float ref = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sl2;
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float x0 = fmaf(__uint_as_float(sv[2 * c]), sl2, -ref);
                    const float x1 = fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -ref);
                    const float p0 = ex2_approx(x0);
                    const float p1 = ex2_approx(x1);
                    if (!SUMV) ps[c & 3] += p0 + p1;
                    pk[c] = pack_bf16(p0, p1);
                }
                if (!SUMV) l = (ps[0] + ps[1]) + (ps[2] + ps[3]);
            }
            tmem_st32(t_s, *reinterpret_cast<uint32_t(*)[32]>(pk));
            tmem_st32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
            tmem_st_wait();
            fence_before_sync();
            mbar_arrive(&p_full[g]);
            // O / l to global memory: each warp stages its 32 rows and stores them
            // with consecutive lanes on consecutive 16-byte pieces of a token row;
            // the token rows come from the unit's buffer, whose next load waits
            // for that buffer's release by P V and is two units away
            if (!mbar_wait_warp(&o_full[g], ph, abort, status, sc.wait_ns)) break;
            fence_after_sync();
            uint8_t *stg = sm + L::OFF_STG + (warp - 4) * L::WSTG - (warp % 4) * 32 * pitch;
            int *orow = reinterpret_cast<int *>(sm + L::OFF_OROW) + (warp - 4) * 32;
            orow[lane] = qrow;
            {
                uint32_t ov[DPAD];
                tmem_ld32(t_o, *reinterpret_cast<uint32_t(*)[32]>(ov));
                tmem_ld32(t_o + 32, *reinterpret_cast<uint32_t(*)[32]>(ov + 32));
                if (DPAD > 64) tmem_ld16(t_o + 64, *reinterpret_cast<uint32_t(*)[16]>(ov + 64));
                tmem_ld_wait();
                fence_before_sync();
                mbar_arrive(&o_free[g]);  // O is read: the slot's next P V may overwrite it
                // SUMV: column d = DPAD - 8 of O holds the row sum of P
                const float inv = 1.f / (SUMV ? __uint_as_float(ov[DPAD - 8]) : l);
#pragma unroll
                for (int uu = 0; uu < DPAD / 8; ++uu)
                    if (uu < nch) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(ov[8 * uu + 0]) * inv, __uint_as_float(ov[8 * uu + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(ov[8 * uu + 2]) * inv, __uint_as_float(ov[8 * uu + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(ov[8 * uu + 4]) * inv, __uint_as_float(ov[8 * uu + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(ov[8 * uu + 6]) * inv, __uint_as_float(ov[8 * uu + 7]) * inv);
                        *reinterpret_cast<uint4 *>(stg + r * pitch + uu * 16) = v;
                    }
            }
            __syncwarp();
            {
                // unit i of the warp's 32 x nch pieces: row r0 + i / nch, piece i % nch,
                // walked incrementally (i advances by 32 per step)
                const int r0 = (warp % 4) * 32;
                const int drow = 32 / nch, dpc = 32 % nch;
                int row = r0 + lane / nch, pc = lane % nch;
                __nv_bfloat16 *obase = og + (long)h * d;
                for (int i = lane; i < 32 * nch; i += 32) {
                    const int orw = orow[row - r0];
                    if (orw >= 0)
                        *reinterpret_cast<uint4 *>(obase + (long)orw * a.ldo + pc * 8) =
                            *reinterpret_cast<const uint4 *>(stg + row * pitch + pc * 16);
                    row += drow;
                    pc += dpc;
                    if (pc >= nch) {
                        pc -= nch;
                        ++row;
                    }
                }
            }
            __syncwarp();  // the staging rows are free for the warp's next unit
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
cudaError_t launch_win(const AttnArgs &a, cudaStream_t s) {
    using L = WinLayout<DPAD>;
    int *status = device_status_ptr();
    if (!status) return cudaErrorInvalidValue;
    // the tiles are the tiled-head-layout blocks the window projection wrote
    if (a.tq.mode != THL_WINDOW || a.tk.mode != THL_WINDOW || a.tv.mode != THL_WINDOW ||
        a.tq.vpad || a.tk.vpad || a.tv.vpad || L::TILE != (int)thl_block_bytes(a.d, 0))
        return cudaErrorInvalidValue;
    WinSched sc;
    const int pack = BQ / a.geom.n;
    sc.tiles = (a.geom.nwin + pack - 1) / pack;
    sc.units = a.B * sc.tiles * a.heads;
    sc.wait_ns = debug_wait_limit_ns();
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int grid = (sc.units + 1) / 2 < sms ? (sc.units + 1) / 2 : sms;
    cudaError_t e = cudaFuncSetAttribute(attn_win_kernel<DPAD, SUMV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_win_kernel<DPAD, SUMV>, dim3(grid), dim3(kThreads), L::BYTES, s, a, sc,
                      status);
}

}  // namespace

cudaError_t launch_attention_win_tc(const AttnArgs &a, cudaStream_t s) {
    if (a.d < 8 || a.d > 80 || a.d % 8) return cudaErrorInvalidValue;
    const int n = a.geom.n;
    if (n != 16 && n != 32 && n != 64 && n != 128) return cudaErrorInvalidValue;
    // d = 72: the row sums come out of P V through V's ones column (column 72);
    // other widths sum P in the softmax (a ones column, if any, goes unread)
    if (a.d == 72 && a.tv.ones) return launch_win<80, true>(a, s);
    return a.d <= 64 ? launch_win<64, false>(a, s) : launch_win<80, false>(a, s);
}

}  // namespace ptdit
