// Backward of window and shifted-window self-attention (one TCM branch of the
// Qihoo-T2X reading note, §3 Method, Eq. TCM) on the tensor cores: given the
// window tiles of Q, K, V and of dO = dL/d(attention output), it writes dQ, dK
// and dV.  Per head, with S = c Q K^T (c = 1/sqrt(d), masked pairs -inf) and P
// its row softmax:
//   dV = P^T dO,   dP = dO V^T,   dS = P * (dP - rowsum(P * dP)),
//   dQ = c dS K,   dK = c dS^T Q.
// A window lies inside one 128-row tile (one window of 128 tokens, or two of
// 64, four of 32, eight of 16 packed side by side), so every sum above stays
// inside the tile: a unit (tile, head) needs nothing from any other unit.
//
// One persistent CTA per SM, units in the forward kernel's order (the heads
// of one tile follow each other).  Two load buffers (Q, K, V, dO blocks of the
// tiled head layout, thl.cuh) keep the next unit's loads in flight:
//   warp 8       loader: four bulk copies per unit; the tile rows' key masks
//                (window in tile x wrap bits, built with ballots as in the
//                forward kernel) once per (batch item, tile) and buffer
//   warp 9       MMA issuer (warps 10 and 11 only pad the CTA to whole warpgroups): S = Q K^T and dP = dO V^T into TMEM (K-major
//                operands); once the softmax warpgroup has written P and dS to
//                shared memory: dV = P^T dO, dK = dS^T Q (P and dS read as
//                MN-major A operands) and dQ = dS K (dS as K-major A), with
//                dO, Q, K as MN-major B operands (head columns 0..63 with the
//                128-byte swizzle, 64..79 with the 32-byte swizzle: an N = 64
//                and an N = 16 MMA per K step).  dQ accumulates in dP's
//                columns (the softmax has read dP by then), so the next unit's
//                S is issued as soon as this unit's softmax has read S and dP,
//                its dP once the epilogue has read dQ.
//   warps 0-3    softmax warpgroup, thread r = query row r: reads its
//                window's scores once (max, exponentials, sum), keeps P
//                normalised as bf16 pairs in registers, then rowsum(P * dP) and
//                dS (c folded in) from two reads of dP, and writes P and dS as
//                bf16 rows of 128 x 128 tiles with the 128-byte swizzle; zeros
//                for keys of other windows and for rows without a token.
//   warps 4-7    epilogue, thread r = tile row r: dQ, dK, dV of row r (its
//                token is both a query and a key of the window) to the
//                row-major [B N, 3 D] gradient buffer (dQ, dK, dV column blocks,
//                head h at columns h d .. h d + d - 1 of each).
// TMEM (every accumulator and load starts on a 64-column boundary): S 0-127,
// dP and then dQ 128-255, dV 256-383, dK 384-511 (head columns 0..63 at the
// base, 64..79 at base + 64).  Every wait is bounded (2 s).
#include <type_traits>

#include "tc_util.cuh"
#include "thl.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 128, T_DV = 256, T_DK = 384;
constexpr int NBUF = 2;

template <int DPAD>
struct BwdLayout {
    static constexpr bool HAS_B = DPAD > 64;            // head columns 64..79
    static constexpr int TILE_A = BQ * 128;             // columns 0..63, 128-byte swizzle
    static constexpr int TILE_B = HAS_B ? BQ * 32 : 0;  // columns 64..79, 32-byte swizzle
    static constexpr int TILE = TILE_A + TILE_B;
    static constexpr int BUF = 4 * TILE;                // Q, K, V, dO of one unit
    static constexpr int OFF_P = NBUF * BUF;            // P: 2 key halves x 128 rows x 128 B
    static constexpr int OFF_DS = OFF_P + 2 * TILE_A;   // dS: same layout
    static constexpr int OFF_INFO = OFF_DS + 2 * TILE_A;  // int8 info[NBUF][128]
    // float exchange[warpgroup][2][BQ]: (max, sum), then rowsum(P dP) in the sum's place
    static constexpr int OFF_X = OFF_INFO + NBUF * BQ;
    static constexpr int OFF_BAR = OFF_X + 2 * 2 * BQ * 4;
    // ld_full[NBUF], buf_free[NBUF], s_full, dp_full, sp_free, pds_full, pds_free, acc_full,
    // dq_free, acc_free, drain, x_full[2], x_read, stg_done
    static constexpr int NBARS = 2 * NBUF + 13;
    // no alignment slack: the kernel checks that the base is 1 KB aligned
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16;
    static_assert(TILE_A % 1024 == 0 && TILE % 1024 == 0, "swizzled tiles stay 1 KB aligned");
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct BwdSched {
    int tiles;  // tiles per batch item
    int units;  // B x tiles x heads
};

// Byte offset of 16-byte chunk c (keys 8c .. 8c + 7) of row r in a 128 x 128
// bf16 tile stored as two 64-key halves with the 128-byte swizzle.
__device__ __forceinline__ uint32_t pds_chunk(int r, int c) {
    return (c >> 3) * (BQ * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

template <int DPAD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_win_bwd_kernel(const __grid_constant__ AttnArgs a, const void *__restrict__ dout,
                        __nv_bfloat16 *__restrict__ dqkv, long ldg, BwdSched sc, int *status) {
    using L = BwdLayout<DPAD>;
    extern __shared__ uint8_t sm_raw[];
    // the swizzled tiles need a 1 KB aligned base; the allocation has no slack, so a
    // base that is not aligned is reported instead of used
    if (smem_u32(sm_raw) & 1023u) {
        if (threadIdx.x == 0) atomicExch(status, 5 /* PTDIT_ERR_CUDA */);
        return;
    }
    uint8_t *sm = sm_raw;
    int8_t *info = reinterpret_cast<int8_t *>(sm + L::OFF_INFO);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *ld_full = bars, *buf_free = bars + NBUF;
    uint64_t *s_full = bars + 2 * NBUF, *dp_full = s_full + 1, *sp_free = s_full + 2;
    uint64_t *pds_full = s_full + 3, *pds_free = s_full + 4, *acc_full = s_full + 5;
    uint64_t *dq_free = s_full + 6, *acc_free = s_full + 7, *drain = s_full + 8;
    uint64_t *x_full = s_full + 9;  // the warpgroups' exchanges of a unit: max and sum, rowsum
    uint64_t *x_read = s_full + 11; // each warpgroup has read the other's max and sum
    uint64_t *stg_done = s_full + 12;  // both warpgroups have staged a unit's gradients
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, n = a.geom.n, D = a.heads * a.d;

    if (threadIdx.x == 0) {
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&ld_full[b], 32);  // the loader's 32 lanes (masks) + the four blocks' bytes
            mbar_init(&buf_free[b], 1);  // the unit's last MMA has read its blocks
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(sp_free, 2 * BQ);   // both warpgroups
        mbar_init(pds_full, 2 * BQ);
        mbar_init(pds_free, 1);
        mbar_init(acc_full, 1);
        mbar_init(dq_free, BQ);       // warpgroup 0 reads dQ
        mbar_init(acc_free, 2 * BQ);
        mbar_init(&x_full[0], 2 * BQ);
        mbar_init(&x_full[1], 2 * BQ);
        mbar_init(x_read, 2 * BQ);
        mbar_init(stg_done, 2 * BQ);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    pdl_wait();  // the projections that wrote Q, K, V and dO have completed
    pdl_trigger();

    const int u0 = (int)((long)blockIdx.x * sc.units / gridDim.x);
    const int u1 = (int)((long)(blockIdx.x + 1) * sc.units / gridDim.x);
    const int nunits = u1 - u0;  // local unit k: buffer k % NBUF

    if (warp == 8) {
        // ------------------------------------------------------------ loader
        const uint8_t *src[4] = {static_cast<const uint8_t *>(a.q), static_cast<const uint8_t *>(a.k),
                                 static_cast<const uint8_t *>(a.v),
                                 static_cast<const uint8_t *>(dout)};
        const WinGeom &geo = a.geom;
        const int pack = BQ / n;
        int held0 = -1, held1 = -1;  // (batch item, tile) whose masks each buffer holds
        for (int k = 0; k < nunits; ++k) {
            const int u = u0 + k, bf = k % NBUF;
            const int h = u % a.heads, rest = u / a.heads, tile = rest % sc.tiles,
                      b = rest / sc.tiles;
            if (!mbar_wait_warp(&buf_free[bf], ((k / NBUF) & 1) ^ 1, abort, status)) break;
            if (lane == 0) {
                const long blk = ((long)b * sc.tiles + tile) * a.heads + h;
                mbar_expect_tx_only(&ld_full[bf], 4 * L::TILE);
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    bulk_load(sm + bf * L::BUF + m * L::TILE, src[m] + blk * L::TILE, L::TILE,
                              &ld_full[bf]);
            }
            // window in tile and wrap bits of every tile row (rows of one tile attend each
            // other iff these agree): once per (batch item, tile) and buffer
            const int held = bf == 0 ? held0 : held1;
            if (rest != held) {
                if (bf == 0) held0 = rest; else held1 = rest;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int r = q * 32 + lane;
                    const int wit = r / n, win = tile * pack + wit, slot = r - wit * n;
                    int in = -1;
                    if (win < geo.nwin) {
                        int wrap;
                        (void)window_token(geo, win, slot, &wrap);
                        in = wit * 8 + wrap;
                    }
                    info[bf * BQ + r] = static_cast<int8_t>(in);
                }
            }
            __syncwarp();
            mbar_arrive(&ld_full[bf]);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs the loop with warp-uniform operands; lane 0 issues)
        {
            constexpr uint32_t id_s = idesc_bf16(BQ, BQ);                 // K-major A and B
            constexpr uint32_t id_mm64 = idesc_bf16(BQ, 64, true, true);  // MN-major A and B
            constexpr uint32_t id_mm16 = idesc_bf16(BQ, 16, true, true);
            constexpr uint32_t id_km64 = idesc_bf16(BQ, 64, true, false); // K-major A, MN-major B
            constexpr uint32_t id_km16 = idesc_bf16(BQ, 16, true, false);
            const uint32_t aP = smem_u32(sm + L::OFF_P), aDS = smem_u32(sm + L::OFF_DS);
            bool ok = true, any = false;
            // X (rows x head columns) times Y^T into TMEM column d_col
            auto scores = [&](uint32_t d_col, uint32_t aX, uint32_t aY) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    warp_mma_bf16(tmem + d_col, sdesc_sw128(aX + kk * 32), sdesc_sw128(aY + kk * 32), id_s,
                             kk > 0);
                if (L::HAS_B)
                    warp_mma_bf16(tmem + d_col, sdesc_sw32(aX + L::TILE_A), sdesc_sw32(aY + L::TILE_A),
                             id_s, 1);
            };
            // S = Q K^T of unit k (waits for its blocks)
            auto issue_s = [&](int k) {
                const int bf = k % NBUF;
                if (!mbar_wait_warp(&ld_full[bf], (k / NBUF) & 1, abort, status)) return false;
                fence_after_sync();
                const uint32_t aQ = smem_u32(sm + bf * L::BUF);
                scores(T_S, aQ, aQ + L::TILE);
                warp_mma_commit(s_full);
                any = true;
                return true;
            };
            // dP = dO V^T of unit k (its blocks are in, S(k) waited for them)
            auto issue_dp = [&](int k) {
                const uint32_t aQ = smem_u32(sm + (k % NBUF) * L::BUF);
                scores(T_DP, aQ + 3 * L::TILE, aQ + 2 * L::TILE);
                warp_mma_commit(dp_full);
            };
            // D (rows of the reduction: K steps of 16) += A^T-or-A times the head
            // columns of the MN-major B operand at aB (N = 64, then N = 16)
            auto grad = [&](uint32_t d_col, uint64_t a_desc, uint32_t aB, int ks, bool a_mn) {
                warp_mma_bf16(tmem + d_col, a_desc, sdesc_sw128_mn(aB + ks * 2048, L::TILE_A),
                         a_mn ? id_mm64 : id_km64, ks > 0);
                if (L::HAS_B)
                    warp_mma_bf16(tmem + d_col + 64, a_desc, sdesc_sw32_mn(aB + L::TILE_A + ks * 512),
                             a_mn ? id_mm16 : id_km16, ks > 0);
            };
            auto issue_grads = [&](int k) {
                const int bf = k % NBUF;
                if (!mbar_wait_warp(pds_full, k & 1, abort, status)) return false;
                if (k > 0 && !mbar_wait_warp(acc_free, (k - 1) & 1, abort, status)) return false;
                fence_after_sync();
                const uint32_t aQ = smem_u32(sm + bf * L::BUF), aK = aQ + L::TILE,
                               aO = aQ + 3 * L::TILE;
#pragma unroll
                for (int ks = 0; ks < BQ / 16; ++ks) {
                    // A = P^T / dS^T: the 16 query rows ks of the tile, MN-major (keys contiguous)
                    const uint64_t pT = sdesc_sw128_mn(aP + ks * 2048, L::TILE_A);
                    const uint64_t sT = sdesc_sw128_mn(aDS + ks * 2048, L::TILE_A);
                    // A = dS: keys 16 ks .. 16 ks + 15 of every query row, K-major
                    const uint64_t sK = sdesc_sw128(aDS + (ks >> 2) * L::TILE_A + (ks & 3) * 32);
                    grad(T_DV, pT, aO, ks, true);   // dV += P^T dO
                    grad(T_DK, sT, aQ, ks, true);   // dK += dS^T Q
                    grad(T_DQ, sK, aK, ks, false);  // dQ += dS K
                }
                warp_mma_commit(acc_full);
                warp_mma_commit(pds_free);
                warp_mma_commit(&buf_free[bf]);
                return true;
            };
            if (nunits > 0) {
                ok = issue_s(0);
                if (ok) issue_dp(0);
            }
            for (int k = 0; k < nunits && ok; ++k) {
                // the softmax has read this unit's S and dP: the next S may overwrite S,
                // and the gradients (dQ in dP's columns) may start
                if (!mbar_wait_warp(sp_free, k & 1, abort, status)) break;
                if (k + 1 < nunits) ok = issue_s(k + 1);
                if (ok) ok = issue_grads(k);
                if (ok && k + 1 < nunits) {
                    // the epilogue has read dQ(k) out of dP's columns
                    if (!mbar_wait_warp(dq_free, k & 1, abort, status)) break;
                    fence_after_sync();
                    issue_dp(k + 1);
                }
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                warp_mma_commit(drain);
                volatile int never = 0;
                mbar_wait_warp(drain, 0, &never, status);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax + epilogue
        // Warpgroup g = warp / 4 takes half of every row's keys (thread r: query row r,
        // its TMEM lane): keys 64 g .. 64 g + 63 of a 128-token window, or 32 of the
        // 64 keys of a smaller window's half of the tile.  The halves' maxima and sums
        // are combined once per unit (each half exponentiates against its own max;
        // the shared scale is 2^(m_g - m) / l), and rowsum(P * dP) once more.
        const int g = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const float c = a.scale, sl2 = a.scale * 1.4426950408889634f;
        uint8_t *sP = sm + L::OFF_P, *sDS = sm + L::OFF_DS;
        float *xch = reinterpret_cast<float *>(sm + L::OFF_X);  // [g][2][BQ]
        const int c_lo = n < BQ ? (r >> 6) << 6 : 0;            // the row's 64-key half
        const int kofs = n < BQ ? c_lo + 32 * g : 64 * g;       // first key of this warpgroup
        const uint32_t t_s = tmem + lane_base + T_S + kofs, t_dp = tmem + lane_base + T_DP + kofs;
        const WinGeom &geo = a.geom;
        const int pack = BQ / n, nch = d / 8;
        // gradients of unit kk out of TMEM: dQ and dV by warpgroup 0, dK by warpgroup 1
        auto epilogue = [&](int kk) {
            if (!mbar_wait_warp(acc_full, kk & 1, abort, status)) return false;
            fence_after_sync();
            const int u = u0 + kk;
            const int h = u % a.heads, rest = u / a.heads, tile = rest % sc.tiles,
                      b = rest / sc.tiles;
            const int wit = r / n, win = tile * pack + wit, slot = r - wit * n;
            long row = -1;
            if (win < geo.nwin) {
                int wrap;
                row = (long)b * a.k_bstride + window_token(geo, win, slot, &wrap);
            }
            // staging: this warp's 8 KB of the P / dS tiles (the unit's MMAs are done with
            // them; the next P is written only after both warpgroups are through here)
            uint8_t *stg = sm + L::OFF_P + warp * 8192;
            const int pitch = nch * 16 + (nch % 8 == 0 ? 16 : 0);  // an odd number of 16 B units
            // warpgroup 0 writes dQ and dV, warpgroup 1 dK
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                if (g == 1 && i == 1) break;
                const int m = g == 1 ? 1 : (i == 0 ? 0 : 2);  // column block: dQ 0, dK 1, dV 2
                uint32_t v[DPAD];
                const uint32_t t = tmem + lane_base + (m == 0 ? T_DQ : (m == 1 ? T_DK : T_DV));
                tmem_ld32(t, *reinterpret_cast<uint32_t(*)[32]>(v));
                tmem_ld32(t + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                if (DPAD > 64) tmem_ld16(t + 64, *reinterpret_cast<uint32_t(*)[16]>(v + 64));
                tmem_ld_wait();
                if (m == 0) {  // dQ is out of dP's columns: the next dP may go there
                    fence_before_sync();
                    mbar_arrive(dq_free);
                }
                if (m != 0 && (g == 1 || i == 1)) {  // this warpgroup's last TMEM read
                    fence_before_sync();
                    mbar_arrive(acc_free);  // the next unit's gradient MMAs may overwrite TMEM
                }
#pragma unroll
                for (int uu = 0; uu < DPAD / 8; ++uu)
                    if (uu < nch) {
                        uint4 o;
                        o.x = pack_bf16(__uint_as_float(v[8 * uu + 0]), __uint_as_float(v[8 * uu + 1]));
                        o.y = pack_bf16(__uint_as_float(v[8 * uu + 2]), __uint_as_float(v[8 * uu + 3]));
                        o.z = pack_bf16(__uint_as_float(v[8 * uu + 4]), __uint_as_float(v[8 * uu + 5]));
                        o.w = pack_bf16(__uint_as_float(v[8 * uu + 6]), __uint_as_float(v[8 * uu + 7]));
                        *reinterpret_cast<uint4 *>(stg + lane * pitch + uu * 16) = o;
                    }
                __syncwarp();
                // consecutive lanes on consecutive 16-byte pieces of a token row: item j of
                // the warp's 32 x nch pieces is piece j % nch of staging row j / nch, walked
                // incrementally (j advances by 32 per step)
                const int drow = 32 / nch, dpc = 32 % nch;
                int rr = lane / nch, cc = lane % nch;
                __nv_bfloat16 *colbase = dqkv + (long)m * D + (long)h * d;
#pragma unroll 1
                for (int j = lane; j < 32 * nch; j += 32) {
                    const long trow = __shfl_sync(0xffffffffu, row, rr);  // that row's token
                    if (trow >= 0)
                        *reinterpret_cast<uint4 *>(colbase + trow * ldg + 8 * cc) =
                            *reinterpret_cast<const uint4 *>(stg + rr * pitch + cc * 16);
                    rr += drow;
                    cc += dpc;
                    if (cc >= nch) {
                        cc -= nch;
                        ++rr;
                    }
                }
                __syncwarp();  // the staging rows are free for the next block
            }
            return true;
        };
        bool okw = true;
        auto unit = [&](int k, auto NKc) {
            constexpr int NK = decltype(NKc)::value;  // this warpgroup's keys of the row
            const int bf = k % NBUF;
            if (!mbar_wait_warp(&ld_full[bf], (k / NBUF) & 1, abort, status)) { okw = false; return; }
            // key e of this half is allowed iff its window-in-tile and wrap bits equal the
            // row's (a row without a token, qi < 0, allows none)
            const int qi = info[bf * BQ + r];
            uint32_t aw[2] = {0u, 0u};
            {
                const uint32_t *ik = reinterpret_cast<const uint32_t *>(info + bf * BQ + kofs);
#pragma unroll
                for (int i = 0; i < NK / 4; ++i) {
                    const uint32_t wv = ik[i];  // the same word in every lane: a broadcast
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (qi >= 0 && static_cast<int8_t>(wv >> (8 * j)) == qi)
                            aw[(4 * i + j) >> 5] |= 1u << ((4 * i + j) & 31);
                }
            }
            if (!mbar_wait_warp(s_full, k & 1, abort, status)) { okw = false; return; }
            fence_after_sync();
            // this half's scores, read once: its max, its exponentials (bf16 pairs), its sum
            uint32_t pk[NK / 2];
            float ms_g, l_g;
            {
                uint32_t sv[NK];
#pragma unroll
                for (int q = 0; q < NK / 32; ++q)
                    tmem_ld32(t_s + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(sv + 32 * q));
                tmem_ld_wait();
                float mx[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
                // every key of the half allowed (all of WSA, SWSA away from the wrap): no
                // per-key selects
                const bool all = aw[0] == (NK >= 32 ? 0xffffffffu : ((1u << NK) - 1u)) &&
                                 aw[1] == (NK >= 64 ? 0xffffffffu : 0u);
                if (all) {
#pragma unroll
                    for (int e = 0; e < NK; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(sv[e]));
                } else {
#pragma unroll
                    for (int e = 0; e < NK; ++e)
                        if ((aw[e >> 5] >> (e & 31)) & 1u) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(sv[e]));
                }
                ms_g = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
                float ls[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) ls[i] = 0.f;
                if (all) {
#pragma unroll
                    for (int e = 0; e < NK; e += 2) {
                        const float p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, -ms_g));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), sl2, -ms_g));
                        ls[(e >> 1) & 7] += p0 + p1;
                        pk[e / 2] = pack_bf16(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < NK; e += 2) {
                        const uint32_t w = aw[e >> 5];
                        const float p0 = ((w >> (e & 31)) & 1u) ? ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, -ms_g)) : 0.f;
                        const float p1 = ((w >> ((e + 1) & 31)) & 1u) ? ex2_approx(fmaf(__uint_as_float(sv[e + 1]), sl2, -ms_g)) : 0.f;
                        ls[(e >> 1) & 7] += p0 + p1;
                        pk[e / 2] = pack_bf16(p0, p1);
                    }
                }
                l_g = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
            }
            // combine the halves: m = max(m_0, m_1), l = sum of l_g 2^(m_g - m)
            // (the slots are rewritten only after the other warpgroup has read them: the
            // sum's slot carries rowsum(P dP) once x_read shows it read, and the next
            // unit's values follow sp_free, which needs both warpgroups)
            float *xm = xch + g * 2 * BQ;
            const float *xo = xch + (g ^ 1) * 2 * BQ;
            xm[r] = ms_g;
            xm[BQ + r] = l_g;
            mbar_arrive(&x_full[0]);
            if (!mbar_wait_warp(&x_full[0], k & 1, abort, status)) { okw = false; return; }
            const float ms_o = xo[r], l_o = xo[BQ + r];
            mbar_arrive(x_read);
            const float msx = fmaxf(ms_g, ms_o);
            const float f_g = ms_g == -INFINITY ? 0.f : ex2_approx(ms_g - msx);
            const float f_o = ms_o == -INFINITY ? 0.f : ex2_approx(ms_o - msx);
            const float lsum = l_g * f_g + l_o * f_o;
            const float scale = lsum > 0.f ? f_g / lsum : 0.f;  // no allowed key: P = 0
#pragma unroll
            for (int e = 0; e < NK / 2; ++e) {
                const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pk[e]));
                pk[e] = pack_bf16(pr.x * scale, pr.y * scale);
            }
            // the previous unit's gradients out of TMEM (their dQ read lets this unit's
            // dP go into dP's columns)
            if (k > 0) {
                if (!epilogue(k - 1)) { okw = false; return; }
                // the other warpgroup's staging (in the P / dS tiles) is done too
                mbar_arrive(stg_done);
                if (!mbar_wait_warp(stg_done, (k - 1) & 1, abort, status)) { okw = false; return; }
            }
            // the previous unit's MMAs have read P and dS; this unit's dP is in
            if (!mbar_wait_warp(pds_free, (k & 1) ^ 1, abort, status) ||
                !mbar_wait_warp(dp_full, k & 1, abort, status)) {
                okw = false;
                return;
            }
            fence_after_sync();
#pragma unroll
            for (int q = 0; q < NK / 8; ++q)
                *reinterpret_cast<uint4 *>(sP + pds_chunk(r, (kofs >> 3) + q)) =
                    make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            // this half of dP, read once: rowsum(P * dP) over both halves, then dS
            uint32_t dv[NK];
#pragma unroll
            for (int q = 0; q < NK / 32; ++q)
                tmem_ld32(t_dp + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(dv + 32 * q));
            tmem_ld_wait();
            float dl[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) dl[i] = 0.f;
#pragma unroll
            for (int e = 0; e < NK; e += 2) {
                const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pk[e / 2]));
                dl[e & 7] = fmaf(pr.x, __uint_as_float(dv[e]), dl[e & 7]);
                dl[(e & 7) + 1] = fmaf(pr.y, __uint_as_float(dv[e + 1]), dl[(e & 7) + 1]);
            }
            const float d_g = ((dl[0] + dl[1]) + (dl[2] + dl[3])) + ((dl[4] + dl[5]) + (dl[6] + dl[7]));
            if (!mbar_wait_warp(x_read, k & 1, abort, status)) { okw = false; return; }
            xm[BQ + r] = d_g;
            mbar_arrive(&x_full[1]);
            if (!mbar_wait_warp(&x_full[1], k & 1, abort, status)) { okw = false; return; }
            const float delta = d_g + xo[BQ + r];
#pragma unroll
            for (int q = 0; q < NK / 8; ++q) {
                uint32_t o[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int e = 8 * q + 2 * t;
                    const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pk[e / 2]));
                    o[t] = pack_bf16(c * pr.x * (__uint_as_float(dv[e]) - delta),
                                     c * pr.y * (__uint_as_float(dv[e + 1]) - delta));
                }
                *reinterpret_cast<uint4 *>(sDS + pds_chunk(r, (kofs >> 3) + q)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_before_sync();
            mbar_arrive(sp_free);  // S and dP are read
            // the keys of the tile's other window half: zero weights and gradients
            if (n < BQ) {
                const int o0 = ((64 - c_lo) >> 3) + 4 * g;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    *reinterpret_cast<uint4 *>(sP + pds_chunk(r, o0 + q)) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(sDS + pds_chunk(r, o0 + q)) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_async_smem();  // the tensor cores read what these threads wrote
            mbar_arrive(pds_full);
        };
        for (int k = 0; k < nunits && okw; ++k) {
            if (n < BQ)
                unit(k, std::integral_constant<int, 32>{});
            else
                unit(k, std::integral_constant<int, 64>{});
        }
        if (okw && nunits > 0) epilogue(nunits - 1);
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

template <int DPAD>
cudaError_t launch_bwd(const AttnArgs &a, const void *dout, void *dqkv, long ldg, cudaStream_t s) {
    using L = BwdLayout<DPAD>;
    int *status = device_status_ptr();
    if (!status) return cudaErrorInvalidValue;
    if (a.tq.mode != THL_WINDOW || a.tk.mode != THL_WINDOW || a.tv.mode != THL_WINDOW ||
        a.tq.vpad || a.tk.vpad || a.tv.vpad || L::TILE != (int)thl_block_bytes(a.d, 0))
        return cudaErrorInvalidValue;
    BwdSched sc;
    const int pack = BQ / a.geom.n;
    sc.tiles = (a.geom.nwin + pack - 1) / pack;
    sc.units = a.B * sc.tiles * a.heads;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int grid = sc.units < sms ? sc.units : sms;
    cudaError_t e = cudaFuncSetAttribute(attn_win_bwd_kernel<DPAD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_win_bwd_kernel<DPAD>, dim3(grid), dim3(kThreads), L::BYTES, s, a, dout,
                      static_cast<__nv_bfloat16 *>(dqkv), ldg, sc, status);
}

}  // namespace

cudaError_t launch_attention_win_bwd(const AttnArgs &a, const void *dout, void *dqkv, long ldg,
                                     cudaStream_t s) {
    if (a.d < 8 || a.d > 80 || a.d % 8) return cudaErrorInvalidValue;
    const int n = a.geom.n;
    if (n != 16 && n != 32 && n != 64 && n != 128) return cudaErrorInvalidValue;
    return a.d <= 64 ? launch_bwd<64>(a, dout, dqkv, ldg, s) : launch_bwd<80>(a, dout, dqkv, ldg, s);
}

}  // namespace ptdit
