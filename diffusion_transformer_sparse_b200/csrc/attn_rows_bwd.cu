// Backward of row-mode attention on the tensor cores: GIIM's latent -> proxy
// cross-attention and proxy self-attention (Qihoo-T2X reading note, §3 Method,
// Eq. GIIM).  Per head, with S = c Q K^T (c = 1/sqrt(d)) and P = exp2(S log2 e
// - lse) (lse: each query row's log-sum-exp from the forward pass), given dO:
//   dP = dO V^T,  dS = P * (dP - delta),  delta = rowsum(dO * O) (precomputed),
//   dV = P^T dO,  dK = c dS^T Q,  dQ = c dS K.
// dK and dV sum over every query row, dQ over every key: a CTA owns one
// (batch item, head, 128-key tile) over a slice of the query tiles, keeps that
// key tile's dK and dV in TMEM across the slice and adds them into fp32 [B nk, D]
// outputs once (vector reductions), and writes dQ of each (query tile, key tile)
// into its own column block of a bf16 [B nq, KT D] buffer (the caller sums the KT
// blocks: the input-gradient projection takes K = KT D with the weights stacked).
// The caller passes keys less their mean over each item's keys (the softmax
// ignores a shift common to all keys, so the forward's output is the same and
// its log-sum-exp is taken with the same keys): dQ = c dS (K - m) is then the
// exact gradient, and the rounding of the bf16 dS no longer multiplies the keys'
// common component (proxy keys are averages and share most of their value).
//
// One persistent CTA per SM, 384 threads:
//   warp 8       loader: the item's K and V blocks (tiled head layout,
//                thl.cuh, no V padding), and each query tile's Q and dO blocks
//                (two buffers)
//   warp 9       MMA issuer: S = Q K^T into TMEM, dP = dO V^T into S's columns
//                once S is read; once P and dS are in shared memory: dV += P^T dO,
//                dK += dS^T Q (accumulated over the item's query tiles) and dQ =
//                dS K.  Within an item a tile's work is issued as S(t+1), dV(t),
//                dK(t), dP(t+1), dQ(t): the warpgroups compute P(t+1) while dV(t)
//                and dK(t) run; P is released after dV, dS after dQ.  An item's
//                last tile issues its gradients first (the next item's K and V
//                load once dQ has read K).
//   warps 0-7    two warpgroups, 64 keys of every row each (thread r: query row
//                r): P from lse, dS from delta (no exchange between them), then
//                the previous query tile's dQ through their own staging rows with
//                coalesced stores, and at an item's end the key tile's dK (warp-
//                group 1) and dV (warpgroup 0)
// TMEM (64-column aligned): S then dP 0-127, dQ 128-255, dV 256-383, dK 384-511.
// Every wait is bounded (2 s).
#include <type_traits>

#include "tc_util.cuh"
#include "thl.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_S = 0, T_DP = 0, T_DQ = 128, T_DV = 256, T_DK = 384;
constexpr int NQB = 2;  // query-tile buffers

template <int DPAD>
struct RbLayout {
    static constexpr bool HAS_B = DPAD > 64;
    static constexpr int TILE_A = BQ * 128;
    static constexpr int TILE_B = HAS_B ? BQ * 32 : 0;
    static constexpr int TILE = TILE_A + TILE_B;
    static constexpr int OFF_K = 0, OFF_V = TILE;        // the item's key tile
    static constexpr int OFF_Q = 2 * TILE;               // [NQB] Q, then dO
    static constexpr int OFF_P = OFF_Q + NQB * 2 * TILE; // P, dS: 2 key halves x 128 rows x 128 B
    static constexpr int OFF_DS = OFF_P + 2 * TILE_A;
    static constexpr int OFF_STG = OFF_DS + 2 * TILE_A;  // [8 warps][32 rows][96 B] dQ staging
    static constexpr int OFF_BAR = OFF_STG + 8 * 32 * 96;
    // kv_full, kv_free, q_full[NQB], q_free[NQB], s_full, dp_full, s_read, pds_full,
    // p_free, dq_full, dq_free, kvacc_full, kvacc_free, drain
    static constexpr int NBARS = 2 * NQB + 12;
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16;  // the kernel checks 1 KB alignment
    static_assert(TILE_A % 1024 == 0 && TILE % 1024 == 0, "swizzled tiles stay 1 KB aligned");
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct RbSched {
    int qt, kt;    // query and key tiles per batch item
    int splits;    // query-tile slices per (batch item, head, key tile)
    int items;     // B x heads x kt x splits
};

// Item it: slice `sp` of the query tiles of key tile j of head h of batch item b.
__device__ __forceinline__ void rb_decode(const AttnArgs &a, const RbSched &sc, int it, int &b,
                                          int &h, int &j, int &q0, int &q1) {
    const int sp = it % sc.splits;
    int rest = it / sc.splits;
    j = rest % sc.kt;
    rest /= sc.kt;
    h = rest % a.heads;
    b = rest / a.heads;
    q0 = (int)((long)sp * sc.qt / sc.splits);
    q1 = (int)((long)(sp + 1) * sc.qt / sc.splits);
}

__device__ __forceinline__ uint32_t pds_chunk(int r, int c) {
    return (c >> 3) * (BQ * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void red_add_v4(float *p, float x, float y, float z, float w) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(x), "f"(y), "f"(z),
                 "f"(w)
                 : "memory");
}

template <int DPAD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_rows_bwd_kernel(const __grid_constant__ AttnArgs a, const void *__restrict__ dout,
                         const float *__restrict__ lse, const float *__restrict__ delta,
                         __nv_bfloat16 *__restrict__ dq, long ldq, float *__restrict__ dk,
                         float *__restrict__ dv, RbSched sc, int *status) {
    using L = RbLayout<DPAD>;
    extern __shared__ uint8_t sm_raw[];
    if (smem_u32(sm_raw) & 1023u) {  // no alignment slack in the allocation
        if (threadIdx.x == 0) atomicExch(status, 5 /* PTDIT_ERR_CUDA */);
        return;
    }
    uint8_t *sm = sm_raw;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *kv_full = bars, *kv_free = bars + 1, *q_full = bars + 2, *q_free = q_full + NQB;
    uint64_t *s_full = q_free + NQB, *dp_full = s_full + 1, *s_read = s_full + 2;
    uint64_t *pds_full = s_full + 3, *p_free = s_full + 4, *dq_full = s_full + 5;
    uint64_t *dq_free = s_full + 6, *kvacc_full = s_full + 7, *kvacc_free = s_full + 8;
    uint64_t *drain = s_full + 9;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d = a.d, D = a.heads * a.d, nch = d / 8;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(kv_free, 1);
        for (int i = 0; i < NQB; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_free[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(s_read, 2 * BQ);
        mbar_init(pds_full, 2 * BQ);
        mbar_init(p_free, 1);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, 2 * BQ);
        mbar_init(kvacc_full, 1);
        mbar_init(kvacc_free, 2 * BQ);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    pdl_wait();  // the kernels that wrote Q, K, V, dO, lse and delta have completed
    pdl_trigger();

    const int i0 = (int)((long)blockIdx.x * sc.items / gridDim.x);
    const int i1 = (int)((long)(blockIdx.x + 1) * sc.items / gridDim.x);
    // the CTA's query tiles, counted over its items: tile t of item it
    auto item_tiles = [&](int it) {
        int b, h, j, q0, q1;
        rb_decode(a, sc, it, b, h, j, q0, q1);
        return q1 - q0;
    };

    if (warp == 8) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            const uint8_t *qg = static_cast<const uint8_t *>(a.q), *kg = static_cast<const uint8_t *>(a.k);
            const uint8_t *vg = static_cast<const uint8_t *>(a.v), *og = static_cast<const uint8_t *>(dout);
            auto block = [&](const uint8_t *base, const ThlDesc &t, int b, int tile, int h) {
                return base + (((long)b * t.tiles + tile) * a.heads + h) * (long)L::TILE;
            };
            int t = 0, n_item = 0;  // n_item counts the items that have query tiles
            bool ok = true;
            for (int it = i0; it < i1 && ok; ++it) {
                int b, h, j, q0, q1;
                rb_decode(a, sc, it, b, h, j, q0, q1);
                if (q1 <= q0) continue;
                if (!mbar_wait(kv_free, (n_item++ & 1) ^ 1, abort, status)) break;
                mbar_expect_tx(kv_full, 2 * L::TILE);
                bulk_load(sm + L::OFF_K, block(kg, a.tk, b, j, h), L::TILE, kv_full);
                bulk_load(sm + L::OFF_V, block(vg, a.tv, b, j, h), L::TILE, kv_full);
                for (int qi = q0; qi < q1; ++qi, ++t) {
                    const int bf = t % NQB;
                    if (!mbar_wait(&q_free[bf], ((t / NQB) & 1) ^ 1, abort, status)) { ok = false; break; }
                    mbar_expect_tx(&q_full[bf], 2 * L::TILE);
                    uint8_t *dst = sm + L::OFF_Q + bf * 2 * L::TILE;
                    bulk_load(dst, block(qg, a.tq, b, qi, h), L::TILE, &q_full[bf]);
                    bulk_load(dst + L::TILE, block(og, a.tq, b, qi, h), L::TILE, &q_full[bf]);
                }
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs the loop with warp-uniform operands; lane 0 issues)
        {
            constexpr uint32_t id_s = idesc_bf16(BQ, BQ);
            constexpr uint32_t id_mm64 = idesc_bf16(BQ, 64, true, true);
            constexpr uint32_t id_mm16 = idesc_bf16(BQ, 16, true, true);
            constexpr uint32_t id_km64 = idesc_bf16(BQ, 64, true, false);
            constexpr uint32_t id_km16 = idesc_bf16(BQ, 16, true, false);
            const uint32_t aP = smem_u32(sm + L::OFF_P), aDS = smem_u32(sm + L::OFF_DS);
            const uint32_t aK = smem_u32(sm + L::OFF_K), aV = smem_u32(sm + L::OFF_V);
            auto qbuf = [&](int t) { return smem_u32(sm + L::OFF_Q + (t % NQB) * 2 * L::TILE); };
            auto scores = [&](uint32_t d_col, uint32_t aX, uint32_t aY) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    warp_mma_bf16(tmem + d_col, sdesc_sw128(aX + kk * 32), sdesc_sw128(aY + kk * 32), id_s,
                             kk > 0);
                if (L::HAS_B)
                    warp_mma_bf16(tmem + d_col, sdesc_sw32(aX + L::TILE_A), sdesc_sw32(aY + L::TILE_A),
                             id_s, 1);
            };
            auto grad = [&](uint32_t d_col, uint64_t a_desc, uint32_t aB, int ks, bool a_mn,
                            bool acc) {
                warp_mma_bf16(tmem + d_col, a_desc, sdesc_sw128_mn(aB + ks * 2048, L::TILE_A),
                         a_mn ? id_mm64 : id_km64, acc);
                if (L::HAS_B)
                    warp_mma_bf16(tmem + d_col + 64, a_desc, sdesc_sw32_mn(aB + L::TILE_A + ks * 512),
                             a_mn ? id_mm16 : id_km16, acc);
            };
            // the CTA's query tiles in order, with their item's ordinal and position
            int T = 0;
            for (int it = i0; it < i1; ++it) T += item_tiles(it);
            bool ok = true, any = false;
            int it = i0, n_item = 0, pos = 0;  // item of tile t, its ordinal, t's place in it
            while (it < i1 && item_tiles(it) == 0) ++it;
            auto advance = [&](int &itx, int &nix, int &posx) {
                if (++posx == item_tiles(itx)) {
                    posx = 0;
                    ++nix;
                    do { ++itx; } while (itx < i1 && item_tiles(itx) == 0);
                }
            };
            // S(t) into columns 0-127 (K of item nix when t opens it)
            auto issue_s = [&](int t, bool new_item, int nix) {
                if (new_item && !mbar_wait_warp(kv_full, nix & 1, abort, status)) return false;
                if (!mbar_wait_warp(&q_full[t % NQB], (t / NQB) & 1, abort, status)) return false;
                fence_after_sync();
                scores(T_S, qbuf(t), aK);
                warp_mma_commit(s_full);
                any = true;
                return true;
            };
            // dP(t) into the same columns once the warpgroups have read S(t)
            auto issue_dp = [&](int t) {
                if (!mbar_wait_warp(s_read, t & 1, abort, status)) return false;
                fence_after_sync();
                scores(T_DP, qbuf(t) + L::TILE, aV);
                warp_mma_commit(dp_full);
                return true;
            };
            // dV += P^T dO, then dK += dS^T Q of tile t (the item's first tile overwrites)
            auto issue_dvdk = [&](int t, bool first) {
                const uint32_t aQ = qbuf(t), aO = aQ + L::TILE;
#pragma unroll
                for (int ks = 0; ks < BQ / 16; ++ks)
                    grad(T_DV, sdesc_sw128_mn(aP + ks * 2048, L::TILE_A), aO, ks, true,
                         !first || ks > 0);
                warp_mma_commit(p_free);  // P is read
#pragma unroll
                for (int ks = 0; ks < BQ / 16; ++ks)
                    grad(T_DK, sdesc_sw128_mn(aDS + ks * 2048, L::TILE_A), aQ, ks, true,
                         !first || ks > 0);
                warp_mma_commit(&q_free[t % NQB]);  // Q and dO are read
            };
            // dQ = dS K of tile t in its own columns, once the previous dQ is read
            auto issue_dq = [&](int t) {
                if (t > 0 && !mbar_wait_warp(dq_free, (t - 1) & 1, abort, status)) return false;
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < BQ / 16; ++ks)
                    grad(T_DQ, sdesc_sw128(aDS + (ks >> 2) * L::TILE_A + (ks & 3) * 32), aK, ks,
                         false, ks > 0);
                warp_mma_commit(dq_full);  // dQ is in TMEM and dS is read
                return true;
            };
            if (T > 0) ok = issue_s(0, true, 0) && issue_dp(0);
            for (int t = 0; t < T && ok; ++t) {
                const bool first = pos == 0, last = pos + 1 == item_tiles(it);
                int it2 = it, n2 = n_item, pos2 = pos;
                advance(it2, n2, pos2);  // tile t + 1
                // P(t) and dS(t) written, dP(t) read (S's columns are free)
                if (!mbar_wait_warp(pds_full, t & 1, abort, status)) break;
                if (first && n_item > 0 && !mbar_wait_warp(kvacc_free, (n_item - 1) & 1, abort, status))
                    break;
                fence_after_sync();
                if (!last) {
                    // within an item: the next S, this tile's dV and dK, the next dP, this
                    // dQ, so that the warpgroups compute the next P while dV and dK run
                    if (!issue_s(t + 1, false, n2)) break;
                    issue_dvdk(t, first);
                    ok = issue_dp(t + 1) && issue_dq(t);
                } else {
                    // the item's last tile: its gradients first (the next item's K and V
                    // load only once dQ has read K)
                    issue_dvdk(t, first);
                    if (!issue_dq(t)) break;
                    warp_mma_commit(kvacc_full);
                    warp_mma_commit(kv_free);
                    if (t + 1 < T) ok = issue_s(t + 1, true, n2) && issue_dp(t + 1);
                }
                it = it2;
                n_item = n2;
                pos = pos2;
            }
            if (any) {
                warp_mma_commit(drain);
                volatile int never = 0;
                mbar_wait_warp(drain, 0, &never, status);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ two warpgroups
        const int g = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const float c = a.scale, sl2 = a.scale * 1.4426950408889634f;
        uint8_t *sP = sm + L::OFF_P, *sDS = sm + L::OFF_DS;
        uint8_t *stg = sm + L::OFF_STG + warp * 32 * 96;
        const int kofs = 64 * g;
        // dQ of tile tt (query tile qi of item (b, h, j)) out of TMEM: warpgroup 0 writes
        // the head's pieces 0-3, warpgroup 1 pieces 4..
        auto dq_epilogue = [&](int tt, int b, int h, int j, int qi, bool wait) {
            if (wait && !mbar_wait_warp(dq_full, tt & 1, abort, status)) return false;
            fence_after_sync();
            uint32_t v[48];
            const uint32_t t = tmem + lane_base + T_DQ + 32 * g;
            tmem_ld32(t, *reinterpret_cast<uint32_t(*)[32]>(v));
            if (g == 1 && DPAD > 64) tmem_ld16(t + 32, *reinterpret_cast<uint32_t(*)[16]>(v + 32));
            tmem_ld_wait();
            fence_before_sync();
            mbar_arrive(dq_free);  // dQ is read: the next dQ may go to these columns
            const int u0 = g == 0 ? 0 : 4, nu = g == 0 ? min(4, nch) : max(0, nch - 4);
#pragma unroll
            for (int uu = 0; uu < 6; ++uu)
                if (uu < nu) {
                    uint4 o;
                    o.x = pack_bf16(__uint_as_float(v[8 * uu + 0]), __uint_as_float(v[8 * uu + 1]));
                    o.y = pack_bf16(__uint_as_float(v[8 * uu + 2]), __uint_as_float(v[8 * uu + 3]));
                    o.z = pack_bf16(__uint_as_float(v[8 * uu + 4]), __uint_as_float(v[8 * uu + 5]));
                    o.w = pack_bf16(__uint_as_float(v[8 * uu + 6]), __uint_as_float(v[8 * uu + 7]));
                    *reinterpret_cast<uint4 *>(stg + lane * 96 + 16 * uu) = o;
                }
            __syncwarp();
            if (nu > 0) {
                // consecutive lanes on consecutive 16-byte pieces of the warp's 32 rows
                const int drow = 32 / nu, dpc = 32 % nu;
                int rr = lane / nu, cc = lane % nu;
                const long q0 = (long)qi * BQ + (warp & 3) * 32;  // query of staging row 0
                __nv_bfloat16 *base = dq + (long)j * D + (long)h * d + 8 * u0;
#pragma unroll 1
                for (int jj = lane; jj < 32 * nu; jj += 32) {
                    if (q0 + rr < a.nq)
                        *reinterpret_cast<uint4 *>(base + ((long)b * a.nq + q0 + rr) * ldq + 8 * cc) =
                            *reinterpret_cast<const uint4 *>(stg + rr * 96 + cc * 16);
                    rr += drow;
                    cc += dpc;
                    if (cc >= nu) {
                        cc -= nu;
                        ++rr;
                    }
                }
            }
            __syncwarp();
            return true;
        };
        // the key tile's dK (warpgroup 1) or dV (warpgroup 0) into the fp32 outputs
        auto kv_flush = [&](int nix, int b, int h, int j) {
            if (!mbar_wait_warp(kvacc_full, nix & 1, abort, status)) return false;
            fence_after_sync();
            uint32_t v[DPAD];
            const uint32_t t = tmem + lane_base + (g == 0 ? T_DV : T_DK);
            tmem_ld32(t, *reinterpret_cast<uint32_t(*)[32]>(v));
            tmem_ld32(t + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
            if (DPAD > 64) tmem_ld16(t + 64, *reinterpret_cast<uint32_t(*)[16]>(v + 64));
            tmem_ld_wait();
            fence_before_sync();
            mbar_arrive(kvacc_free);
            const long key = (long)j * BQ + r;
            if (key < a.nk) {
                float *row = (g == 0 ? dv : dk) + ((long)b * a.nk + key) * D + (long)h * d;
#pragma unroll
                for (int e = 0; e < DPAD; e += 4)
                    if (e < d)
                        red_add_v4(row + e, __uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                   __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
            }
            return true;
        };
        bool okw = true;
        int t = 0, n_item = 0;
        // the previous tile (for its dQ) and whether it closed an item (for dK, dV)
        int pb = 0, ph = 0, pj = 0, pqi = 0, pnix = 0;
        bool have_prev = false, prev_last = false;
        for (int it = i0; it < i1 && okw; ++it) {
            int b, h, j, q0, q1;
            rb_decode(a, sc, it, b, h, j, q0, q1);
            if (q1 <= q0) continue;
            const long key0 = (long)j * BQ + kofs;
            for (int qi = q0; qi < q1 && okw; ++qi, ++t) {
                const long q = (long)qi * BQ + r;
                const bool qv = q < a.nq;
                const long bh = (long)b * a.heads + h;
                const float l2 = qv ? lse[bh * a.nq + q] : 0.f;
                const float dl = qv ? delta[bh * a.nq + q] : 0.f;
                if (!mbar_wait_warp(s_full, t & 1, abort, status)) { okw = false; break; }
                fence_after_sync();
                // P of this warpgroup's 64 keys from the forward's log-sum-exp
                uint32_t pk[32];
                {
                    uint32_t sv[64];
                    tmem_ld32(tmem + lane_base + T_S + kofs, *reinterpret_cast<uint32_t(*)[32]>(sv));
                    tmem_ld32(tmem + lane_base + T_S + kofs + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                    tmem_ld_wait();
                    fence_before_sync();
                    mbar_arrive(s_read);  // S is read: dP may go to its columns
                    if (qv && key0 + 64 <= a.nk) {  // every key of the half is valid
#pragma unroll
                        for (int e = 0; e < 64; e += 2)
                            pk[e / 2] = pack_bf16(ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, -l2)),
                                                  ex2_approx(fmaf(__uint_as_float(sv[e + 1]), sl2, -l2)));
                    } else {
                        const int nv = qv ? (int)max(0L, min(64L, (long)a.nk - key0)) : 0;
#pragma unroll
                        for (int e = 0; e < 64; e += 2) {
                            const float p0 = e < nv ? ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, -l2)) : 0.f;
                            const float p1 = e + 1 < nv ? ex2_approx(fmaf(__uint_as_float(sv[e + 1]), sl2, -l2)) : 0.f;
                            pk[e / 2] = pack_bf16(p0, p1);
                        }
                    }
                }
                // P into shared memory once the previous tile's dV has read it
                if (t > 0 && !mbar_wait_warp(p_free, (t - 1) & 1, abort, status)) { okw = false; break; }
#pragma unroll
                for (int qq = 0; qq < 8; ++qq)
                    *reinterpret_cast<uint4 *>(sP + pds_chunk(r, (kofs >> 3) + qq)) =
                        make_uint4(pk[4 * qq], pk[4 * qq + 1], pk[4 * qq + 2], pk[4 * qq + 3]);
                // dS = c P (dP - delta) in registers, then into shared memory once the
                // previous tile's dK and dQ have read it
                if (!mbar_wait_warp(dp_full, t & 1, abort, status)) { okw = false; break; }
                fence_after_sync();
                uint32_t ds[32];
                {
                    uint32_t dvv[64];
                    tmem_ld32(tmem + lane_base + T_DP + kofs, *reinterpret_cast<uint32_t(*)[32]>(dvv));
                    tmem_ld32(tmem + lane_base + T_DP + kofs + 32, *reinterpret_cast<uint32_t(*)[32]>(dvv + 32));
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pk[e / 2]));
                        ds[e / 2] = pack_bf16(c * pr.x * (__uint_as_float(dvv[e]) - dl),
                                              c * pr.y * (__uint_as_float(dvv[e + 1]) - dl));
                    }
                }
                if (t > 0 && !mbar_wait_warp(dq_full, (t - 1) & 1, abort, status)) { okw = false; break; }
#pragma unroll
                for (int qq = 0; qq < 8; ++qq)
                    *reinterpret_cast<uint4 *>(sDS + pds_chunk(r, (kofs >> 3) + qq)) =
                        make_uint4(ds[4 * qq], ds[4 * qq + 1], ds[4 * qq + 2], ds[4 * qq + 3]);
                fence_before_sync();  // dP is read: the next S may go to its columns
                fence_async_smem();
                mbar_arrive(pds_full);
                // the previous tile's dQ (its dq_full is complete), and its item's dK, dV
                // when it closed one
                if (have_prev) {
                    if (!dq_epilogue(t - 1, pb, ph, pj, pqi, false)) { okw = false; break; }
                    if (prev_last && !kv_flush(pnix, pb, ph, pj)) { okw = false; break; }
                }
                have_prev = true;
                pb = b; ph = h; pj = j; pqi = qi; pnix = n_item;
                prev_last = qi + 1 == q1;
            }
            ++n_item;
        }
        if (okw && have_prev) {
            if (dq_epilogue(t - 1, pb, ph, pj, pqi, true) && prev_last) kv_flush(pnix, pb, ph, pj);
        }
    }
    if (*abort) {
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
cudaError_t launch_rb(const AttnArgs &a, const void *dout, const float *lse, const float *delta,
                      void *dq, long ldq, float *dk, float *dv, cudaStream_t s) {
    using L = RbLayout<DPAD>;
    int *status = device_status_ptr();
    if (!status) return cudaErrorInvalidValue;
    if (a.tq.mode != THL_IDENTITY || a.tk.mode != THL_IDENTITY || a.tv.mode != THL_IDENTITY ||
        a.tq.vpad || a.tk.vpad || a.tv.vpad || L::TILE != (int)thl_block_bytes(a.d, 0))
        return cudaErrorInvalidValue;
    RbSched sc;
    sc.qt = (a.nq + BQ - 1) / BQ;
    sc.kt = (a.nk + BQ - 1) / BQ;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int base = a.B * a.heads * sc.kt;
    // about four items per SM, each of several query tiles where there are enough
    int splits = (4 * sms + base - 1) / base;
    splits = splits < sc.qt ? splits : sc.qt;
    sc.splits = splits < 1 ? 1 : splits;
    sc.items = base * sc.splits;
    const int grid = sc.items < sms ? sc.items : sms;
    cudaError_t e = cudaFuncSetAttribute(attn_rows_bwd_kernel<DPAD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_rows_bwd_kernel<DPAD>, dim3(grid), dim3(kThreads), L::BYTES, s, a, dout,
                      lse, delta, static_cast<__nv_bfloat16 *>(dq), ldq, dk, dv, sc, status);
}

}  // namespace

cudaError_t launch_attention_rows_bwd(const AttnArgs &a, const void *dout, const float *lse,
                                      const float *delta, void *dq, long ldq, float *dk, float *dv,
                                      cudaStream_t s) {
    if (a.d < 8 || a.d > 80 || a.d % 8 || a.nq < 1 || a.nk < 1) return cudaErrorInvalidValue;
    return a.d <= 64 ? launch_rb<64>(a, dout, lse, delta, dq, ldq, dk, dv, s)
                     : launch_rb<80>(a, dout, lse, delta, dq, ldq, dk, dv, s);
}

}  // namespace ptdit
