// One TCM branch's window Q/K/V projection and window attention in one kernel
// (Qihoo-T2X reading note, §3 Method, Eq. TCM): for windows of 128 tokens, the
// projection of a window's tokens onto one head's Q, K and V stays on chip and
// feeds that head's attention, so Q, K and V never travel through HBM.
//
// A unit is one window of one batch item; a job is one head of a unit.  One
// persistent CTA per SM takes a contiguous range of units, 320 threads:
//   warp 8       loader: per 64-channel block of a job, the window's 128 token
//                rows of z (a 5-D tensor map over [B, F, H, W, D]; a window of the
//                rolled grid is loaded as nb sub-boxes of R = 128 / nb rows, each
//                at its original coordinates, so a window that the roll wraps
//                needs no copy of z) and the head's weight rows [Wq_h; Wk_h; Wv_h]
//                (repacked as N = 3 d rounded up to 16 rows per head), three
//                stages.
//   warp 9       MMA issuer: the projection [Q K V] = Z [Wq_h; Wk_h; Wv_h]^T (M = 128,
//                N, K = D) into TMEM columns 0..N-1; while job j's projection runs,
//                job j-1's attention: S = Q K^T into columns 256..383 (once the
//                warpgroups have moved j-1's projection into shared memory), then
//                O = P V into the same columns (P from TMEM, written by the
//                softmax over S).
//   warps 0-7    both warpgroups move each job's projection out of TMEM as bf16
//                Q, K and V tiles (tiled head layout: the operands the attention
//                MMAs read), freeing the projection's columns for the next head;
//                warpgroup 1 then takes the job's softmax (thread r: query row r,
//                128 keys in two 64-key passes; keys in a sub-box the roll wrapped
//                apart from the row's masked) and its output O / l, written to the
//                tokens' rows of the [B N, D] output at the head's columns.
// TMEM: projection 0-255, S then O 256-383, P (bf16 pairs) 384-447.
// Every wait is bounded (2 s).
#include <math.h>

#include "tc_util.cuh"
#include "thl.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BQ = 128;            // token rows of a window
constexpr int kThreads = 320;
constexpr int KB = 64;             // channels per k-block
constexpr int NST = 3;             // operand stages
constexpr int kNMax = 240;         // weight rows per head: 3 d rounded up to 16 (d <= 80)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_ACC = 0, T_SO = 256, T_P = 384;

template <int DPAD>
struct FuLayout {
    static constexpr bool HAS_B = DPAD > 64;
    static constexpr int TILE_A = BQ * 128;
    static constexpr int TILE_B = HAS_B ? BQ * 32 : 0;
    static constexpr int TILE = TILE_A + TILE_B;       // one Q, K or V tile
    static constexpr int A_BYTES = BQ * 128;           // 128 rows x 64 channels
    static constexpr int B_BYTES = kNMax * 128;        // up to 240 weight rows x 64 channels
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int OFF_QKV = NST * STAGE;
    static constexpr int PITCH = DPAD * 2 + 16;        // output staging row pitch
    static constexpr int OFF_STG = OFF_QKV + 3 * TILE; // [4 warps][32 rows][PITCH]
    static constexpr int OFF_OROW = OFF_STG + 4 * 32 * PITCH;  // [128] output row of each tile row
    static constexpr int OFF_BAR = OFF_OROW + BQ * 8;
    // full[NST], empty[NST], acc_full, drained, s_full, p_full, o_full, o_free, qkv_free, drain
    static constexpr int NBARS = 2 * NST + 8;
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16;  // the kernel checks 1 KB alignment
    static_assert(STAGE % 1024 == 0 && OFF_QKV % 1024 == 0 && TILE % 1024 == 0,
                  "swizzled tiles stay 1 KB aligned");
    static_assert(BYTES <= 232448, "shared memory budget");
};

// Window u of the rolled grid: batch item and the window's origin (rolled frame).
struct UnitGeom {
    int b, t0, y0, x0;
    int lastt, lasty, lastx;  // the window is the last one along the dimension
};

__device__ __forceinline__ UnitGeom unit_geom(const WinFusedParams &p, int u) {
    const int nwx = p.W / p.wx, nwy = p.H / p.wy, nwt = p.F / p.wt;
    const int nwin = nwx * nwy * nwt;
    UnitGeom g;
    g.b = u / nwin;
    const int w = u - g.b * nwin;
    const int ix = w % nwx, iy = (w / nwx) % nwy, it = w / (nwx * nwy);
    g.t0 = it * p.wt;
    g.y0 = iy * p.wy;
    g.x0 = ix * p.wx;
    g.lastt = it == nwt - 1;
    g.lasty = iy == nwy - 1;
    g.lastx = ix == nwx - 1;
    return g;
}

// Sub-box i of the window: its origin in original coordinates and its region
// code (one bit per dimension: the part of a wrapped window that the roll
// brought from the grid's other end).
__device__ __forceinline__ void sub_box(const WinFusedParams &p, const UnitGeom &g, int i, int &t,
                                        int &y, int &x, int &code) {
    const int nbx = p.wx / p.bx, nby = p.wy / p.by;
    const int bxi = i % nbx, byi = (i / nbx) % nby, bti = i / (nbx * nby);
    const int rt = bti * p.bt, ry = byi * p.by, rx = bxi * p.bx;  // within the window
    t = (g.t0 + rt + p.st) % p.F;
    y = (g.y0 + ry + p.sy) % p.H;
    x = (g.x0 + rx + p.sx) % p.W;
    code = ((g.lastt && p.st > 0 && rt >= p.wt - p.st) ? 1 : 0) |
           ((g.lasty && p.sy > 0 && ry >= p.wy - p.sy) ? 2 : 0) |
           ((g.lastx && p.sx > 0 && rx >= p.wx - p.sx) ? 4 : 0);
}

// 10 warps: three share a sub-partition's 16384 registers, so 168 per thread at most.
template <int DPAD>
__global__ void __maxnreg__(168)
    win_fused_kernel(const __grid_constant__ CUtensorMap mz, const __grid_constant__ CUtensorMap mw,
                     const __grid_constant__ WinFusedParams p) {
    using L = FuLayout<DPAD>;
    extern __shared__ uint8_t sm_raw[];
    if (smem_u32(sm_raw) & 1023u) {  // no alignment slack in the allocation
        if (threadIdx.x == 0) atomicExch(p.status, 5 /* PTDIT_ERR_CUDA */);
        return;
    }
    uint8_t *sm = sm_raw;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *full = bars, *empty = bars + NST;
    uint64_t *acc_full = bars + 2 * NST, *drained = acc_full + 1, *s_full = acc_full + 2;
    uint64_t *p_full = acc_full + 3, *o_full = acc_full + 4, *o_free = acc_full + 5;
    uint64_t *qkv_free = acc_full + 6, *drain = acc_full + 7;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + L::NBARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);
    int *status = p.status;
    const uint64_t wns = p.wait_ns;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drained, 2 * BQ);
        mbar_init(s_full, 1);
        mbar_init(p_full, BQ);
        mbar_init(o_full, 1);
        mbar_init(o_free, BQ);
        mbar_init(qkv_free, 1);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    // the Q, K, V tiles' columns past the head are never written: zeros
    for (int i = threadIdx.x; i < 3 * L::TILE / 16; i += kThreads)
        reinterpret_cast<uint4 *>(sm + L::OFF_QKV)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    pdl_wait();  // the kernel that wrote z (and the repacked weights) has completed
    pdl_trigger();

    const int u0 = (int)((long)blockIdx.x * p.units / gridDim.x);
    const int u1 = (int)((long)(blockIdx.x + 1) * p.units / gridDim.x);
    const int J = (u1 - u0) * p.heads;  // jobs: (unit, head), head fastest
    const int KT = p.D / KB;

    if (warp == 8) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            prefetch_tensormap(&mz);
            prefetch_tensormap(&mw);
            int c = 0;
            bool ok = true;
            for (int j = 0; j < J && ok; ++j) {
                const int u = u0 + j / p.heads, h = j % p.heads;
                const UnitGeom g = unit_geom(p, u);
                for (int kb = 0; kb < KT; ++kb, ++c) {
                    const int s = c % NST;
                    if (!mbar_wait(&empty[s], ((c / NST) & 1) ^ 1, abort, status, wns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&full[s], L::A_BYTES + p.N * 128);
                    uint8_t *st = sm + s * L::STAGE;
                    for (int i = 0; i < p.nb; ++i) {
                        int t, y, x, code;
                        sub_box(p, g, i, t, y, x, code);
                        tma_load_5d(st + i * p.R * 128, &mz, &full[s], kb * KB, x, y, t, g.b);
                    }
                    tma_load_2d(st + L::A_BYTES, &mw, &full[s], kb * KB, h * p.N);
                }
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs the loop with warp-uniform operands; lane 0 issues)
        {
            constexpr uint32_t id_s = idesc_bf16(BQ, BQ);
            constexpr uint32_t id_o = idesc_bf16(BQ, 64, true);   // V columns 0..63
            constexpr uint32_t id_ob = idesc_bf16(BQ, 16, true);  // V columns 64..79
            const uint32_t id_acc = idesc_bf16(BQ, p.N);
            const uint32_t aQ = smem_u32(sm + L::OFF_QKV), aK = aQ + L::TILE, aV = aK + L::TILE;
            bool ok = true, any = false;
            // S(j) = Q K^T, once O(j - 1) has been read out of the same columns
            auto issue_s = [&](int j) {
                if (j >= 1 && !mbar_wait_warp(o_free, (j - 1) & 1, abort, status, wns)) return false;
                fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    warp_mma_bf16(tmem + T_SO, sdesc_sw128(aQ + kk * 32), sdesc_sw128(aK + kk * 32), id_s,
                             kk > 0);
                if (L::HAS_B)
                    warp_mma_bf16(tmem + T_SO, sdesc_sw32(aQ + L::TILE_A), sdesc_sw32(aK + L::TILE_A),
                             id_s, 1);
                warp_mma_commit(s_full);
                return true;
            };
            // O(j) = P(j) V into S's columns (P from TMEM, written by the softmax)
            auto issue_pv = [&]() {
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < BQ / 16; ++ks) {
                    warp_mma_bf16_ts(tmem + T_SO, tmem + T_P + ks * 8,
                                sdesc_sw128_mn(aV + ks * 2048, L::TILE_A), id_o, ks > 0);
                    if (L::HAS_B)
                        warp_mma_bf16_ts(tmem + T_SO + 64, tmem + T_P + ks * 8,
                                    sdesc_sw32_mn(aV + L::TILE_A + ks * 512), id_ob, ks > 0);
                }
                warp_mma_commit(o_full);
                warp_mma_commit(qkv_free);  // S and P V have read Q, K and V
            };
            int c = 0;
            for (int j = 0; j < J && ok; ++j) {
                bool pv_done = j == 0;
                if (j >= 1) {
                    // job j-1's projection is out of TMEM (its Q, K, V in shared memory)
                    if (!mbar_wait_warp(drained, (j - 1) & 1, abort, status, wns) || !issue_s(j - 1)) break;
                }
                for (int kb = 0; kb < KT; ++kb, ++c) {
                    const int s = c % NST;
                    if (!mbar_wait_warp(&full[s], (c / NST) & 1, abort, status, wns)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    const uint32_t aA = smem_u32(sm + s * L::STAGE), aB = aA + L::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        warp_mma_bf16(tmem + T_ACC, sdesc_sw128(aA + kk * 32), sdesc_sw128(aB + kk * 32),
                                 id_acc, kb > 0 || kk > 0);
                    warp_mma_commit(&empty[s]);
                    any = true;
                    // job j-1's P V as soon as its softmax is done (lane 0's answer
                    // for the whole warp, so that the warp stays converged)
                    if (!pv_done &&
                        __shfl_sync(0xffffffffu, (int)mbar_test_wait(p_full, (j - 1) & 1), 0)) {
                        issue_pv();
                        pv_done = true;
                    }
                }
                if (!ok) break;
                warp_mma_commit(acc_full);
                if (!pv_done) {
                    if (!mbar_wait_warp(p_full, (j - 1) & 1, abort, status, wns)) break;
                    issue_pv();
                }
            }
            // the last job's attention
            if (ok && J > 0 && mbar_wait_warp(drained, (J - 1) & 1, abort, status, wns) && issue_s(J - 1) &&
                mbar_wait_warp(p_full, (J - 1) & 1, abort, status, wns))
                issue_pv();
            if (any) {  // every issued MMA has finished before TMEM is released
                warp_mma_commit(drain);
                volatile int never = 0;
                mbar_wait_warp(drain, 0, &never, status);
            }
        }
    } else {
        // ------------------------------------------------------------ warps 0-7
        const int g = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int d = p.d, ncu = d / 8, nchunk = p.N / 16;
        const float sl2 = p.scale * 1.4426950408889634f;
        uint8_t *qkv = sm + L::OFF_QKV;
        int cur_u = -1;
        long orow_r = 0;         // this row's output row
        uint32_t allow = 0xffffu;  // sub-boxes whose keys this row may attend
        bool masked = false;
        for (int j = 0; j < J; ++j) {
            // ---- both warpgroups: the projection out of TMEM as bf16 Q, K, V tiles
            if (!mbar_wait_warp(acc_full, j & 1, abort, status, wns)) break;
            if (j >= 1 && !mbar_wait_warp(qkv_free, (j - 1) & 1, abort, status, wns)) break;
            fence_after_sync();
            for (int ck = g; ck < nchunk; ck += 4) {
                // 16-column chunks ck and ck + 2 (warpgroup g takes chunks = g mod 2)
                uint32_t v[32];
                const bool two = ck + 2 < nchunk;
                tmem_ld16(tmem + lane_base + T_ACC + 16 * ck, *reinterpret_cast<uint32_t(*)[16]>(v));
                if (two)
                    tmem_ld16(tmem + lane_base + T_ACC + 16 * (ck + 2),
                              *reinterpret_cast<uint32_t(*)[16]>(v + 16));
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (q >= 2 && !two) break;
                    const int unit = q < 2 ? 2 * ck + q : 2 * (ck + 2) + (q - 2);
                    const int m = unit / ncu, pc = unit - m * ncu;
                    if (m >= 3) continue;  // the rows past 3 d (zero weights)
                    const uint32_t *w = v + 8 * q;
                    uint4 o;
                    o.x = pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1]));
                    o.y = pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3]));
                    o.z = pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5]));
                    o.w = pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7]));
                    *reinterpret_cast<uint4 *>(qkv + m * L::TILE + thl_unit(r, pc, 0)) = o;
                }
            }
            fence_async_smem();
            fence_before_sync();
            mbar_arrive(drained);
            if (g == 0) continue;
            // ---- warpgroup 1: softmax, then O / l
            const int u = u0 + j / p.heads, h = j % p.heads;
            if (u != cur_u) {
                cur_u = u;
                const UnitGeom ug = unit_geom(p, u);
                const int i = r / p.R, o = r - i * p.R;
                int t, y, x, code;
                sub_box(p, ug, i, t, y, x, code);
                const int ox = o % p.bx, oy = (o / p.bx) % p.by, ot = o / (p.bx * p.by);
                orow_r = (((long)ug.b * p.F + t + ot) * p.H + y + oy) * p.W + x + ox;
                allow = 0u;
                for (int k = 0; k < p.nb; ++k) {
                    int tk, yk, xk, ck2;
                    sub_box(p, ug, k, tk, yk, xk, ck2);
                    if (ck2 == code) allow |= 1u << k;
                }
                masked = allow != (p.nb >= 32 ? 0xffffffffu : ((1u << p.nb) - 1u));
            }
            if (!mbar_wait_warp(s_full, j & 1, abort, status, wns)) break;
            fence_after_sync();
            float mx = -INFINITY;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t sv[64];
                tmem_ld32(tmem + lane_base + T_SO + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(sv));
                tmem_ld32(tmem + lane_base + T_SO + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                tmem_ld_wait();
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (!masked) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(sv[e]));
                } else {
#pragma unroll
                    for (int e = 0; e < 64; ++e)
                        if ((allow >> ((64 * hf + e) / p.R)) & 1u)
                            m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(sv[e]));
                }
                mx = fmaxf(mx, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
            }
            const float ref = mx * sl2;  // the row's own key is always allowed: finite
            float l = 0.f;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t sv[64];
                tmem_ld32(tmem + lane_base + T_SO + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(sv));
                tmem_ld32(tmem + lane_base + T_SO + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                tmem_ld_wait();
                uint32_t pk[32];
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
                if (!masked) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), sl2, -ref));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -ref));
                        ps[c & 3] += p0 + p1;
                        pk[c] = pack_bf16(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e = 64 * hf + 2 * c;
                        const float p0 = ((allow >> (e / p.R)) & 1u)
                                             ? ex2_approx(fmaf(__uint_as_float(sv[2 * c]), sl2, -ref))
                                             : 0.f;
                        const float p1 = ((allow >> ((e + 1) / p.R)) & 1u)
                                             ? ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -ref))
                                             : 0.f;
                        ps[c & 3] += p0 + p1;
                        pk[c] = pack_bf16(p0, p1);
                    }
                }
                l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
                tmem_st32(tmem + lane_base + T_P + 32 * hf, pk);
            }
            tmem_st_wait();
            fence_before_sync();
            mbar_arrive(p_full);
            // O / l to the tokens' rows: each warp stages its 32 rows and stores them with
            // consecutive lanes on consecutive 16-byte pieces of a row
            if (!mbar_wait_warp(o_full, j & 1, abort, status, wns)) break;
            fence_after_sync();
            const int wq = warp & 3;
            uint8_t *stg = sm + L::OFF_STG + wq * 32 * L::PITCH;
            long *orow = reinterpret_cast<long *>(sm + L::OFF_OROW) + wq * 32;  // 32 rows per warp
            {
                uint32_t ov[DPAD];
                tmem_ld32(tmem + lane_base + T_SO, *reinterpret_cast<uint32_t(*)[32]>(ov));
                tmem_ld32(tmem + lane_base + T_SO + 32, *reinterpret_cast<uint32_t(*)[32]>(ov + 32));
                if (DPAD > 64) tmem_ld16(tmem + lane_base + T_SO + 64, *reinterpret_cast<uint32_t(*)[16]>(ov + 64));
                tmem_ld_wait();
                fence_before_sync();
                mbar_arrive(o_free);  // O is read: the next S may go to these columns
                const float inv = 1.f / l;
#pragma unroll
                for (int uu = 0; uu < DPAD / 8; ++uu)
                    if (uu < ncu) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(ov[8 * uu + 0]) * inv, __uint_as_float(ov[8 * uu + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(ov[8 * uu + 2]) * inv, __uint_as_float(ov[8 * uu + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(ov[8 * uu + 4]) * inv, __uint_as_float(ov[8 * uu + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(ov[8 * uu + 6]) * inv, __uint_as_float(ov[8 * uu + 7]) * inv);
                        *reinterpret_cast<uint4 *>(stg + lane * L::PITCH + uu * 16) = v;
                    }
            }
            orow[lane] = orow_r;
            __syncwarp();
            {
                const int drow = 32 / ncu, dpc = 32 % ncu;
                int row = lane / ncu, pc = lane % ncu;
                __nv_bfloat16 *obase = p.o + (long)h * d;
#pragma unroll 1
                for (int i = lane; i < 32 * ncu; i += 32) {
                    *reinterpret_cast<uint4 *>(obase + orow[row] * p.ldo + pc * 8) =
                        *reinterpret_cast<const uint4 *>(stg + row * L::PITCH + pc * 16);
                    row += drow;
                    pc += dpc;
                    if (pc >= ncu) {
                        pc -= ncu;
                        ++row;
                    }
                }
            }
            __syncwarp();
        }
    }
    if (*abort) {  // a role gave up: let the copies and MMAs in flight land
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

// [Wq_h; Wk_h; Wv_h] rows of every head, N rows per head (rows past 3 d zero): one thread
// per 16-byte piece of a row.
__global__ void repack_qkv_kernel(const __nv_bfloat16 *__restrict__ wq,
                                  const __nv_bfloat16 *__restrict__ wk,
                                  const __nv_bfloat16 *__restrict__ wv, int heads, int d, int D,
                                  int N, __nv_bfloat16 *__restrict__ out) {
    pdl_wait();
    pdl_trigger();
    const int pieces = D / 8;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)heads * N * pieces) return;
    const int pc = static_cast<int>(idx % pieces);
    const long row = idx / pieces;
    const int h = static_cast<int>(row / N), n = static_cast<int>(row - (long)h * N);
    const int m = n / d, c = n - m * d;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m < 3) {
        const __nv_bfloat16 *w = m == 0 ? wq : (m == 1 ? wk : wv);
        v = *reinterpret_cast<const uint4 *>(w + ((long)h * d + c) * D + 8 * pc);
    }
    *reinterpret_cast<uint4 *>(out + row * D + 8 * pc) = v;
}

int gcd_int(int a, int b) {
    while (b) {
        const int t = a % b;
        a = b;
        b = t;
    }
    return a;
}

}  // namespace

bool win_fused_plan(int D, int heads, int d, const int window[3], const int shift[3],
                    WinFusedParams *p) {
    if (d < 8 || d > 80 || d % 8 || D % KB || D != heads * d) return false;
    if (window[0] * window[1] * window[2] != BQ) return false;
    int box[3];
    for (int k = 0; k < 3; ++k) {
        if (shift[k] < 0 || shift[k] >= window[k]) return false;
        box[k] = shift[k] == 0 ? window[k] : gcd_int(window[k], shift[k]);
    }
    const int nb = BQ / (box[0] * box[1] * box[2]);
    const int R = BQ / nb;
    if (nb > 16 || R % 8 || box[2] > 256 || box[1] > 256 || box[0] > 256) return false;
    memset(p, 0, sizeof *p);
    p->D = D;
    p->heads = heads;
    p->d = d;
    p->N = (3 * d + 15) / 16 * 16;
    p->wt = window[0]; p->wy = window[1]; p->wx = window[2];
    p->st = shift[0]; p->sy = shift[1]; p->sx = shift[2];
    p->bt = box[0]; p->by = box[1]; p->bx = box[2];
    p->nb = nb;
    p->R = R;
    return p->N <= kNMax;
}

size_t win_fused_weight_bytes(const WinFusedParams &p) {
    return (size_t)p.heads * p.N * p.D * 2;
}

cudaError_t launch_repack_qkv(const void *wq, const void *wk, const void *wv,
                              const WinFusedParams &p, void *out, cudaStream_t s) {
    const long n = (long)p.heads * p.N * (p.D / 8);
    const int threads = 256;
    return launch_pdl(repack_qkv_kernel, dim3((unsigned)((n + threads - 1) / threads)),
                      dim3(threads), 0, s, static_cast<const __nv_bfloat16 *>(wq),
                      static_cast<const __nv_bfloat16 *>(wk), static_cast<const __nv_bfloat16 *>(wv),
                      p.heads, p.d, p.D, p.N, static_cast<__nv_bfloat16 *>(out));
}

cudaError_t launch_win_fused(const void *z, const void *wr, WinFusedParams p, cudaStream_t s) {
    if (p.F % p.wt || p.H % p.wy || p.W % p.wx || p.B < 1) return cudaErrorInvalidValue;
    CUtensorMap mz, mw;
    if (!encode_map_grid_bf16(&mz, z, p.B, p.F, p.H, p.W, p.D, KB, p.bx, p.by, p.bt))
        return cudaErrorInvalidValue;
    if (!encode_map_2d_bf16(&mw, wr, p.D, (uint64_t)p.heads * p.N, (uint64_t)p.D * 2, KB, p.N))
        return cudaErrorInvalidValue;
    p.units = p.B * (p.F / p.wt) * (p.H / p.wy) * (p.W / p.wx);
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorInvalidValue;
    p.wait_ns = debug_wait_limit_ns();
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int grid = p.units < sms ? p.units : sms;
    if (p.d <= 64) {
        using L = FuLayout<64>;
        cudaError_t e = cudaFuncSetAttribute(win_fused_kernel<64>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
        if (e != cudaSuccess) return e;
        return launch_pdl(win_fused_kernel<64>, dim3(grid), dim3(kThreads), L::BYTES, s, mz, mw, p);
    }
    using L = FuLayout<80>;
    cudaError_t e = cudaFuncSetAttribute(win_fused_kernel<80>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(win_fused_kernel<80>, dim3(grid), dim3(kThreads), L::BYTES, s, mz, mw, p);
}

}  // namespace ptdit
