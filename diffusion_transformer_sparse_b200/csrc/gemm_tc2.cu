// Projections y = x W^T (+ residual) on pairs of SMs: tcgen05.mma.cta_group::2.
//
// A cluster of two CTAs computes a 256 x BN output tile with one MMA stream:
// each CTA loads its own 128 rows of A and its own BN/2 rows of the weight
// tile, and the pair's tensor cores read both halves.  Every operand byte is
// written into shared memory once (TMA) and read once (MMA), so the tile's
// bytes per FLOP set the shared-memory traffic per MMA: a 256 x 256 pair tile
// moves 16 KB per SM per K = 16 step of 128 tensor cycles, a 256 x 192 tile
// 14 KB per 96 cycles.  The last tile of a matrix whose width is not a
// multiple of BN is narrower (e.g. 1152 = 4 x 256 + 128): its MMAs run with
// the smaller N and its weight rows are split between the CTAs by that N.
//
//   warp 0     producer (both CTAs): TMA loads (the .cta_group::2 form, no
//              multicast) of the CTA's A and B halves; both CTAs' copies
//              complete on the leader CTA's full barrier, which the leader
//              alone arms with the byte count of the pair.
//   warp 1     MMA issuer (leader CTA only): 4 x tcgen05.mma.cta_group::2
//              (M = 256, K = 16) per stage; tcgen05.commit multicast frees
//              the stage in both CTAs and hands the accumulator to both
//              epilogues.
//   warps 2-5  epilogue (both CTAs): each warp owns 32 rows of its CTA's TMEM
//              half.  Before it waits for a tile's accumulator it starts the
//              TMA load of its residual rows into its own staging tile, so
//              that load overlaps the MMAs.  It then reads the accumulator
//              32 columns at a time, adds the residual from shared memory,
//              rounds, writes the result back over the staging tile, tells
//              the leader (a remote mbarrier arrive from the peer) that the
//              accumulator is free, and writes the tile out with TMA stores:
//              whole 64-byte row segments instead of one 16-byte piece per
//              row and instruction.  An output in tiled head layout (the Q,
//              K and V operands of the attention kernels) is written
//              instead straight from registers, 16 bytes (8 columns of one
//              head) at a time, into its (tile, head) block at the row's
//              place in the swizzled tile; the block's padding columns are
//              written as zeros by the lane that writes the head's last
//              columns.
// Two TMEM accumulators overlap the next tile's MMAs with this tile's
// epilogue.  Every wait is bounded (2 s); a timeout records
// PTDIT_ERR_TIMEOUT in the status word.
#include <algorithm>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include "tc_util.cuh"
#include "thl.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BMC = 128, BK = 64;  // rows of A per CTA, K per stage
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

// Output and residual maps: box of 32 columns x 32 rows, 64-byte swizzle.
struct Tc2Maps {
    CUtensorMap C[3], R[3];
};

constexpr int kMaxPairs = 128;   // pairs a schedule can describe
constexpr int kMaxSched = 4096;  // tiles a schedule can describe (larger launches: round robin)

struct Tc2Params {
    void *C[3];
    const void *R[3];
    const void *bias[3];  // row-major outputs: bias added before act and the residual
    int act;              // GemmAct
    Thl thl[3];  // mode THL_OFF: row-major output through the staging tiles
    int heads, d;     // tiled outputs: heads and head width
    int nunits[3];    // tiled outputs: 16-byte units per block row
    FastDiv f_d;
    uint32_t blk[3];  // tiled outputs: bytes per (tile, head) block
    long ldc;
    int rows, nseg, nmat;
    int n_tiles;  // output tiles per weight matrix (the last may be narrower)
    int tiles;    // all pair tiles
    int kblocks;
    int *status;
    // Tile schedule: pair q runs tiles sched[first[q]] .. sched[first[q + 1] - 1] in
    // that order; nsched == 0 means round robin (tile t to pair t % pairs).
    int nsched;
    uint16_t first[kMaxPairs + 1];
    uint16_t sched[kMaxSched];
};

// STAGING: the row-major epilogue's staging tiles exist (launches whose outputs
// are all in tiled head layout leave them out and use the room for stages).
template <int BN, int STAGES, bool STAGING, int SCH>
struct Layout2 {
    static constexpr int A_BYTES = BMC * BK * 2;       // 16 KB: this CTA's rows of A
    static constexpr int B_BYTES = (BN / 2) * BK * 2;  // this CTA's half of the weight tile
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int CHUNK_BYTES = 32 * 64;          // 32 rows x 32 bf16 columns
    static constexpr int WARP_STAGE = STAGING ? SCH * CHUNK_BYTES : 0;  // SCH chunks per pass
    static constexpr int EPI_OFF = STAGES * STAGE_BYTES;  // 4 epilogue warps' staging tiles
    static constexpr int BAR_OFF = EPI_OFF + 4 * WARP_STAGE;
    static constexpr int NBARS = 2 * STAGES + 9;  // full, empty, tfull[2], tempty[2], rfull[4], drain
    static constexpr int BYTES = BAR_OFF + NBARS * 8 + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t ACC_STRIDE = BN <= 128 ? 128 : 256;
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "stage tiles stay 1 KB aligned");
    static_assert(2 * ACC_STRIDE <= kTmemCols, "two accumulators must fit in TMEM");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// Shared-memory address of `local`'s counterpart in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void *local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
    return r;
}

__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map,
                                                 uint32_t leader_bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
        : "memory");
}

// The issuer runs as a whole converged warp (warp-uniform operands); lane 0
// alone issues, under a predicate inside each instruction sequence.
//
// D (+)= A B^T on the CTA pair: M = 256, each CTA holding its 128 rows of A and
// half of B's rows, the accumulator in each CTA's TMEM.
__device__ __forceinline__ void warp_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                   uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .u32 l;\n\t"
        "mov.u32 l, %%laneid;\n\t"
        "setp.eq.u32 e, l, 0;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on `bar` in both CTAs of the pair once the pair's MMAs so far have completed.
__device__ __forceinline__ void warp_mma_commit_pair(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .u32 l;\n\t"
        "mov.u32 l, %%laneid;\n\t"
        "setp.eq.u32 e, l, 0;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}
// The same, arriving on this CTA's `bar` only.
__device__ __forceinline__ void warp_mma_commit_pair_local(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .u32 l;\n\t"
        "mov.u32 l, %%laneid;\n\t"
        "setp.eq.u32 e, l, 0;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

__device__ __forceinline__ void decode_tile2(const Tc2Params &p, int t, int &m_tile, int &seg,
                                             int &n_tile) {
    const int per_m = p.nmat * p.n_tiles;
    m_tile = t / per_m;
    const int n = t % per_m;
    seg = n / p.n_tiles;
    n_tile = n % p.n_tiles;
}

// The k-th tile of pair `pair` (-1 when it has no more).
__device__ __forceinline__ int pair_tile(const Tc2Params &p, int pair, int npairs, int k) {
    if (p.nsched) {
        const int i = p.first[pair] + k;
        return i < p.first[pair + 1] ? p.sched[i] : -1;
    }
    const int t = pair + k * npairs;
    return t < p.tiles ? t : -1;
}

// Output columns of tile n_tile: BN, or what is left of the matrix for the last one.
template <int BN>
__device__ __forceinline__ int tile_width(const Tc2Params &p, int n_tile) {
    const int w = p.nseg - n_tile * BN;
    return w < BN ? w : BN;
}

template <int BN, int STAGES, bool STAGING, int SCH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB0,
                    const __grid_constant__ CUtensorMap mB1,
                    const __grid_constant__ CUtensorMap mB2, const __grid_constant__ Tc2Maps mo,
                    const __grid_constant__ Tc2Params p) {
    using L = Layout2<BN, STAGES, STAGING, SCH>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *rfull = tempty + 2;
    uint64_t *drain = rfull + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x / 2, npairs = gridDim.x / 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 8);  // one arrive per epilogue warp of both CTAs
        }
        for (int w = 0; w < 4; ++w) mbar_init(&rfull[w], 1);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    cluster_sync();  // barriers of both CTAs are initialised before anyone signals them
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // everything above touched only this CTA: from here on, the previous
    // kernel's outputs (A, the residual) must be complete
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&mA);
            prefetch_tensormap(&mB0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kt = 0, t; ok && (t = pair_tile(p, pair, npairs, kt)) >= 0; ++kt) {
                int m_tile, seg, n_tile;
                decode_tile2(p, t, m_tile, seg, n_tile);
                const CUtensorMap *mb = seg == 0 ? &mB0 : (seg == 1 ? &mB1 : &mB2);
                const int arow = m_tile * 2 * BMC + rank * BMC;
                const int brow = n_tile * BN + rank * (tile_width<BN>(p, n_tile) / 2);
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * L::STAGE_BYTES;
                    const uint32_t lbar = cluster_addr(&full[stage], 0);
                    if (leader) mbar_expect_tx(&full[stage], 2 * L::STAGE_BYTES);
                    tma_load_2d_pair(sa, &mA, lbar, kb * BK, arow);
                    tma_load_2d_pair(sa + L::A_BYTES, mb, lbar, kb * BK, brow);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // the MMA issuer: the whole warp of the pair's leader CTA runs the loop,
        // lane 0 issues
        if (leader) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, any = false;
            for (int kt = 0, t; ok && (t = pair_tile(p, pair, npairs, kt)) >= 0; ++kt) {
                int m_tile, seg, n_tile;
                decode_tile2(p, t, m_tile, seg, n_tile);
                const uint32_t idesc = idesc_bf16(2 * BMC, tile_width<BN>(p, n_tile));
                if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1, abort, p.status)) break;
                fence_after_sync();
                const uint32_t d = tmem + acc * L::ACC_STRIDE;
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait_warp(&full[stage], phase, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    const uint32_t sa = smem_u32(smem + stage * L::STAGE_BYTES);
                    const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        warp_mma_bf16_pair(d, sdesc_sw128(sa + kk * 32), sdesc_sw128(sb + kk * 32),
                                           idesc, (kb | kk) != 0);
                    any = true;
                    warp_mma_commit_pair(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                warp_mma_commit_pair(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                warp_mma_commit_pair_local(drain);
                volatile int never = 0;
                mbar_wait_warp(drain, 0, &never, p.status);
            }
        }
    } else {
        const int q = warp % 4;  // TMEM lanes 32q .. 32q+31 belong to this warp
        uint8_t *stg = smem + L::EPI_OFF + q * L::WARP_STAGE;
        const uint32_t tempty_leader0 = cluster_addr(&tempty[0], 0);
        const uint32_t tempty_leader1 = cluster_addr(&tempty[1], 0);
        // 64-byte swizzle of the staging tiles: 16-byte unit j of row r sits at
        // unit j ^ ((r >> 1) & 3), which spreads a warp's row accesses over all banks
        const uint32_t row_off = lane * 64;
        const uint32_t sw = (lane >> 1) & 3;
        int acc = 0;
        uint32_t acc_phase = 0, r_phase = 0;
        for (int kt = 0, t; (t = pair_tile(p, pair, npairs, kt)) >= 0; ++kt) {
            int m_tile, seg, n_tile;
            decode_tile2(p, t, m_tile, seg, n_tile);
            const int row0 = m_tile * 2 * BMC + rank * BMC + q * 32;
            const int col0 = n_tile * BN;
            // 32-column chunks; a tile whose width is 16 past a multiple of 32 ends in a
            // half chunk (its other 16 columns are outside the matrix: not stored)
            const int cend = col0 + tile_width<BN>(p, n_tile);
            const int nchunk = (tile_width<BN>(p, n_tile) + 31) / 32;
            if (p.thl[seg].mode != THL_OFF) {
                // ---- tiled head layout: this lane's row, 8 columns per store
                const Thl &tl = p.thl[seg];
                const int grow = row0 + lane;
                uint8_t *rbase = nullptr;
                int tr = 0;
                if (grow < p.rows) {
                    const int b = grow / static_cast<int>(tl.rows_pb);
                    int tile;
                    thl_locate(tl, grow - static_cast<long>(b) * tl.rows_pb, tile, tr);
                    rbase = static_cast<uint8_t *>(p.C[seg]) +
                            ((long)b * tl.tiles + tile) * p.heads * (long)p.blk[seg];
                }
                if (!mbar_wait(&tfull[acc], acc_phase, abort, p.status)) break;
                fence_after_sync();
                const uint32_t tbase =
                    tmem + acc * L::ACC_STRIDE + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
                for (int c = 0; c < nchunk; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tbase + 32 * c, r);
                    tmem_ld_wait();
                    if (!rbase) continue;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int col = col0 + 32 * c + 8 * j;
                        if (col >= cend) break;
                        const int h = fdiv(p.f_d, col), u = (col - h * p.d) >> 3;
                        uint8_t *hb = rbase + (long)h * p.blk[seg];
                        uint4 o;
                        o.x = pack_bf16(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
                        o.y = pack_bf16(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
                        o.z = pack_bf16(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
                        o.w = pack_bf16(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
                        *reinterpret_cast<uint4 *>(hb + thl_unit(tr, u, tl.vpad)) = o;
                        if (8 * (u + 1) == p.d)  // the head's last columns: write the padding units
                            for (int z = u + 1; z < p.nunits[seg]; ++z)
                                *reinterpret_cast<uint4 *>(hb + thl_unit(tr, z, tl.vpad)) =
                                    (tl.ones && z == u + 1) ? thl_ones_unit() : make_uint4(0, 0, 0, 0);
                    }
                }
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
                continue;
            }
            if (!STAGING) break;  // not launched with row-major outputs
            const bool has_r = p.R[seg] != nullptr;
            const uint32_t tbase = tmem + acc * L::ACC_STRIDE + (static_cast<uint32_t>(q * 32) << 16);
            bool ok = true;
            // the tile's chunks in passes of SCH through the warp's staging tiles
#pragma unroll 1
            for (int c0 = 0; c0 < nchunk && ok; c0 += SCH) {
                const int c1 = c0 + SCH < nchunk ? c0 + SCH : nchunk;
                if (lane == 0) {
                    bulk_wait_read_all();  // the previous pass's stores have left the staging tiles
                    if (has_r) {
                        mbar_expect_tx(&rfull[q], (c1 - c0) * L::CHUNK_BYTES);
#pragma unroll 1
                        for (int c = c0; c < c1; ++c)
                            tma_load_2d(stg + (c - c0) * L::CHUNK_BYTES, &mo.R[seg], &rfull[q],
                                        col0 + 32 * c, row0);
                    }
                }
                __syncwarp();
                if (c0 == 0 && !mbar_wait(&tfull[acc], acc_phase, abort, p.status)) { ok = false; break; }
                if (has_r) {
                    if (!mbar_wait(&rfull[q], r_phase, abort, p.status)) { ok = false; break; }
                    r_phase ^= 1;
                }
                fence_after_sync();
#pragma unroll 1
                for (int c = c0; c < c1; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tbase + 32 * c, r);
                    tmem_ld_wait();
                    uint8_t *chunk = stg + (c - c0) * L::CHUNK_BYTES + row_off;
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                    if (p.bias[seg]) {  // the 32 columns of this chunk: the same for every lane
                        const uint4 *bp = reinterpret_cast<const uint4 *>(
                            static_cast<const __nv_bfloat16 *>(p.bias[seg]) + col0 + 32 * c);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (col0 + 32 * c + 8 * j >= cend) break;
                            const uint4 bv = __ldg(bp + j);
                            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&bv);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = __bfloat1622float2(h[e]);
                                v[8 * j + 2 * e] += f.x;
                                v[8 * j + 2 * e + 1] += f.y;
                            }
                        }
                    }
                    if (p.act == ACT_GELU_TANH) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = gelu_tanh_fast(v[i]);
                    }
                    if (has_r) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint4 rv = *reinterpret_cast<const uint4 *>(chunk + ((j ^ sw) << 4));
                            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&rv);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = __bfloat1622float2(h[e]);
                                v[8 * j + 2 * e] += f.x;
                                v[8 * j + 2 * e + 1] += f.y;
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint4 o;
                        o.x = pack_bf16(v[8 * j + 0], v[8 * j + 1]);
                        o.y = pack_bf16(v[8 * j + 2], v[8 * j + 3]);
                        o.z = pack_bf16(v[8 * j + 4], v[8 * j + 5]);
                        o.w = pack_bf16(v[8 * j + 6], v[8 * j + 7]);
                        *reinterpret_cast<uint4 *>(chunk + ((j ^ sw) << 4)) = o;
                    }
                }
                fence_before_sync();
                fence_async_smem();  // the staging writes become visible to the TMA stores
                __syncwarp();
                if (lane == 0) {
                    if (c1 == nchunk)  // the accumulator is read: the next tile may overwrite it
                        mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
#pragma unroll 1
                    for (int c = c0; c < c1; ++c)
                        tma_store_2d(&mo.C[seg], stg + (c - c0) * L::CHUNK_BYTES, col0 + 32 * c, row0);
                    bulk_commit();
                }
            }
            if (!ok) break;
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
        if (lane == 0) bulk_wait_all();
    }
    if (*abort) {
        // give copies still in flight into this CTA a moment to land
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 100000) {
        }
    }
    fence_before_sync();
    cluster_sync();  // no CTA leaves while its peer may still signal it
    if (warp == 0) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// Longest-processing-time schedule of the pair tiles: tiles by decreasing
// width (the work of a tile is proportional to its columns), each to the pair
// with the least work so far; each pair then runs its tiles in index order
// (row blocks of A in sequence, as the pairs together sweep A).  Cached per
// launch shape; only for launches of at most kMaxSched tiles, where the
// round robin's imbalance (a few tiles per pair, some of half width) costs.
struct SchedKey {
    int tiles, per_m, n_tiles, nseg, bn, pairs;
    bool operator<(const SchedKey &o) const {
        return std::tie(tiles, per_m, n_tiles, nseg, bn, pairs) <
               std::tie(o.tiles, o.per_m, o.n_tiles, o.nseg, o.bn, o.pairs);
    }
};
struct SchedVal {
    std::vector<uint16_t> first, tile;
};

// Whether a launch of `tiles` tiles on `pairs` pairs runs a schedule (else round robin).
bool takes_schedule(int tiles, int pairs, int nseg, int bn) {
    return tiles <= kMaxSched && pairs <= kMaxPairs && nseg % bn != 0;
}

const SchedVal *tile_schedule(const SchedKey &k) {
    static std::mutex mu;
    static std::map<SchedKey, SchedVal> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(k);
    if (it != cache.end()) return &it->second;
    std::vector<int> order(k.tiles), width(k.tiles);
    for (int t = 0; t < k.tiles; ++t) {
        const int n_tile = (t % k.per_m) % k.n_tiles;
        const int w = k.nseg - n_tile * k.bn;
        width[t] = w < k.bn ? w : k.bn;
        order[t] = t;
    }
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return width[a] > width[b]; });
    std::vector<std::vector<int>> lists(k.pairs);
    std::priority_queue<std::pair<long, int>, std::vector<std::pair<long, int>>,
                        std::greater<std::pair<long, int>>>
        load;
    for (int q = 0; q < k.pairs; ++q) load.push({0L, q});
    for (int t : order) {
        auto top = load.top();
        load.pop();
        lists[top.second].push_back(t);
        load.push({top.first + width[t], top.second});
    }
    SchedVal v;
    v.first.push_back(0);
    for (auto &l : lists) {
        std::sort(l.begin(), l.end());
        for (int t : l) v.tile.push_back(static_cast<uint16_t>(t));
        v.first.push_back(static_cast<uint16_t>(v.tile.size()));
    }
    return &cache.emplace(k, std::move(v)).first->second;
}

template <int BN, int STAGES, bool STAGING, int SCH>
cudaError_t launch_bn2(const GemmArgs &a, cudaStream_t s) {
    using L = Layout2<BN, STAGES, STAGING, SCH>;
    CUtensorMap mA, mB[3];
    // a refused tensor map sends the caller to another kernel
    if (!encode_map_2d_bf16(&mA, a.A, a.K, a.rows, a.lda * 2, BK, BMC)) return cudaErrorNotSupported;
    for (int i = 0; i < 3; ++i) {
        const void *w = i < a.nmat ? a.W[i] : a.W[0];
        if (!encode_map_2d_bf16(&mB[i], w, a.K, a.nseg, (uint64_t)a.K * 2, BK, BN / 2))
            return cudaErrorNotSupported;
    }
    Tc2Params p;
    Tc2Maps mo;
    memset(&p, 0, sizeof p);
    p.heads = a.heads;
    p.d = a.d > 0 ? a.d : 1;
    p.f_d = make_fastdiv(p.d);
    for (int i = 0; i < 3; ++i) {
        p.C[i] = i < a.nmat ? a.C[i] : nullptr;
        p.R[i] = i < a.nmat ? a.R[i] : nullptr;
        p.bias[i] = i < a.nmat ? a.bias[i] : nullptr;
        if (i < a.nmat && a.thl[i]) {
            p.thl[i] = *a.thl[i];
            p.blk[i] = thl_block_bytes(a.d, a.thl[i]->vpad);
            p.nunits[i] = thl_units(a.d, a.thl[i]->vpad);
        }
        // unused slots get a valid map over C[0] that no tile refers to
        const void *c = p.C[i] ? p.C[i] : a.C[0];
        const void *r = p.R[i] ? p.R[i] : c;
        if (!encode_map_2d_bf16_sw(&mo.C[i], c, a.nseg, a.rows, (uint64_t)a.ldc * 2, 32, 32, 64) ||
            !encode_map_2d_bf16_sw(&mo.R[i], r, a.nseg, a.rows, (uint64_t)a.ldc * 2, 32, 32, 64))
            return cudaErrorNotSupported;
    }
    p.act = a.act;
    p.ldc = a.ldc;
    p.rows = a.rows;
    p.nseg = a.nseg;
    p.nmat = a.nmat;
    p.n_tiles = (a.nseg + BN - 1) / BN;
    p.kblocks = (a.K + BK - 1) / BK;  // a last partial K block reads zeros past K
    const int m_tiles = (a.rows + 2 * BMC - 1) / (2 * BMC);
    p.tiles = m_tiles * a.nmat * p.n_tiles;
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gemm_tc2_kernel<BN, STAGES, STAGING, SCH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    // persistent grid: as many pairs as can be resident at once (pairs must
    // share a GPC, so this can be below half the SM count)
    static int max_pairs = 0;
    if (!max_pairs) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 74, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = L::ALLOC;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<BN, STAGES, STAGING, SCH>, &cfg) != cudaSuccess || n < 1)
            n = (num_sms() > 0 ? num_sms() : 148) / 2;
        (void)cudaGetLastError();
        max_pairs = n;
    }
    const int pairs = p.tiles < max_pairs ? p.tiles : max_pairs;
    p.nsched = 0;
    if (takes_schedule(p.tiles, pairs, a.nseg, BN)) {
        const SchedVal *sv =
            tile_schedule(SchedKey{p.tiles, p.nmat * p.n_tiles, p.n_tiles, p.nseg, BN, pairs});
        memcpy(p.first, sv->first.data(), sv->first.size() * sizeof(uint16_t));
        memcpy(p.sched, sv->tile.data(), sv->tile.size() * sizeof(uint16_t));
        p.nsched = p.tiles;
    }
    return launch_pdl(gemm_tc2_kernel<BN, STAGES, STAGING, SCH>, dim3(2 * pairs), dim3(kThreads), L::ALLOC, s,
                      mA, mB[0], mB[1], mB[2], mo, p);
}

}  // namespace

bool gemm_tc2_supported(const GemmArgs &a) {
    if (a.dtype != DT_BF16 || a.nmat < 1 || a.nmat > 3) return false;
    // rows past the end (a matrix shorter than a tile) read as zeros through the
    // tensor map and are never written
    // K: whole 16-byte rows for the tensor maps (a last partial K block reads
    // zeros); nseg: tile widths N with N % 16 == 0 (N / 2 weight rows per CTA)
    if (a.K < 8 || a.K % 8 || a.rows < 1 || a.lda % 8 || a.ldc % 8) return false;
    if (a.nseg < 16 || a.nseg % 16) return false;
    if ((uintptr_t)a.A % 16) return false;
    for (int i = 0; i < a.nmat; ++i) {
        if ((uintptr_t)a.W[i] % 16 || (uintptr_t)a.C[i] % 16 || (uintptr_t)a.R[i] % 16 ||
            (uintptr_t)a.bias[i] % 16)
            return false;
        // tiled head layout: whole 8-column units per head, no residual, bias or activation
        if (a.thl[i] && (a.R[i] || a.bias[i] || a.act != ACT_NONE || a.d < 8 || a.d % 8 ||
                         a.heads * a.d != a.nseg))
            return false;
    }
    return true;
}

int gemm_tc2_schedule(long rows, int nseg, int nmat, int pairs, int32_t *first, int32_t *tile,
                      int *tiles, int *scheduled) {
    constexpr int BN = 256;  // the tile width both launch variants use
    if (rows < 1 || nseg < 16 || nseg % 16 || nmat < 1 || nmat > 3 || pairs < 1) return -1;
    const long n_tiles = (nseg + BN - 1) / BN;
    const long all = (rows + 2 * BMC - 1) / (2 * BMC) * nmat * n_tiles;
    if (all > (1L << 30)) return -1;
    *tiles = static_cast<int>(all);
    *scheduled = takes_schedule(*tiles, pairs, nseg, BN) ? 1 : 0;
    if (!*scheduled || !first || !tile) return 0;
    const SchedVal *sv = tile_schedule(
        SchedKey{*tiles, nmat * static_cast<int>(n_tiles), static_cast<int>(n_tiles), nseg, BN, pairs});
    for (size_t i = 0; i < sv->first.size(); ++i) first[i] = sv->first[i];
    for (size_t i = 0; i < sv->tile.size(); ++i) tile[i] = sv->tile[i];
    return 0;
}

cudaError_t launch_gemm_tc2(const GemmArgs &a, cudaStream_t s) {
    bool all_tiled = true;
    for (int i = 0; i < a.nmat; ++i) all_tiled = all_tiled && a.thl[i] != nullptr;
    // outputs in tiled head layout need no staging tiles: two more pipeline stages
    if (all_tiled) return launch_bn2<256, 7, false, 8>(a, s);
    // row-major outputs: half a tile's columns staged per pass leaves room for a
    // sixth pipeline stage (O projections 1246 -> 1270 TFLOP/s on the long video)
    return launch_bn2<256, 6, true, 4>(a, s);
}

}  // namespace ptdit
