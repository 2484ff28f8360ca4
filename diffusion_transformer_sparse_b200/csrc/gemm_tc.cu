// Projections y = x W^T (+ residual) on the 5th-generation tensor cores.
//
// Every QKV and O projection of the PT-Block attention path (proxy SA,
// cross-attention, WSA, SWSA) is this kernel: bf16 operands, fp32 accumulation
// in tensor memory, one rounding to bf16 in the epilogue (after the residual
// add, in fp32).
//
// Design (one persistent CTA per SM, 6 warps, warp-specialised):
//   warp 0  TMA producer: 128 x 64 A tile and BN x 64 weight tile per stage,
//           128-byte swizzle, STAGES-deep ring of shared-memory buffers.
//   warp 1  MMA issuer: 4 x tcgen05.mma (K = 16 each) per stage into a TMEM
//           accumulator of 128 lanes x BN fp32 columns; tcgen05.commit frees
//           the stage and, after the last K block, hands the tile to the
//           epilogue.  Two accumulators let the next tile's MMAs overlap the
//           previous tile's epilogue.
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time (one row per thread),
//           + residual, round, 16-byte stores.
// Output tiles run n-fastest so concurrently resident CTAs share A rows in L2.
// Up to three weight matrices (a fused Q/K/V projection) are one launch.
// Every mbarrier wait is bounded (2 s): on expiry the kernel records
// PTDIT_ERR_TIMEOUT in the library's status word and winds down.
#include "tc_util.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int BM = 128, BK = 64;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

struct TcParams {
    void *C[3];
    const void *R[3];
    long ldc;
    int rows, nseg, nmat;
    int n_tiles;  // output tiles per weight matrix
    int tiles;    // all output tiles
    int kblocks;
    int *status;
};

template <int BN, int STAGES>
struct Layout {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    static constexpr int NBARS = 2 * STAGES + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr int BYTES = BAR_OFF + NBARS * 8 + 16;
    static constexpr int ALLOC = BYTES + 1024;  // slack to align the base to 1024 B
    static constexpr uint32_t ACC_STRIDE = BN <= 128 ? 128 : 256;
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "stage tiles must stay 1 KB aligned");
    static_assert(2 * ACC_STRIDE <= kTmemCols, "two accumulators must fit in TMEM");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

__device__ __forceinline__ void decode_tile(const TcParams &p, int t, int &m_tile, int &seg,
                                            int &n_tile) {
    const int per_m = p.nmat * p.n_tiles;
    m_tile = t / per_m;
    const int n = t % per_m;
    seg = n / p.n_tiles;
    n_tile = n % p.n_tiles;
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB0,
                   const __grid_constant__ CUtensorMap mB1,
                   const __grid_constant__ CUtensorMap mB2, TcParams p) {
    using L = Layout<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&mA);
            prefetch_tensormap(&mB0);
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
                int m_tile, seg, n_tile;
                decode_tile(p, t, m_tile, seg, n_tile);
                const CUtensorMap *mb = seg == 0 ? &mB0 : (seg == 1 ? &mB1 : &mB2);
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * L::STAGE_BYTES;
                    mbar_expect_tx(&full[stage], L::STAGE_BYTES);
                    tma_load_2d(sa, &mA, &full[stage], kb * BK, m_tile * BM);
                    tma_load_2d(sa + L::A_BYTES, mb, &full[stage], kb * BK, n_tile * BN);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (*abort) {
                // let the copies still in flight land before the CTA exits
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && i < issued; ++i) {
                    if (--s < 0) {
                        s = STAGES - 1;
                        ph ^= 1;
                    }
                    volatile int never = 0;
                    mbar_wait(&full[s], ph, &never, p.status);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, any = false;
            for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort, p.status)) break;
                fence_after_sync();
                const uint32_t d = tmem + acc * L::ACC_STRIDE;
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    const uint32_t sa = smem_u32(smem + stage * L::STAGE_BYTES);
                    const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_bf16(d, sdesc_sw128(sa + kk * 32), sdesc_sw128(sb + kk * 32), idesc,
                                 (kb | kk) != 0);
                    any = true;
                    mma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (any) {
                // every issued MMA has finished before TMEM is released
                mma_commit(drain);
                volatile int never = 0;
                mbar_wait(drain, 0, &never, p.status);
            }
        }
    } else {
        const int q = warp % 4;  // TMEM lanes 32q .. 32q+31 belong to this warp
        const int r_in_tile = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x) {
            int m_tile, seg, n_tile;
            decode_tile(p, t, m_tile, seg, n_tile);
            if (!mbar_wait(&tfull[acc], acc_phase, abort, p.status)) break;
            fence_after_sync();
            const long row = static_cast<long>(m_tile) * BM + r_in_tile;
            const bool live = row < p.rows;
            __nv_bfloat16 *C = static_cast<__nv_bfloat16 *>(p.C[seg]) + row * p.ldc + n_tile * BN;
            const __nv_bfloat16 *R = static_cast<const __nv_bfloat16 *>(p.R[seg]);
            if (R) R += row * p.ldc + n_tile * BN;
            const uint32_t tbase = tmem + acc * L::ACC_STRIDE + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tbase + c0, r);
                tmem_ld_wait();
                if (live) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                    if (R) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4 rv = *reinterpret_cast<const uint4 *>(R + c0 + 8 * j);
                            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&rv);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float2 f = __bfloat1622float2(h[e]);
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
                        *reinterpret_cast<uint4 *>(C + c0 + 8 * j) = o;
                    }
                }
            }
            fence_before_sync();
            mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int BN, int STAGES>
cudaError_t launch_bn(const GemmArgs &a, cudaStream_t s) {
    using L = Layout<BN, STAGES>;
    CUtensorMap mA, mB[3];
    if (!encode_map_2d_bf16(&mA, a.A, a.K, a.rows, a.lda * 2, BK, BM)) return cudaErrorInvalidValue;
    for (int i = 0; i < 3; ++i) {
        const void *w = i < a.nmat ? a.W[i] : a.W[0];
        if (!encode_map_2d_bf16(&mB[i], w, a.K, a.nseg, (uint64_t)a.K * 2, BK, BN))
            return cudaErrorInvalidValue;
    }
    TcParams p;
    for (int i = 0; i < 3; ++i) {
        p.C[i] = i < a.nmat ? a.C[i] : nullptr;
        p.R[i] = i < a.nmat ? a.R[i] : nullptr;
    }
    p.ldc = a.ldc;
    p.rows = a.rows;
    p.nseg = a.nseg;
    p.nmat = a.nmat;
    p.n_tiles = a.nseg / BN;
    p.kblocks = a.K / BK;
    const int m_tiles = (a.rows + BM - 1) / BM;
    p.tiles = m_tiles * a.nmat * p.n_tiles;
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorInvalidValue;
    const int sms = num_sms();
    const int grid = p.tiles < sms ? p.tiles : sms;
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, STAGES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<BN, STAGES><<<grid, kThreads, L::ALLOC, s>>>(mA, mB[0], mB[1], mB[2], p);
    return cudaGetLastError();
}

// Output-tile width: the candidate with the fewest tile-columns of work in
// its last wave (persistent grid of one CTA per SM).
int choose_bn(const GemmArgs &a) {
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int m_tiles = (a.rows + BM - 1) / BM;
    int best = 0;
    long best_cost = 0;
    for (int bn : {192, 128}) {
        if (a.nseg % bn) continue;
        const long tiles = (long)m_tiles * a.nmat * (a.nseg / bn);
        const long waves = (tiles + sms - 1) / sms;
        const long cost = waves * bn;
        if (!best || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

}  // namespace

bool gemm_tc_supported(const GemmArgs &a) {
    if (a.dtype != DT_BF16 || a.nmat < 1 || a.nmat > 3) return false;
    if (a.K < BK || a.K % BK || a.rows < BM || a.lda % 8 || a.ldc % 8) return false;
    if (choose_bn(a) == 0) return false;
    if ((uintptr_t)a.A % 16) return false;
    for (int i = 0; i < a.nmat; ++i)
        if ((uintptr_t)a.W[i] % 16 || (uintptr_t)a.C[i] % 16 || (uintptr_t)a.R[i] % 16)
            return false;
    return true;
}

cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s) {
    switch (choose_bn(a)) {
        case 192: return launch_bn<192, 5>(a, s);
        case 128: return launch_bn<128, 6>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ptdit
