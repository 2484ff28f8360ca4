// Weight gradients of the projections: dW_i = G_i^T X_i, a reduction over the
// token rows (backward of y = x W^T: dL/dW = (dL/dy)^T x).
//
// G_i is a column block of a row-major [rows, ldg] gradient buffer and X_i a
// row-major [rows, ldx] activation; dW_i is fp32 [M][N] row-major.  Both MMA
// operands are MN-major: a TMA box of 64 token rows x 64 columns lands in
// shared memory as eight 8-row x 128-byte atoms (128-byte swizzle), which is
// the MN-major operand layout of tcgen05.mma with the reduction (token) index
// as K.  One CTA per SM computes a 128 x 256 tile of one dW_i over one slice of
// the token rows (split-K, so that the few output tiles still fill every SM)
// and adds it into dW_i with 16-byte vector reductions (red.global.add.v4.f32);
// the caller zeroes dW first.
//
//   warp 0     producer: per stage two 64 x 64 boxes of G_i and four of X_i
//              (rows past the end read as zeros; so do X columns past N)
//   warp 1     MMA issuer: four 128 x N x 16 MMAs per stage (N = the tile's
//              width, 256 or the 128 left at the edge) into one of two TMEM
//              accumulators, so the next item's MMAs overlap this epilogue
//   warps 2-5  epilogue: each warp owns 32 rows of the accumulator and reduces
//              them into dW_i, 32 columns per TMEM load
// Every wait is bounded (2 s).
#include "tc_util.cuh"

namespace ptdit {
namespace {

using namespace tc;

constexpr int WM = 128, WN = 256, WK = 64;  // output rows, output columns, token rows per stage
constexpr int WSTAGES = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int BOX = 64 * 64 * 2;  // one 64 x 64 bf16 box: 8 KB

struct WgLayout {
    static constexpr int A_BYTES = 2 * BOX;  // 128 columns of G_i
    static constexpr int B_BYTES = 4 * BOX;  // 256 columns of X_i
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int OFF_BAR = WSTAGES * STAGE;
    static constexpr int NBARS = 2 * WSTAGES + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr int BYTES = OFF_BAR + NBARS * 8 + 16 + 1024;
    static_assert(BYTES <= 232448, "shared memory budget");
};

struct WgParams {
    float *dw[kWgradMax];  // outputs [m][n]
    int gsrc[kWgradMax];   // which (G, X) map pair matrix i reads
    int gcol[kWgradMax];   // first column of G_i in its buffer
    int nmat, M, N, rows;
    int m_tiles, n_tiles, splits, kblocks, items;
    int *status;
};

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// Item t: split, then matrix, then output tile (n fastest): the splits of one
// tile run on different CTAs at about the same time.
struct Item {
    int mat, m0, n0, width, kb0, kb1;
};
__device__ __forceinline__ Item decode_item(const WgParams &p, int t) {
    Item it;
    const int tiles = p.m_tiles * p.n_tiles;
    const int per_split = p.nmat * tiles;
    const int sp = t / per_split;
    const int r = t % per_split;
    it.mat = r / tiles;
    const int tile = r % tiles;
    it.m0 = (tile / p.n_tiles) * WM;
    it.n0 = (tile % p.n_tiles) * WN;
    it.width = min(WN, p.N - it.n0);
    it.kb0 = (int)((long)sp * p.kblocks / p.splits);
    it.kb1 = (int)((long)(sp + 1) * p.kblocks / p.splits);
    return it;
}

__global__ void __launch_bounds__(kThreads, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap mG0, const __grid_constant__ CUtensorMap mG1,
                 const __grid_constant__ CUtensorMap mX0, const __grid_constant__ CUtensorMap mX1,
                 const __grid_constant__ WgParams p) {
    using L = WgLayout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *empty = full + WSTAGES, *tfull = empty + WSTAGES, *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tslot + 1);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < WSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);  // one arrive per epilogue warp
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
    pdl_wait();  // the kernels that wrote G and X have completed
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&mG0);
            prefetch_tensormap(&mX0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.items; t += gridDim.x) {
                const Item it = decode_item(p, t);
                const int src = p.gsrc[it.mat];
                const CUtensorMap *mg = src ? &mG1 : &mG0;
                const CUtensorMap *mx = src ? &mX1 : &mX0;
                const int gx = p.gcol[it.mat] + it.m0;
                for (int kb = it.kb0; kb < it.kb1; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort, p.status)) { ok = false; break; }
                    uint8_t *sa = sm + stage * L::STAGE, *sb = sa + L::A_BYTES;
                    mbar_expect_tx(&full[stage], L::STAGE);
                    const int y = kb * WK;
                    tma_load_2d(sa, mg, &full[stage], gx, y);
                    tma_load_2d(sa + BOX, mg, &full[stage], gx + 64, y);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        tma_load_2d(sb + c * BOX, mx, &full[stage], it.n0 + 64 * c, y);
                    if (++stage == WSTAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs the loop with warp-uniform operands; lane 0 issues)
        {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, any = false;
            for (int t = blockIdx.x; ok && t < p.items; t += gridDim.x) {
                const Item it = decode_item(p, t);
                const uint32_t idesc = idesc_bf16(WM, it.width, true, true);
                if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1, abort, p.status)) break;
                fence_after_sync();
                const uint32_t d = tmem + acc * WN;
                for (int kb = it.kb0; kb < it.kb1; ++kb) {
                    if (!mbar_wait_warp(&full[stage], phase, abort, p.status)) { ok = false; break; }
                    fence_after_sync();
                    const uint32_t sa = smem_u32(sm + stage * L::STAGE), sb = sa + L::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < WK / 16; ++kk)
                        warp_mma_bf16(d, sdesc_sw128_mn(sa + kk * 2048, BOX),
                                 sdesc_sw128_mn(sb + kk * 2048, BOX), idesc, (kb > it.kb0) | kk);
                    any = true;
                    warp_mma_commit(&empty[stage]);
                    if (++stage == WSTAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                warp_mma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (any) {  // every issued MMA has finished before TMEM is released
                warp_mma_commit(drain);
                volatile int never = 0;
                mbar_wait_warp(drain, 0, &never, p.status);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp % 4;  // TMEM lanes 32q .. 32q + 31
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < p.items; t += gridDim.x) {
            const Item it = decode_item(p, t);
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort, p.status))) break;
            fence_after_sync();
            const uint32_t tb = tmem + acc * WN + (static_cast<uint32_t>(q * 32) << 16);
            float *row = p.dw[it.mat] + (long)(it.m0 + q * 32 + lane) * p.N + it.n0;
            // an empty slice (more splits than token blocks) left the accumulator unwritten
            const bool has = it.kb1 > it.kb0;
#pragma unroll 1
            for (int c = 0; c < it.width; c += 32) {
                uint32_t v[32];
                tmem_ld32(tb + c, v);
                tmem_ld_wait();
                if (has)
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        red_add_v4(row + c + j, __uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                   __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            }
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool wgrad_supported(const WgradArgs &a) {
    if (a.nmat < 1 || a.nmat > kWgradMax || a.rows < 1) return false;
    if (a.M % WM || a.N % 64 || a.N < 64) return false;  // whole 128-row tiles; 64-column boxes
    for (int i = 0; i < 2; ++i)
        if (a.G[i] && (a.ldg[i] % 8 || a.ldx[i] % 8)) return false;  // 16-byte row strides
    for (int i = 0; i < a.nmat; ++i) {
        const int s = a.src[i];
        if (s < 0 || s > 1 || !a.G[s] || !a.X[s] || !a.dW[i]) return false;
        if (a.gcol[i] < 0 || a.gcol[i] + a.M > a.ldg[s] || a.N > a.ldx[s]) return false;
    }
    return true;
}

cudaError_t launch_wgrad(const WgradArgs &a, cudaStream_t s) {
    using L = WgLayout;
    if (!wgrad_supported(a)) return cudaErrorInvalidValue;
    CUtensorMap mG[2], mX[2];
    for (int i = 0; i < 2; ++i) {
        const int j = a.G[i] ? i : 0;  // an unused pair repeats pair 0
        if (!encode_map_2d_bf16(&mG[i], a.G[j], a.ldg[j], a.rows, (uint64_t)a.ldg[j] * 2, 64, 64) ||
            !encode_map_2d_bf16(&mX[i], a.X[j], a.N, a.rows, (uint64_t)a.ldx[j] * 2, 64, 64))
            return cudaErrorNotSupported;
    }
    WgParams p;
    memset(&p, 0, sizeof p);
    for (int i = 0; i < a.nmat; ++i) {
        p.dw[i] = a.dW[i];
        p.gsrc[i] = a.src[i];
        p.gcol[i] = a.gcol[i];
    }
    p.nmat = a.nmat;
    p.M = a.M;
    p.N = a.N;
    p.rows = a.rows;
    p.m_tiles = a.M / WM;
    p.n_tiles = (a.N + WN - 1) / WN;
    p.kblocks = (a.rows + WK - 1) / WK;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int tiles = a.nmat * p.m_tiles * p.n_tiles;
    // enough slices for about four items per SM, each of at least 8 token blocks
    int splits = (4 * sms + tiles - 1) / tiles;
    splits = min(splits, max(1, p.kblocks / 8));
    p.splits = max(1, splits);
    p.items = tiles * p.splits;
    p.status = device_status_ptr();
    if (!p.status) return cudaErrorInvalidValue;
    cudaError_t e =
        cudaFuncSetAttribute(wgrad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return e;
    const int grid = p.items < sms ? p.items : sms;
    return launch_pdl(wgrad_kernel, dim3(grid), dim3(kThreads), L::BYTES, s, mG[0], mG[1], mX[0],
                      mX[1], p);
}

}  // namespace ptdit
