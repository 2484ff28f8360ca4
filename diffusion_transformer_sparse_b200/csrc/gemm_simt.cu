// Projections y = x W^T on the CUDA cores (FFMA): the fp32 path, and any
// shape the tensor-core GEMM does not take.
//
// 64 x 64 output tile per CTA, K staged 16 at a time through shared memory,
// 4 x 4 outputs per thread, fp32 accumulation in ascending k.  blockIdx.z picks
// one of up to three weight matrices (the fused Q/K/V projection writes three
// outputs).  The epilogue adds the residual in fp32 and rounds once.
#include "common.cuh"

namespace ptdit {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs a) {
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    const int s = blockIdx.z;
    const T *__restrict__ A = static_cast<const T *>(a.A);
    const T *__restrict__ W = static_cast<const T *>(a.W[s]);
    T *C = static_cast<T *>(a.C[s]);
    const T *R = static_cast<const T *>(a.R[s]);
    const T *bias = static_cast<const T *>(a.bias[s]);
    const int row0 = blockIdx.y * BM, col0 = blockIdx.x * BN;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int lr = tid / 4, lk = (tid % 4) * 4;  // loader: row (or weight row), 4 consecutive k

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < a.K; k0 += BK) {
        const int gr = row0 + lr, gc = col0 + lr;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int k = k0 + lk + u;
            As[lk + u][lr] = (gr < a.rows && k < a.K) ? to_f32(A[(long)gr * a.lda + k]) : 0.f;
            Bs[lk + u][lr] = (gc < a.nseg && k < a.K) ? to_f32(W[(long)gc * a.K + k]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty * 4 + i;
        if (r >= a.rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = col0 + tx * 4 + j;
            if (c >= a.nseg) continue;
            float v = acc[i][j];
            if (bias) v += to_f32(bias[c]);
            if (a.act == ACT_GELU_TANH) v = gelu_tanh_exact(v);
            if (R) v += to_f32(R[(long)r * a.ldc + c]);
            C[(long)r * a.ldc + c] = from_f32<T>(v);
        }
    }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmArgs &a, cudaStream_t s) {
    dim3 grid((a.nseg + BN - 1) / BN, (a.rows + BM - 1) / BM, a.nmat);
    if (a.dtype == DT_BF16)
        gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
    else
        gemm_simt_kernel<float><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ptdit
