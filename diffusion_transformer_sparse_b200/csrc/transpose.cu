// Transposes of the projection weights for the backward pass (dL/dx = dL/dy W
// is the projection kernel's x W'^T with W' = W^T): dst[c][r] = src[r][c],
// through a 32 x 33 shared-memory tile so that both the reads and the writes
// are coalesced.
#include "common.cuh"

namespace ptdit {
namespace {

__global__ void transpose_bf16_kernel(const __nv_bfloat16 *__restrict__ src, int rows, int cols,
                                      __nv_bfloat16 *__restrict__ dst, long ldd) {
    __shared__ __nv_bfloat16 t[32][33];
    pdl_wait();
    pdl_trigger();
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) t[i][threadIdx.x] = src[(long)r * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (c < cols && r < rows) dst[(long)c * ldd + r] = t[threadIdx.x][i];
    }
}

}  // namespace

cudaError_t launch_transpose_bf16(const void *src, int rows, int cols, void *dst, long ldd,
                                  cudaStream_t s) {
    if (rows < 1 || cols < 1 || ldd < rows) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)((cols + 31) / 32), (unsigned)((rows + 31) / 32));
    return launch_pdl(transpose_bf16_kernel, grid, dim3(32, 8), 0, s,
                      static_cast<const __nv_bfloat16 *>(src), rows, cols,
                      static_cast<__nv_bfloat16 *>(dst), ldd);
}

}  // namespace ptdit
