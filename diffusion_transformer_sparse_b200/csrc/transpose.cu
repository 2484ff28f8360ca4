// Transposes of the projection weights for the backward pass (dL/dx = dL/dy W
// is the projection kernel's x W'^T with W' = W^T): dst[c][r] = src[r][c] for a
// batch of matrices in one launch (grid z = matrix).  A CTA moves a 64 x 64 tile
// through shared memory: 16-byte loads along the source rows, 16-byte stores
// along the destination rows (8 source rows of one column gathered from shared
// memory per store).
#include "common.cuh"

namespace ptdit {
namespace {

constexpr int kT = 64;         // tile side
constexpr int kPitch = kT + 8;  // shared-memory row pitch in elements (144 B: 16-byte aligned)

__global__ void __launch_bounds__(256) transpose_batch_kernel(TransposeBatch jb) {
    __shared__ __align__(16) __nv_bfloat16 t[kT][kPitch];
    pdl_wait();
    pdl_trigger();
    const TransposeJob &j = jb.job[blockIdx.z];
    const int c0 = blockIdx.x * kT, r0 = blockIdx.y * kT;
    if (c0 >= j.cols || r0 >= j.rows) return;  // this matrix is smaller than the grid
    const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(j.src);
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(j.dst);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = threadIdx.x + 256 * h;
        const int rr = i / 8, ch = i % 8;  // tile row, 8-column piece
        const int r = r0 + rr, c = c0 + 8 * ch;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < j.rows && c < j.cols) v = *reinterpret_cast<const uint4 *>(src + (long)r * j.cols + c);
        *reinterpret_cast<uint4 *>(&t[rr][8 * ch]) = v;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = threadIdx.x + 256 * h;
        const int cc = i / 8, k = i % 8;  // destination row (source column), 8-row piece
        const int c = c0 + cc, r = r0 + 8 * k;
        if (c >= j.cols || r >= j.rows) continue;
        __align__(16) __nv_bfloat16 o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = t[8 * k + e][cc];
        *reinterpret_cast<uint4 *>(dst + (long)c * j.ldd + r) = *reinterpret_cast<const uint4 *>(o);
    }
}

}  // namespace

cudaError_t launch_transpose_batch_bf16(const TransposeBatch &jb, cudaStream_t s) {
    if (jb.n < 1 || jb.n > kTransposeMax) return cudaErrorInvalidValue;
    int mr = 0, mc = 0;
    for (int i = 0; i < jb.n; ++i) {
        const TransposeJob &j = jb.job[i];
        // 16-byte pieces: every row and column count, stride and base a multiple of 8
        if (j.rows < 1 || j.cols < 1 || j.ldd < j.rows || j.rows % 8 || j.cols % 8 || j.ldd % 8 ||
            reinterpret_cast<uintptr_t>(j.src) % 16 || reinterpret_cast<uintptr_t>(j.dst) % 16)
            return cudaErrorInvalidValue;
        mr = mr > j.rows ? mr : j.rows;
        mc = mc > j.cols ? mc : j.cols;
    }
    const dim3 grid((unsigned)((mc + kT - 1) / kT), (unsigned)((mr + kT - 1) / kT), (unsigned)jb.n);
    return launch_pdl(transpose_batch_kernel, grid, dim3(256), 0, s, jb);
}

}  // namespace ptdit
