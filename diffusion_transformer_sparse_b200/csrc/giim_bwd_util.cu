// Element-wise steps of GIIM's backward pass (the attention and projection work
// runs on the tensor-core kernels):
//   row_delta        delta[b][h][q] = sum over the head's columns of dO * O, the
//                    rowsum(P * dP) of the softmax backward (it equals dO . O);
//                    dO in tiled head layout, O row-major
//   proxy_broadcast  the averaging's adjoint: every token of proxy window m
//                    receives dP_a[m] / P, added to the residual's dL/dout
//   to_bf16          the fp32 key and value gradients to bf16 operands
//   key_mean         per (batch item, head) the mean of the valid key rows (fp32),
//                    read from the tiled head layout
//   center_keys      the key rows less that mean, in place (the backward then
//                    takes dQ = c dS (K - mean), which is exact: every row of dS
//                    sums to zero)
//   sum_blocks       dQ summed over the key tiles: dst = sum over j of the column
//                    blocks [j D, (j + 1) D) of src (bf16, fp32 sums)
//   center_to_bf16   the fp32 key gradient less its mean over each batch item's keys,
//                    as bf16 (the projection of the softmax backward onto its
//                    exact constraint: every row of dS sums to zero, so the exact
//                    key gradient of every head sums to zero over the keys)
#include "thl.cuh"

namespace ptdit {
namespace {

// One thread per (row, head): dO in tiled head layout (identity tiles, no padding),
// O row-major with row stride ld; the head's d columns as 16-byte pieces.
__global__ void row_delta_kernel(const uint8_t *__restrict__ dO, const __nv_bfloat16 *__restrict__ O,
                                 int B, int nq, int heads, int d, long ld, float *__restrict__ delta) {
    pdl_wait();
    pdl_trigger();
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)B * nq * heads) return;
    const long row = idx / heads;
    const int h = static_cast<int>(idx - row * heads);
    const long b = row / nq;
    const int q = static_cast<int>(row - b * nq);
    const int tiles = (nq + kThlRows - 1) / kThlRows, tile = q / kThlRows, tr = q % kThlRows;
    const uint8_t *blk = dO + (((long)b * tiles + tile) * heads + h) * (long)thl_block_bytes(d, 0);
    const __nv_bfloat16 *o = O + row * ld + (long)h * d;
    float s = 0.f;
    for (int u = 0; u < d / 8; ++u) {
        const uint4 va = *reinterpret_cast<const uint4 *>(blk + thl_unit(tr, u, 0));
        const uint4 vo = *reinterpret_cast<const uint4 *>(o + 8 * u);
        const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wo[4] = {vo.x, vo.y, vo.z, vo.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wa[t]));
            const float2 fo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wo[t]));
            s = fmaf(fa.x, fo.x, fmaf(fa.y, fo.y, s));
        }
    }
    delta[(b * heads + h) * nq + q] = s;
}

// One warp per token row: dz = (dout +) dPa[proxy of the token] / P, the proxy index
// computed once per row, the lanes on consecutive 16-byte pieces.
__global__ void proxy_broadcast_kernel(ProxyGeom g, int B, int D, const __nv_bfloat16 *__restrict__ dPa,
                                       const __nv_bfloat16 *__restrict__ dout,
                                       __nv_bfloat16 *__restrict__ dz) {
    pdl_wait();
    pdl_trigger();
    const int pieces = D / 8, lane = threadIdx.x % 32;
    const long N = (long)g.f * g.h * g.w;
    const long tok = ((long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    if (tok >= (long)B * N) return;
    const long b = tok / N;
    const int m = proxy_of_token(g, static_cast<int>(tok - b * N));
    const float inv = 1.f / static_cast<float>(g.P);
    const __nv_bfloat16 *prow = dPa + ((long)b * g.M + m) * D;
    const __nv_bfloat16 *rrow = dout ? dout + tok * D : nullptr;
    __nv_bfloat16 *orow = dz + tok * D;
    for (int pc = lane; pc < pieces; pc += 32) {
        const uint4 vp = *reinterpret_cast<const uint4 *>(prow + 8 * pc);
        uint4 vr = make_uint4(0, 0, 0, 0);
        if (rrow) vr = *reinterpret_cast<const uint4 *>(rrow + 8 * pc);
        const uint32_t wp[4] = {vp.x, vp.y, vp.z, vp.w}, wr[4] = {vr.x, vr.y, vr.z, vr.w};
        uint32_t o[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float2 fp = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wp[t]));
            const float2 fr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wr[t]));
            const __nv_bfloat162 v = __floats2bfloat162_rn(fmaf(fp.x, inv, fr.x), fmaf(fp.y, inv, fr.y));
            o[t] = *reinterpret_cast<const uint32_t *>(&v);
        }
        *reinterpret_cast<uint4 *>(orow + 8 * pc) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__global__ void to_bf16_kernel(const float *__restrict__ src, long rows, int cols,
                               __nv_bfloat16 *__restrict__ dst, long ldd) {
    pdl_wait();
    pdl_trigger();
    const long idx = ((long)blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (idx >= rows * cols) return;
    const long r = idx / cols;
    const int c = static_cast<int>(idx - r * cols);
    const float4 a = *reinterpret_cast<const float4 *>(src + idx);
    const float4 b = *reinterpret_cast<const float4 *>(src + idx + 4);
    __nv_bfloat162 o[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                           __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
    *reinterpret_cast<uint4 *>(dst + r * ldd + c) = *reinterpret_cast<const uint4 *>(o);
}

// One thread per 8 columns of one row: the nblk blocks' 16-byte pieces summed in fp32.
__global__ void sum_blocks_kernel(const __nv_bfloat16 *__restrict__ src, long rows, int nblk,
                                  int D, long lds, __nv_bfloat16 *__restrict__ dst, long ldd) {
    pdl_wait();
    pdl_trigger();
    const int pieces = D / 8;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= rows * pieces) return;
    const long r = idx / pieces;
    const int c = static_cast<int>(idx - r * pieces) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const __nv_bfloat16 *p = src + r * lds + c;
    for (int j = 0; j < nblk; ++j) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p + (long)j * D);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[t]));
            acc[2 * t] += f.x;
            acc[2 * t + 1] += f.y;
        }
    }
    __nv_bfloat162 o[4] = {__floats2bfloat162_rn(acc[0], acc[1]), __floats2bfloat162_rn(acc[2], acc[3]),
                           __floats2bfloat162_rn(acc[4], acc[5]), __floats2bfloat162_rn(acc[6], acc[7])};
    *reinterpret_cast<uint4 *>(dst + r * ldd + c) = *reinterpret_cast<const uint4 *>(o);
}

// One CTA per (batch item, head): thread (row lane, 16-byte unit) sums its unit over
// the rows of its lane; the lanes meet in shared memory.
__global__ void key_mean_kernel(const uint8_t *__restrict__ K, int nk, int heads, int d,
                                float *__restrict__ mean) {
    pdl_wait();
    pdl_trigger();
    constexpr int kLanes = 16;
    __shared__ float part[kLanes][80];
    const int bh = blockIdx.x, b = bh / heads, h = bh - b * heads;
    const int u = threadIdx.x % 16, lane = threadIdx.x / 16;
    const int tiles = (nk + kThlRows - 1) / kThlRows;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (u < d / 8) {
        for (int k = lane; k < nk; k += kLanes) {
            const int tile = k / kThlRows, tr = k % kThlRows;
            const uint8_t *blk = K + (((long)b * tiles + tile) * heads + h) * (long)thl_block_bytes(d, 0);
            const uint4 v = *reinterpret_cast<const uint4 *>(blk + thl_unit(tr, u, 0));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[t]));
                acc[2 * t] += f.x;
                acc[2 * t + 1] += f.y;
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) part[lane][8 * u + e] = acc[e];
    }
    __syncthreads();
    if (threadIdx.x < d) {
        float s = 0.f;
        for (int l = 0; l < kLanes; ++l) s += part[l][threadIdx.x];
        mean[(long)b * heads * d + (long)h * d + threadIdx.x] = s / static_cast<float>(nk);
    }
}

// One thread per (batch item, key row, head, 16-byte unit) of the valid rows.
__global__ void center_keys_kernel(uint8_t *__restrict__ K, int B, int nk, int heads, int d,
                                   const float *__restrict__ mean) {
    pdl_wait();
    pdl_trigger();
    const int units = d / 8;
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long)B * nk * heads * units) return;
    const int u = static_cast<int>(idx % units);
    long rest = idx / units;
    const int h = static_cast<int>(rest % heads);
    rest /= heads;
    const int k = static_cast<int>(rest % nk);
    const long b = rest / nk;
    const int tiles = (nk + kThlRows - 1) / kThlRows, tile = k / kThlRows, tr = k % kThlRows;
    uint4 *p = reinterpret_cast<uint4 *>(K + ((b * tiles + tile) * heads + h) * (long)thl_block_bytes(d, 0) +
                                         thl_unit(tr, u, 0));
    const float *m = mean + b * heads * d + (long)h * d + 8 * u;
    const uint4 v = *p;
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[t]));
        const __nv_bfloat162 o = __floats2bfloat162_rn(f.x - m[2 * t], f.y - m[2 * t + 1]);
        w[t] = *reinterpret_cast<const uint32_t *>(&o);
    }
    *p = make_uint4(w[0], w[1], w[2], w[3]);
}

// One CTA per (batch item, 32 columns): lane = column, the 8 warps stride over the
// item's M rows, first for the column sums, then for the centred bf16 values.
__global__ void center_to_bf16_kernel(const float *__restrict__ src, int M, int cols,
                                      __nv_bfloat16 *__restrict__ dst, long ldd) {
    pdl_wait();
    pdl_trigger();
    __shared__ float part[8][32];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const long b = blockIdx.x;
    const int c = blockIdx.y * 32 + lane;
    const float *s0 = src + b * M * cols;
    float acc = 0.f;
    if (c < cols)
        for (int r = warp; r < M; r += 8) acc += s0[(long)r * cols + c];
    part[warp][lane] = acc;
    __syncthreads();
    float m = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) m += part[w][lane];
    m /= static_cast<float>(M);
    if (c < cols)
        for (int r = warp; r < M; r += 8)
            dst[(b * M + r) * ldd + c] = __float2bfloat16_rn(s0[(long)r * cols + c] - m);
}

}  // namespace

cudaError_t launch_sum_blocks_bf16(const void *src, long rows, int nblk, int D, long lds,
                                  void *dst, long ldd, cudaStream_t s) {
    if (rows < 1 || nblk < 1 || D % 8 || lds % 8 || ldd % 8) return cudaErrorInvalidValue;
    const long n = rows * (D / 8);
    const int threads = 256;
    return launch_pdl(sum_blocks_kernel, dim3((unsigned)((n + threads - 1) / threads)),
                      dim3(threads), 0, s, static_cast<const __nv_bfloat16 *>(src), rows, nblk, D,
                      lds, static_cast<__nv_bfloat16 *>(dst), ldd);
}

cudaError_t launch_key_mean(const void *K_tiles, int B, int nk, int heads, int d, float *mean,
                            cudaStream_t s) {
    if (B < 1 || nk < 1 || d < 8 || d % 8 || d > 80) return cudaErrorInvalidValue;
    return launch_pdl(key_mean_kernel, dim3((unsigned)(B * heads)), dim3(256), 0, s,
                      static_cast<const uint8_t *>(K_tiles), nk, heads, d, mean);
}

cudaError_t launch_center_keys(void *K_tiles, int B, int nk, int heads, int d, const float *mean,
                               cudaStream_t s) {
    if (B < 1 || nk < 1 || d < 8 || d % 8 || d > 80) return cudaErrorInvalidValue;
    const long n = (long)B * nk * heads * (d / 8);
    const int threads = 256;
    return launch_pdl(center_keys_kernel, dim3((unsigned)((n + threads - 1) / threads)),
                      dim3(threads), 0, s, static_cast<uint8_t *>(K_tiles), B, nk, heads, d, mean);
}

cudaError_t launch_center_to_bf16(const float *src, int B, int M, int cols, void *dst, long ldd,
                                  cudaStream_t s) {
    if (B < 1 || M < 1 || cols < 1) return cudaErrorInvalidValue;
    return launch_pdl(center_to_bf16_kernel, dim3((unsigned)B, (unsigned)((cols + 31) / 32)),
                      dim3(256), 0, s, src, M, cols, static_cast<__nv_bfloat16 *>(dst), ldd);
}

cudaError_t launch_to_bf16(const float *src, long rows, int cols, void *dst, long ldd,
                           cudaStream_t s) {
    if (rows < 1 || cols % 8 || ldd % 8) return cudaErrorInvalidValue;
    const long n = rows * cols / 8;
    const int threads = 256;
    return launch_pdl(to_bf16_kernel, dim3((unsigned)((n + threads - 1) / threads)), dim3(threads),
                      0, s, src, rows, cols, static_cast<__nv_bfloat16 *>(dst), ldd);
}

cudaError_t launch_row_delta(const void *dO_tiles, const void *O, int B, int nq, int heads,
                             int d, long ld, float *delta, cudaStream_t s) {
    if (B < 1 || nq < 1 || d % 8 || d > 80 || ld % 8) return cudaErrorInvalidValue;
    const long n = (long)B * nq * heads;
    const int threads = 256;
    return launch_pdl(row_delta_kernel, dim3((unsigned)((n + threads - 1) / threads)),
                      dim3(threads), 0, s, static_cast<const uint8_t *>(dO_tiles),
                      static_cast<const __nv_bfloat16 *>(O), B, nq, heads, d, ld, delta);
}

cudaError_t launch_proxy_broadcast(const ProxyGeom &g, int B, int D, const void *dPa,
                                   const void *dout, void *dz, cudaStream_t s) {
    if (D % 8) return cudaErrorInvalidValue;
    const long n = (long)B * g.f * g.h * g.w * 32;  // one warp per token
    const int threads = 256;
    return launch_pdl(proxy_broadcast_kernel, dim3((unsigned)((n + threads - 1) / threads)),
                      dim3(threads), 0, s, g, B, D, static_cast<const __nv_bfloat16 *>(dPa),
                      static_cast<const __nv_bfloat16 *>(dout), static_cast<__nv_bfloat16 *>(dz));
}

}  // namespace ptdit
