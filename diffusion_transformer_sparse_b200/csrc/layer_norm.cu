// LayerNorm over the model width, the pre-norm of every sub-layer of the
// complete PT-Block (Qihoo-T2X reading note, §3 Method, the PT-Block diagram;
// code-comparison section, proxy_norm1 and norm_hidden_states):
//   y[r, :] = (x[r, :] - mean_r) / sqrt(var_r + eps) * gamma + beta,
// var_r the mean squared deviation of row r.
//
// An HBM stream: every element is read once and written once.  One warp per
// row; a row of up to 64 x 32 elements (bf16: 16-byte pieces, fp32: 16-byte
// pieces of 4) stays in registers between the mean, the variance (taken
// around the mean, not as E[x^2] - mean^2) and the output; statistics in
// fp32, one rounding of the output.  Wider or unaligned rows take the same
// arithmetic reading the row from memory three times.
#include "common.cuh"

namespace ptdit {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
struct Piece;  // 16 bytes of a row
template <>
struct Piece<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float *v) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, const float *v) {
        uint4 o;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        *reinterpret_cast<uint4 *>(p) = o;
    }
};
template <>
struct Piece<float> {
    static constexpr int E = 4;
    __device__ __forceinline__ static void load(const float *p, float *v) {
        const float4 f = *reinterpret_cast<const float4 *>(p);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
    __device__ __forceinline__ static void store(float *p, const float *v) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};

// Rows whose 16-byte pieces (D / E of them) fit MAXP per lane.
template <typename T, int MAXP>
__global__ void __launch_bounds__(256) layer_norm_kernel(const T *__restrict__ x,
                                                         const T *__restrict__ gamma,
                                                         const T *__restrict__ beta,
                                                         T *__restrict__ y, long rows, int D,
                                                         float eps) {
    pdl_wait();
    pdl_trigger();
    constexpr int E = Piece<T>::E;
    const long row = (long)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int np = D / E;
    const T *xr = x + row * D;
    float v[MAXP][E];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < MAXP; ++j) {
        const int p = lane + 32 * j;
        if (p < np) {
            Piece<T>::load(xr + p * E, v[j]);
#pragma unroll
            for (int e = 0; e < E; ++e) s += v[j][e];
        }
    }
    const float mean = warp_sum(s) / (float)D;
    float q = 0.f;
#pragma unroll
    for (int j = 0; j < MAXP; ++j) {
        const int p = lane + 32 * j;
        if (p < np) {
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float c = v[j][e] - mean;
                q = fmaf(c, c, q);
            }
        }
    }
    const float rstd = rsqrtf(warp_sum(q) / (float)D + eps);
    T *yr = y + row * D;
#pragma unroll
    for (int j = 0; j < MAXP; ++j) {
        const int p = lane + 32 * j;
        if (p < np) {
            float g[E], b[E], o[E];
            Piece<T>::load(gamma + p * E, g);
            Piece<T>::load(beta + p * E, b);
#pragma unroll
            for (int e = 0; e < E; ++e) o[e] = fmaf((v[j][e] - mean) * rstd, g[e], b[e]);
            Piece<T>::store(yr + p * E, o);
        }
    }
}

// Any width and alignment: the same arithmetic, element by element.
template <typename T>
__global__ void __launch_bounds__(256) layer_norm_any_kernel(const T *__restrict__ x,
                                                             const T *__restrict__ gamma,
                                                             const T *__restrict__ beta,
                                                             T *__restrict__ y, long rows, int D,
                                                             float eps) {
    pdl_wait();
    pdl_trigger();
    const long row = (long)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const T *xr = x + row * D;
    float s = 0.f;
    for (int c = lane; c < D; c += 32) s += to_f32(xr[c]);
    const float mean = warp_sum(s) / (float)D;
    float q = 0.f;
    for (int c = lane; c < D; c += 32) {
        const float d = to_f32(xr[c]) - mean;
        q = fmaf(d, d, q);
    }
    const float rstd = rsqrtf(warp_sum(q) / (float)D + eps);
    T *yr = y + row * D;
    for (int c = lane; c < D; c += 32)
        yr[c] = from_f32<T>(fmaf((to_f32(xr[c]) - mean) * rstd, to_f32(gamma[c]), to_f32(beta[c])));
}

template <typename T>
cudaError_t launch_ln(long rows, int D, const void *x, const void *gamma, const void *beta,
                      float eps, void *y, cudaStream_t s) {
    constexpr int E = Piece<T>::E;
    const dim3 grid((unsigned)((rows + 7) / 8)), block(256);
    const bool aligned = (uintptr_t)x % 16 == 0 && (uintptr_t)y % 16 == 0 &&
                         (uintptr_t)gamma % 16 == 0 && (uintptr_t)beta % 16 == 0 && D % E == 0;
    const T *X = static_cast<const T *>(x), *G = static_cast<const T *>(gamma),
            *Bt = static_cast<const T *>(beta);
    T *Y = static_cast<T *>(y);
    const int per_lane = (D / E + 31) / 32;
    if (aligned && per_lane <= 2)
        return launch_pdl(layer_norm_kernel<T, 2>, grid, block, 0, s, X, G, Bt, Y, rows, D, eps);
    if (aligned && per_lane <= 5)
        return launch_pdl(layer_norm_kernel<T, 5>, grid, block, 0, s, X, G, Bt, Y, rows, D, eps);
    if (aligned && per_lane <= 8)
        return launch_pdl(layer_norm_kernel<T, 8>, grid, block, 0, s, X, G, Bt, Y, rows, D, eps);
    return launch_pdl(layer_norm_any_kernel<T>, grid, block, 0, s, X, G, Bt, Y, rows, D, eps);
}

}  // namespace

cudaError_t launch_layer_norm(int dtype, long rows, int D, const void *x, const void *gamma,
                              const void *beta, float eps, void *y, cudaStream_t s) {
    if (rows < 1) return cudaSuccess;
    return dtype == DT_BF16 ? launch_ln<__nv_bfloat16>(rows, D, x, gamma, beta, eps, y, s)
                            : launch_ln<float>(rows, D, x, gamma, beta, eps, y, s);
}

}  // namespace ptdit
