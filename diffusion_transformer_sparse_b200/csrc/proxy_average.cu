// Window averaging: the proxy tokens of GIIM.
//
// Qihoo-T2X reading note, §3 Method, Eq. GIIM "Averaging" and the code
// listing's get_proxy_token(mode="mean"): every p_f x p_h x p_w window of the
// token grid is averaged into one proxy token.
//
// The kernel is a pure HBM stream: it reads every latent element once and
// writes every proxy element once.  One CTA owns one proxy; its threads are
// (16-byte channel chunk) x (token group), about 8 tokens per group.  A warp
// reads 512 contiguous bytes of one token row per load, each thread issues
// all its (up to 8) independent 16-byte loads before the first add, and the
// token groups are summed through shared memory in a fixed order, so the
// result is bitwise deterministic.
#include "common.cuh"

namespace ptdit {
namespace {

template <typename T, int VEC>
struct Chunk;
template <>
struct Chunk<__nv_bfloat16, 8> {
    uint4 raw;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
        raw = __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ void add_to(float *acc) const {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            acc[2 * i] += f.x;
            acc[2 * i + 1] += f.y;
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
struct Chunk<float, 4> {
    float4 raw;
    __device__ __forceinline__ void load(const float *p) {
        raw = __ldg(reinterpret_cast<const float4 *>(p));
    }
    __device__ __forceinline__ void add_to(float *acc) const {
        acc[0] += raw.x; acc[1] += raw.y; acc[2] += raw.z; acc[3] += raw.w;
    }
    __device__ __forceinline__ static void store(float *p, const float *v) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <typename T>
struct Chunk<T, 1> {
    T raw;
    __device__ __forceinline__ void load(const T *p) { raw = p[0]; }
    __device__ __forceinline__ void add_to(float *acc) const { acc[0] += to_f32(raw); }
    __device__ __forceinline__ static void store(T *p, const float *v) { p[0] = from_f32<T>(v[0]); }
};

// blockIdx.x = b * M + m.  Thread t: chunk lane cl = t % CHT, token group
// gi = t / CHT; the lanes step over the CH chunks of a row CHT at a time.
template <typename T, int VEC>
__global__ void __launch_bounds__(1024) proxy_average_kernel(const T *__restrict__ z,
                                                             T *__restrict__ out, ProxyGeom g,
                                                             int D, int CHT, int G) {
    extern __shared__ float red[];  // [G-1][CHT][VEC]
    pdl_wait();  // z is complete
    pdl_trigger();
    const int CH = D / VEC;
    const int m = blockIdx.x % g.M;
    const int b = blockIdx.x / g.M;
    const int cl = threadIdx.x % CHT;
    const int gi = threadIdx.x / CHT;
    const long N = (long)g.f * g.h * g.w;
    const T *zw = z + (long)b * N * D + (long)proxy_token(g, m, 0) * D;

    for (int c0 = 0; c0 < CH; c0 += CHT) {
        const int c = c0 + cl;
        float acc[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
        if (gi < G && c < CH) {
            const T *zb = zw + (long)c * VEC;
            // token k of the window sits (a*h + r)*w + q tokens after the first one;
            // each batch issues up to 8 independent 16-byte loads before adding
            for (int k0 = gi; k0 < g.P; k0 += 8 * G) {
                Chunk<T, VEC> ch[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int k = k0 + u * G;
                    if (k < g.P) {
                        const int rest = fdiv(g.f_pw, k), q = k - rest * g.pw;
                        const int a = fdiv(g.f_ph, rest), r = rest - a * g.ph;
                        ch[u].load(zb + ((long)(a * g.h + r) * g.w + q) * D);
                    }
                }
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (k0 + u * G < g.P) ch[u].add_to(acc);
            }
        }
        if (gi > 0 && gi < G) {
#pragma unroll
            for (int i = 0; i < VEC; ++i) red[((gi - 1) * CHT + cl) * VEC + i] = acc[i];
        }
        __syncthreads();
        if (gi == 0 && c < CH) {
            for (int j = 1; j < G; ++j) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) acc[i] += red[((j - 1) * CHT + cl) * VEC + i];
            }
            float v[VEC];
#pragma unroll
            for (int i = 0; i < VEC; ++i) v[i] = acc[i] / (float)g.P;
            Chunk<T, VEC>::store(out + ((long)b * g.M + m) * D + (long)c * VEC, v);
        }
        __syncthreads();
    }
}

template <typename T, int VEC>
cudaError_t launch_avg(const ProxyGeom &g, int B, int D, const void *z, void *out,
                       cudaStream_t s) {
    const int CH = D / VEC;
    const int CHT = CH < 512 ? CH : 512;
    // token groups: about 8 loads per thread, at most 1024 threads per CTA
    int G = (g.P + 7) / 8;
    if (G > 1024 / CHT) G = 1024 / CHT;
    if (G < 1) G = 1;
    const int threads = CHT * G;
    const size_t smem = (size_t)(G - 1) * CHT * VEC * sizeof(float);
    return launch_pdl(proxy_average_kernel<T, VEC>, dim3((unsigned)(B * g.M)), dim3(threads), smem, s,
                      static_cast<const T *>(z), static_cast<T *>(out), g, D, CHT, G);
}

template <typename T, int VEC>
struct Vec {
    using type = T;
};
template <>
struct Vec<__nv_bfloat16, 8> {
    using type = uint4;
};
template <>
struct Vec<float, 4> {
    using type = float4;
};

// Single-token proxies: out[b, m] = z[b, member slot(b, m) of window m], with
// slot 0 (the window's first token in (t, y, x) order: its top-left token in
// its first frame) when `slots` is null.  One warp per proxy row, 16-byte
// copies; a slot outside [0, P) leaves the row zero and records
// PTDIT_ERR_SHAPE in the status word.
template <typename T, int VEC>
__global__ void __launch_bounds__(256) proxy_select_kernel(const T *__restrict__ z,
                                                           T *__restrict__ out, ProxyGeom g,
                                                           int B, int D,
                                                           const int32_t *__restrict__ slots,
                                                           int *status) {
    pdl_wait();
    pdl_trigger();
    const long row = (long)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= (long)B * g.M) return;
    const int m = static_cast<int>(row % g.M);
    const long b = row / g.M;
    const int slot = slots ? slots[row] : 0;
    const bool ok = slot >= 0 && slot < g.P;
    if (!ok && lane == 0) atomicExch(status, 2 /* PTDIT_ERR_SHAPE */);
    const long N = (long)g.f * g.h * g.w;
    const T *src = z + (b * N + (ok ? proxy_token(g, m, slot) : 0)) * D;
    T *dst = out + row * D;
    using V = typename Vec<T, VEC>::type;
    const V *vs = reinterpret_cast<const V *>(src);
    V *vd = reinterpret_cast<V *>(dst);
    const int CH = D / VEC;
    for (int c = lane; c < CH; c += 32) vd[c] = ok ? vs[c] : V{};
}

template <typename T, int VEC>
cudaError_t launch_select(const ProxyGeom &g, int B, int D, const void *z, void *out,
                          const int32_t *slots, int *status, cudaStream_t s) {
    const long rows = (long)B * g.M;
    return launch_pdl(proxy_select_kernel<T, VEC>, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, s,
                      static_cast<const T *>(z), static_cast<T *>(out), g, B, D, slots, status);
}

}  // namespace

cudaError_t launch_proxy_select(int dtype, const ProxyGeom &g, int B, int D, const void *z,
                                void *proxies, const int32_t *slots, int *status,
                                cudaStream_t s) {
    const bool aligned = ((uintptr_t)z % 16 == 0) && ((uintptr_t)proxies % 16 == 0);
    if (dtype == DT_BF16) {
        if (aligned && D % 8 == 0)
            return launch_select<__nv_bfloat16, 8>(g, B, D, z, proxies, slots, status, s);
        return launch_select<__nv_bfloat16, 1>(g, B, D, z, proxies, slots, status, s);
    }
    if (aligned && D % 4 == 0) return launch_select<float, 4>(g, B, D, z, proxies, slots, status, s);
    return launch_select<float, 1>(g, B, D, z, proxies, slots, status, s);
}

cudaError_t launch_proxy_average(int dtype, const ProxyGeom &g, int B, int D, const void *z,
                                 void *proxies, cudaStream_t s) {
    const bool aligned = ((uintptr_t)z % 16 == 0) && ((uintptr_t)proxies % 16 == 0);
    if (dtype == DT_BF16) {
        if (aligned && D % 8 == 0) return launch_avg<__nv_bfloat16, 8>(g, B, D, z, proxies, s);
        return launch_avg<__nv_bfloat16, 1>(g, B, D, z, proxies, s);
    }
    if (aligned && D % 4 == 0) return launch_avg<float, 4>(g, B, D, z, proxies, s);
    return launch_avg<float, 1>(g, B, D, z, proxies, s);
}

}  // namespace ptdit
