// Attention core on the CUDA cores: the fp32 path, and any shape the
// tensor-core attention does not take.
//
// Computes, per head, softmax(Q K^T / sqrt(d)) V with an online softmax over
// key tiles (one pass, running row max and row sum), fp32 throughout.
// ATT_ROWS: queries and keys are row ranges of each batch item (proxy SA,
// latent->proxy cross-attention, full SA).  ATT_WINDOW: queries and keys are
// the tokens of one TCM window of the grid rolled by -shift (Qihoo-T2X reading
// note §3, Eq. TCM); the gather and the roll happen in the row address, and
// the shift mask is the comparison of the wrap bits of query and key.
#include <math.h>

#include "common.cuh"

namespace ptdit {
namespace {

constexpr int BQ = 32, BKT = 32, NT = 128;

template <typename T, int DMAX>
__global__ void __launch_bounds__(NT) attn_simt_kernel(AttnArgs a) {
    extern __shared__ float sm[];
    const int d = a.d;
    float *Qs = sm;                         // [BQ][d]
    float *Ks = Qs + BQ * d;                // [BKT][d + 1]
    float *Vs = Ks + BKT * (d + 1);         // [BKT][d]
    float *Ps = Vs + BKT * d;               // [BQ][BKT]
    int *qwrap = reinterpret_cast<int *>(Ps + BQ * BKT);  // [BQ]
    int *kwrap = qwrap + BQ;                              // [BKT]
    long *krow = reinterpret_cast<long *>(kwrap + BKT + (BKT & 1)); // [BKT]
    long *qrow = krow + BKT;                                        // [BQ]

    const T *__restrict__ q = static_cast<const T *>(a.q);
    const T *__restrict__ k = static_cast<const T *>(a.k);
    const T *__restrict__ v = static_cast<const T *>(a.v);
    T *o = static_cast<T *>(a.o);
    const int h = blockIdx.y;
    const int tid = threadIdx.x, r = tid / 4, kg = tid % 4;

    // Query and key sets of this block.
    int b, win = 0, nq, nk;
    if (a.mode == ATT_WINDOW) {
        b = blockIdx.z / a.geom.nwin;
        win = blockIdx.z % a.geom.nwin;
        nq = nk = a.geom.n;
    } else {
        b = blockIdx.z;
        nq = a.nq;
        nk = a.nk;
    }
    const int q0 = blockIdx.x * BQ;
    if (q0 >= nq) return;

    for (int i = tid; i < BQ; i += NT) {
        const int slot = q0 + i;
        long row = -1;
        int wr = 0;
        if (slot < nq) {
            if (a.mode == ATT_WINDOW)
                row = (long)b * a.q_bstride + window_token(a.geom, win, slot, &wr);
            else
                row = (long)b * a.q_bstride + slot;
        }
        qrow[i] = row;
        qwrap[i] = wr;
    }
    __syncthreads();
    for (int idx = tid; idx < BQ * d; idx += NT) {
        const int i = idx / d, c = idx % d;
        const long row = qrow[i];
        Qs[idx] = row >= 0 ? to_f32(q[row * a.ldq + (long)h * d + c]) : 0.f;
    }

    float m_i = -INFINITY, l_i = 0.f;
    float acc[DMAX / 4];
#pragma unroll
    for (int j = 0; j < DMAX / 4; ++j) acc[j] = 0.f;

    for (int k0 = 0; k0 < nk; k0 += BKT) {
        __syncthreads();
        for (int j = tid; j < BKT; j += NT) {
            const int slot = k0 + j;
            long row = -1;
            int wr = 0;
            if (slot < nk) {
                if (a.mode == ATT_WINDOW)
                    row = (long)b * a.k_bstride + window_token(a.geom, win, slot, &wr);
                else
                    row = (long)b * a.k_bstride + slot;
            }
            krow[j] = row;
            kwrap[j] = wr;
        }
        __syncthreads();
        for (int idx = tid; idx < BKT * d; idx += NT) {
            const int j = idx / d, c = idx % d;
            const long row = krow[j];
            Ks[j * (d + 1) + c] = row >= 0 ? to_f32(k[row * a.ldk + (long)h * d + c]) : 0.f;
            Vs[j * d + c] = row >= 0 ? to_f32(v[row * a.ldv + (long)h * d + c]) : 0.f;
        }
        __syncthreads();

        // scores of row r for keys kg, kg+4, ...
        float sc[BKT / 4];
        float tmax = -INFINITY;
#pragma unroll
        for (int u = 0; u < BKT / 4; ++u) {
            const int j = kg + 4 * u;
            float s = -INFINITY;
            const bool ok = krow[j] >= 0 && qrow[r] >= 0 &&
                            (a.mode != ATT_WINDOW || kwrap[j] == qwrap[r]);
            if (ok) {
                float dot = 0.f;
                for (int c = 0; c < d; ++c) dot = fmaf(Qs[r * d + c], Ks[j * (d + 1) + c], dot);
                s = dot * a.scale;
            }
            sc[u] = s;
            tmax = fmaxf(tmax, s);
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float m_new = fmaxf(m_i, tmax);
        // rows with every key so far masked keep m = -inf and contribute nothing
        const float ref = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = (m_i == -INFINITY) ? 0.f : expf(m_i - ref);
        float psum = 0.f;
#pragma unroll
        for (int u = 0; u < BKT / 4; ++u) {
            const float p = (sc[u] == -INFINITY) ? 0.f : expf(sc[u] - ref);
            Ps[r * BKT + kg + 4 * u] = p;
            psum += p;
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 1);
        psum += __shfl_xor_sync(0xffffffffu, psum, 2);
        l_i = l_i * alpha + psum;
        m_i = m_new;
        __syncwarp();
#pragma unroll
        for (int jj = 0; jj < DMAX / 4; ++jj) {
            const int c = kg + 4 * jj;
            if (c < d) {
                float s = acc[jj] * alpha;
                for (int j = 0; j < BKT; ++j) s = fmaf(Ps[r * BKT + j], Vs[j * d + c], s);
                acc[jj] = s;
            }
        }
    }

    const long row = qrow[r];
    if (row >= 0) {
        const float inv = 1.f / l_i;
#pragma unroll
        for (int jj = 0; jj < DMAX / 4; ++jj) {
            const int c = kg + 4 * jj;
            if (c < d) o[row * a.ldo + (long)h * d + c] = from_f32<T>(acc[jj] * inv);
        }
    }
}

template <typename T, int DMAX>
cudaError_t launch_simt(const AttnArgs &a, cudaStream_t s) {
    const int d = a.d;
    const size_t smem = sizeof(float) * (BQ * d + BKT * (d + 1) + BKT * d + BQ * BKT) +
                        sizeof(int) * (BQ + BKT + 1) + sizeof(long) * (BKT + BQ) + 16;
    cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, DMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nq = a.mode == ATT_WINDOW ? a.geom.n : a.nq;
    const int nz = a.mode == ATT_WINDOW ? a.B * a.geom.nwin : a.B;
    dim3 grid((nq + BQ - 1) / BQ, a.heads, nz);
    attn_simt_kernel<T, DMAX><<<grid, NT, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_simt_t(const AttnArgs &a, cudaStream_t s) {
    if (a.d <= 32) return launch_simt<T, 32>(a, s);
    if (a.d <= 64) return launch_simt<T, 64>(a, s);
    if (a.d <= 96) return launch_simt<T, 96>(a, s);
    return launch_simt<T, 128>(a, s);
}

}  // namespace

cudaError_t launch_attention_simt(const AttnArgs &a, cudaStream_t s) {
    if (a.d > 128) return cudaErrorInvalidValue;
    if (a.dtype == DT_BF16) return launch_simt_t<__nv_bfloat16>(a, s);
    return launch_simt_t<float>(a, s);
}

}  // namespace ptdit
