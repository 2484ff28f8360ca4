// Debug exports of the index maps, computed on the device with the same
// address functions (proxy_token / proxy_of_token / window_token) that the
// averaging and attention kernels use.
#include "common.cuh"

namespace ptdit {
namespace {

__global__ void proxy_map_kernel(ProxyGeom g, int32_t *out) {
    const int N = g.f * g.h * g.w;
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < N; t += gridDim.x * blockDim.x) {
        const int m = proxy_of_token(g, t);
        // the token's slot inside its window must lead back to it through the
        // member function the averaging kernel uses; a mismatch writes -1
        const int x = t % g.w, y = (t / g.w) % g.h, tt = t / (g.w * g.h);
        const int k = ((tt % g.pf) * g.ph + y % g.ph) * g.pw + x % g.pw;
        out[t] = (proxy_token(g, m, k) == t) ? m : -1;
    }
}

__global__ void window_map_kernel(WinGeom g, int32_t *tok, uint8_t *allowed) {
    const long total = (long)g.nwin * g.n;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total;
         i += (long)gridDim.x * blockDim.x) {
        const int win = (int)(i / g.n), slot = (int)(i % g.n);
        int wi;
        tok[i] = window_token(g, win, slot, &wi);
        if (allowed) {
            for (int j = 0; j < g.n; ++j) {
                int wj;
                window_token(g, win, j, &wj);
                allowed[i * g.n + j] = (wi == wj) ? 1 : 0;
            }
        }
    }
}

}  // namespace

cudaError_t launch_debug_proxy_map(const ProxyGeom &g, int32_t *out, cudaStream_t s) {
    proxy_map_kernel<<<64, 256, 0, s>>>(g, out);
    return cudaGetLastError();
}

cudaError_t launch_debug_window_map(const WinGeom &g, int32_t *tok, uint8_t *allowed,
                                    cudaStream_t s) {
    window_map_kernel<<<64, 256, 0, s>>>(g, tok, allowed);
    return cudaGetLastError();
}

}  // namespace ptdit


// ------------------------------------------------------------------ status word and timeout
#include "ptdit.h"
#include "tc_util.cuh"

namespace ptdit {
int report_error(int code, const char *text);
void set_debug_wait_limit_ns(unsigned long long ns);
namespace {
// One thread waits on a barrier that nothing arrives on; the bounded wait gives
// up after limit_ns and records PTDIT_ERR_TIMEOUT, as a stalled kernel would.
__global__ void debug_timeout_kernel(int *status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    tc::mbar_init(&bar, 1);
    abort = 0;
    tc::fence_mbar_init();
    (void)tc::mbar_wait(&bar, 0, &abort, status, limit_ns);
}
}  // namespace
}  // namespace ptdit

extern "C" int ptdit_device_status(int reset) {
    int *word = ptdit::device_status_ptr();
    if (!word) return ptdit::report_error(PTDIT_ERR_CUDA, "status word unavailable");
    int v = 0;
    cudaError_t e = cudaMemcpy(&v, word, sizeof v, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && reset) e = cudaMemset(word, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return ptdit::report_error(PTDIT_ERR_CUDA, cudaGetErrorString(e));
    return v;
}

extern "C" int ptdit_debug_timeout(long long limit_ns, ptdit_stream_t stream) {
    if (limit_ns <= 0 || limit_ns > 10000000000LL)
        return ptdit::report_error(PTDIT_ERR_SHAPE, "limit_ns must be in (0, 10 s]");
    int *word = ptdit::device_status_ptr();
    if (!word) return ptdit::report_error(PTDIT_ERR_CUDA, "status word unavailable");
    ptdit::debug_timeout_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(word, (unsigned long long)limit_ns);
    ptdit::count_launch();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return ptdit::report_error(PTDIT_ERR_CUDA, cudaGetErrorString(e));
    return PTDIT_OK;
}

extern "C" int ptdit_debug_wait_limit(long long limit_ns) {
    if (limit_ns < 0 || limit_ns > 10000000000LL)
        return ptdit::report_error(PTDIT_ERR_SHAPE, "limit_ns must be in [0, 10 s]");
    ptdit::set_debug_wait_limit_ns((unsigned long long)limit_ns);
    return PTDIT_OK;
}
