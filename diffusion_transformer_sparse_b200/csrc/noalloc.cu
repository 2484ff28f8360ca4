// ptdit_window_attn_static: one TCM window-attention branch whose scratch is a
// fixed device array inside this library, for callers that cannot allocate
// device memory themselves.
//
// The scratch is a file-scope __device__ array of PTDIT_STATIC_SCRATCH_BYTES.
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the first call on each device, with that device
// current, asks the runtime for the array's device address with
// cudaGetSymbolAddress and keeps it, together with the context that was
// current; later calls on that device reuse it while the same context is
// current, and look it up again in a new one (after cudaDeviceReset the
// module, and with it the array, may sit at another address).  That first
// call may load this file's device code, so make it before any stream capture
// begins.  Nothing here allocates: the call hands the array to
// ptdit_window_attn as its workspace.
#include <cuda.h>
#include <mutex>
#include <stdio.h>

#include "common.cuh"
#include "ptdit.h"

namespace ptdit {
int report_error(int code, const char *text);
}

namespace {

constexpr int kMaxDevices = 64;

// The shared scratch: every call on a device uses the same bytes, and they keep
// the previous call's contents.  The window-attention path writes every
// scratch byte it reads within the call, so nothing needs clearing.  Calls that
// overlap on the GPU (different streams, or different host threads, without
// ordering between them) race on this array.
__device__ __align__(256) unsigned char g_scratch[PTDIT_STATIC_SCRATCH_BYTES];

std::mutex g_mu;
void *g_addr[kMaxDevices] = {};
CUcontext g_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, reached through the runtime (no -lcuda).
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CUcontext current_context() {
    static CtxGetCurrentFn fn = nullptr;
    static bool looked = false;
    if (!looked) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        looked = true;
    }
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

int scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "cudaGetDevice: %s", cudaGetErrorString(e));
        return ptdit::report_error(PTDIT_ERR_CUDA, msg);
    }
    if (dev < 0 || dev >= kMaxDevices)
        return ptdit::report_error(PTDIT_ERR_CUDA, "device ordinal above 63");
    std::lock_guard<std::mutex> lock(g_mu);
    const CUcontext ctx = current_context();
    if (!g_addr[dev] || !ctx || ctx != g_ctx[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof msg, "cudaGetSymbolAddress(static scratch): %s",
                     cudaGetErrorString(e));
            return ptdit::report_error(PTDIT_ERR_CUDA, msg);
        }
        g_addr[dev] = p;
        g_ctx[dev] = ctx;
    }
    *out = g_addr[dev];
    return PTDIT_OK;
}

}  // namespace

extern "C" int ptdit_window_attn_static(const ptdit_shape *shape, const int window[3],
                                        const int shift[3], const ptdit_attn_w *w,
                                        unsigned flags, const void *z_in, void *z_out,
                                        ptdit_stream_t stream) {
    const size_t need = ptdit_workspace_bytes(shape, nullptr, window);
    if (need == 0)  // invalid shape or window: let the regular entry point name the error
        return ptdit_window_attn(shape, window, shift, w, flags, z_in, z_out, nullptr, 0,
                                 stream);
    if (need > (size_t)PTDIT_STATIC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "this shape needs %zu bytes of scratch, above the static scratch of %zu bytes "
                 "(use ptdit_window_attn with a caller-allocated workspace)",
                 need, (size_t)PTDIT_STATIC_SCRATCH_BYTES);
        return ptdit::report_error(PTDIT_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != PTDIT_OK) return rc;
    return ptdit_window_attn(shape, window, shift, w, flags, z_in, z_out, scratch,
                             (size_t)PTDIT_STATIC_SCRATCH_BYTES, stream);
}
