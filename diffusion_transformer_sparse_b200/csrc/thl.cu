// Relayout of a row-major projection output into tiled head layout blocks,
// and the zeroing of tile rows that hold no token (see thl.cuh).  The fused
// projection epilogue writes THL directly; this kernel serves the projection
// paths that write row-major, and the ragged tail rows of the fused path.
#include "thl.cuh"

namespace ptdit {
namespace {

__global__ void thl_fill_kernel(Thl t, int B, int heads, int d, const uint4 *__restrict__ src,
                                long ld, uint8_t *__restrict__ dst, int tile0, long items) {
    pdl_wait();  // the projection output (or the blocks being completed) is complete
    pdl_trigger();
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= items) return;
    const int U = thl_units(d, t.vpad);
    const int u = static_cast<int>(idx % U);
    long rest = idx / U;
    const int r = static_cast<int>(rest % kThlRows);
    rest /= kThlRows;
    const int h = static_cast<int>(rest % heads);
    rest /= heads;
    const int span = t.tiles - tile0;  // tiles covered per batch item
    const int tile = tile0 + static_cast<int>(rest % span);
    const int b = static_cast<int>(rest / span);
    const long tok = thl_token(t, tile, r);
    if (!src && tok >= 0) return;  // only the rows without a token
    uint4 v = make_uint4(0, 0, 0, 0);
    if (src && tok >= 0 && u * 8 < d)
        v = src[(((long)b * t.rows_pb + tok) * ld + (long)h * d + u * 8) / 8];
    else if (src && tok >= 0 && t.ones && u * 8 == d)
        v = thl_ones_unit();
    const long blk = ((long)b * t.tiles + tile) * heads + h;
    *reinterpret_cast<uint4 *>(dst + blk * thl_block_bytes(d, t.vpad) + thl_unit(r, u, t.vpad)) = v;
}

}  // namespace

cudaError_t launch_thl_fill(const Thl &t, int B, int heads, int d, const void *src, long ld,
                            void *dst, cudaStream_t s) {
    // with src == nullptr only the last tile of each batch item can hold empty rows
    const int tile0 = src ? 0 : t.tiles - 1;
    const long items = (long)B * (t.tiles - tile0) * heads * kThlRows * thl_units(d, t.vpad);
    if (items <= 0) return cudaSuccess;
    const int threads = 256;
    const long blocks = (items + threads - 1) / threads;
    return launch_pdl(thl_fill_kernel, dim3((unsigned)blocks), dim3(threads), 0, s, t, B, heads, d,
                      static_cast<const uint4 *>(src), ld, static_cast<uint8_t *>(dst), tile0, items);
}

}  // namespace ptdit
