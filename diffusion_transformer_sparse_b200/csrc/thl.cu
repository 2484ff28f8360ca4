// Zeroing of the tile rows of a tiled-head-layout operand that hold no token
// (see thl.cuh).  The projection epilogue writes every row that holds a token;
// this kernel writes zeros over the ragged tail rows of the last tile of each
// batch item, every unit of them (a V operand's ones column included: a row
// without a token must contribute nothing to any sum).
#include "thl.cuh"

namespace ptdit {
namespace {

__global__ void thl_zero_kernel(Thl t, int B, int heads, int d, uint8_t *__restrict__ dst,
                                long items) {
    pdl_wait();  // the projection writing the blocks' other rows has completed
    pdl_trigger();
    const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= items) return;
    const int U = thl_units(d, t.vpad);
    const int u = static_cast<int>(idx % U);
    long rest = idx / U;
    const int r = static_cast<int>(rest % kThlRows);
    rest /= kThlRows;
    const int h = static_cast<int>(rest % heads);
    const int b = static_cast<int>(rest / heads);
    const int tile = t.tiles - 1;  // only the last tile of a batch item has empty rows
    if (thl_token(t, tile, r) >= 0) return;
    const long blk = ((long)b * t.tiles + tile) * heads + h;
    *reinterpret_cast<uint4 *>(dst + blk * thl_block_bytes(d, t.vpad) + thl_unit(r, u, t.vpad)) =
        make_uint4(0, 0, 0, 0);
}

}  // namespace

cudaError_t launch_thl_zero_rows(const Thl &t, int B, int heads, int d, void *dst,
                                 cudaStream_t s) {
    const long items = (long)B * heads * kThlRows * thl_units(d, t.vpad);
    if (items <= 0 || t.tiles < 1) return cudaSuccess;
    const int threads = 256;
    const long blocks = (items + threads - 1) / threads;
    return launch_pdl(thl_zero_kernel, dim3((unsigned)blocks), dim3(threads), 0, s, t, B, heads, d,
                      static_cast<uint8_t *>(dst), items);
}

}  // namespace ptdit
