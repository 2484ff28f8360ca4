// Tiled head layout (THL) of the attention operands Q, K and V.
//
// The projection that produces Q, K or V writes it as one block per (batch
// item, 128-row tile, head), and each block is byte for byte the shared-memory
// tile the attention kernels' tensor cores read:
//   columns 0..63 of the head   16 atoms of 8 rows x 128 B, 128-byte swizzle
//                               (16-byte unit c of row r at unit c ^ (r & 7))
//   columns 64..79 (d > 64)     either 16 atoms of 8 rows x 32 B, 32-byte
//                               swizzle (unit u of row r at u ^ ((r >> 2) & 1))
//                               or, padded ("vpad", the V operand of the row
//                               kernel, one P V MMA of N = 128), a second set of
//                               128-byte atoms holding columns 64..127
// Columns d..79 (or d..127) and rows that hold no token are zeros, except that
// with "ones" (a V operand whose head is narrower than its tile, d = 72) column
// d of every token row holds 1: the P V product then carries the row sums of P
// in that column, summed in fp32 from exactly the bf16 P values that weight V.  Loading a
// tile is then one contiguous bulk copy; reading a head's 144-byte slice out of
// every 2304-byte token row instead keeps far fewer bytes in flight per SM.
//
// Tile rows: "identity" tiles hold rows 128 t .. 128 t + 127 of a batch item;
// "window" tiles hold the windows of the rolled grid in the order the window
// kernel visits them (BQ / n windows per tile, slots row-major in a window).
#pragma once

#include "common.cuh"

namespace ptdit {

enum ThlMode { THL_OFF = 0, THL_IDENTITY = 1, THL_WINDOW = 2 };
using Thl = ThlDesc;  // the descriptor (common.cuh): mode, vpad, tiles, rows_pb, pack, g

constexpr int kThlRows = 128;

// Bytes of one (tile, head) block.
__host__ __device__ inline uint32_t thl_block_bytes(int d, int vpad) {
    return d <= 64 ? 16384u : (vpad ? 32768u : 20480u);
}

// Byte offset, inside a block, of 16-byte unit p (head columns 8p .. 8p+7) of row r.
__host__ __device__ inline uint32_t thl_unit(int r, int p, int vpad) {
    if (p < 8) return (r >> 3) * 1024 + (r & 7) * 128 + ((p ^ (r & 7)) << 4);
    if (vpad) return 16384 + (r >> 3) * 1024 + (r & 7) * 128 + (((p - 8) ^ (r & 7)) << 4);
    return 16384 + (r >> 3) * 256 + (r & 7) * 32 + (((p - 8) ^ ((r >> 2) & 1)) << 4);
}

// The 16-byte unit holding head column d when "ones" is set: 1 in its first element.
__host__ __device__ inline uint4 thl_ones_unit() { return make_uint4(0x3F80u, 0u, 0u, 0u); }

// 16-byte units per block row (head columns rounded up to the layout's width).
__host__ __device__ inline int thl_units(int d, int vpad) { return d <= 64 ? 8 : (vpad ? 16 : 10); }

// Tile and tile row of token `tok` (0 <= tok < rows_pb) of a batch item.
__host__ __device__ inline void thl_locate(const Thl &t, long tok, int &tile, int &r) {
    if (t.mode == THL_IDENTITY) {
        tile = static_cast<int>(tok / kThlRows);
        r = static_cast<int>(tok % kThlRows);
        return;
    }
    const WinGeom &g = t.g;
    const int x = static_cast<int>(tok % g.w);
    const long ty = tok / g.w;
    const int y = static_cast<int>(ty % g.h), tt = static_cast<int>(ty / g.h);
    // position on the grid rolled by -shift
    int xr = x - g.sw, yr = y - g.sh, trr = tt - g.sf;
    if (xr < 0) xr += g.w;
    if (yr < 0) yr += g.h;
    if (trr < 0) trr += g.f;
    const int win = ((trr / g.wf) * g.nwh + yr / g.wh) * g.nww + xr / g.ww;
    const int slot = ((trr % g.wf) * g.wh + yr % g.wh) * g.ww + xr % g.ww;
    tile = win / t.pack;
    r = (win % t.pack) * g.n + slot;
}

// Token held by tile row r of tile `tile`, or -1 if the row holds none.
__host__ __device__ inline long thl_token(const Thl &t, int tile, int r) {
    if (t.mode == THL_IDENTITY) {
        const long tok = (long)tile * kThlRows + r;
        return tok < t.rows_pb ? tok : -1;
    }
    const int win = tile * t.pack + r / t.g.n;
    if (win >= t.g.nwin) return -1;
    int wrap;
    return window_token(t.g, win, r % t.g.n, &wrap);
}

// Writes zeros into the tile rows that hold no token (the last tile of each
// batch item), for every head of the operand at dst.
cudaError_t launch_thl_zero_rows(const Thl &t, int B, int heads, int d, void *dst, cudaStream_t s);

}  // namespace ptdit
