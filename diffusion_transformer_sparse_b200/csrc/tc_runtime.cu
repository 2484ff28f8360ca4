// Host-side runtime pieces of the tensor-core kernels: tensor-map encoding
// through the driver entry point, the SM count, and the device status word
// that bounded device-side waits write when they give up.
#include <mutex>

#include "tc_util.cuh"

namespace ptdit {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;
std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
int g_sms[kMaxDevices] = {};
int *g_status[kMaxDevices] = {};

__device__ int g_device_status_word;

EncodeTiledFn encode_fn() {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(p);
    }
    return g_encode;
}

}  // namespace

bool encode_map_2d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                        uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
    return encode_map_2d_bf16_sw(map, base, inner, outer, row_stride_bytes, box_inner, box_outer,
                                 128);
}

bool encode_map_2d_bf16_sw(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                           uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                           int swizzle_bytes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                        : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_map_rows_heads_bf16(CUtensorMap *map, const void *base, uint64_t rows,
                                uint64_t row_pitch_bytes, int nch, int heads, int d,
                                uint32_t box_rows, uint32_t box_chunks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {8, rows, (cuuint64_t)nch, (cuuint64_t)heads};
    cuuint64_t strides[3] = {row_pitch_bytes, 16, (cuuint64_t)d * 2};
    cuuint32_t box[4] = {8, box_rows, box_chunks, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_map_head_tile_bf16(CUtensorMap *map, const void *base, uint64_t rows,
                               uint64_t row_pitch_bytes, int heads, int d, uint32_t box_elems,
                               uint32_t box_rows, int swizzle_bytes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, rows, (cuuint64_t)heads};
    cuuint64_t strides[2] = {row_pitch_bytes, (cuuint64_t)d * 2};
    cuuint32_t box[3] = {box_elems, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw =
        swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_map_out_rows_bf16(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                              uint64_t batches, uint64_t row_pitch_bytes,
                              uint64_t batch_pitch_bytes, uint32_t box_cols, uint32_t box_rows,
                              bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {cols, rows, batches};
    cuuint64_t strides[2] = {row_pitch_bytes, batch_pitch_bytes};
    cuuint32_t box[3] = {box_cols, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_map_grid_bf16(CUtensorMap *map, const void *base, int B, int F, int H, int W, int D,
                          uint32_t box_c, uint32_t box_x, uint32_t box_y, uint32_t box_t) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t e = 2;
    cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)F, (cuuint64_t)B};
    cuuint64_t strides[4] = {(cuuint64_t)D * e, (cuuint64_t)W * D * e, (cuuint64_t)H * W * D * e,
                             (cuuint64_t)F * H * W * D * e};
    cuuint32_t box[5] = {box_c, box_x, box_y, box_t, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {
thread_local unsigned long long g_wait_limit_ns = 0;
}

unsigned long long debug_wait_limit_ns() {
    return g_wait_limit_ns ? g_wait_limit_ns : tc::kWaitLimitNs;
}

void set_debug_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns = ns; }

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            g_sms[dev] = n;
    }
    return g_sms[dev];
}

int *device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_status[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status_word) != cudaSuccess) return nullptr;
        g_status[dev] = static_cast<int *>(p);
    }
    return g_status[dev];
}

}  // namespace ptdit
