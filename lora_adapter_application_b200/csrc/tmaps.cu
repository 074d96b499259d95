// 2-D TMA tensor maps for the stacked adapter tensors, encoded on the host
// through the driver entry point the CUDA runtime exposes, and cached: a
// serving loop calls with the same adapter tensors over and over.
#include "kernels.cuh"

#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

namespace lora {
namespace {

struct Entry {
    const void *base;
    uint64_t inner, outer, stride;
    uint32_t box_inner, box_outer;
    int swizzle;
    int dev;
    CUtensorMap map;
};

constexpr int kCache = 256;
std::mutex g_mu;
Entry g_cache[kCache];
int g_used = 0, g_next = 0;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

int tensor_map_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t outer,
                  uint32_t box_inner, uint32_t box_outer, int swizzle, uint64_t row_stride) {
    if (row_stride == 0) row_stride = inner;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_used; ++i) {
        const Entry &e = g_cache[i];
        if (e.base == base && e.inner == inner && e.outer == outer && e.stride == row_stride &&
            e.box_inner == box_inner &&
            e.box_outer == box_outer && e.swizzle == swizzle && e.dev == dev) {
            *out = e.map;
            return LORA_OK;
        }
    }
    auto fn = encoder();
    if (!fn) return cuda_fail("cuTensorMapEncodeTiled: driver entry point not found");
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride * 2};   // bf16 rows
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap m;
    const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                          : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail("cuTensorMapEncodeTiled failed");
    Entry &e = g_cache[g_used < kCache ? g_used++ : (g_next++ % kCache)];
    e.base = base;
    e.inner = inner;
    e.outer = outer;
    e.stride = row_stride;
    e.box_inner = box_inner;
    e.box_outer = box_outer;
    e.swizzle = swizzle;
    e.dev = dev;
    e.map = m;
    *out = m;
    return LORA_OK;
}

// A [rows][inner] bf16 matrix (row stride `row_stride` elements) viewed as
// [inner / 64][rows][64]: boxes of 64 columns x box_rows rows x box_chunks
// consecutive 64-column chunks, 128-byte swizzle.  inner must be a multiple
// of 64; chunks past the end read as zero.
int tensor_map_chunks(CUtensorMap *out, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t row_stride, uint32_t box_rows, uint32_t box_chunks) {
    struct E3 {
        const void *base;
        uint64_t inner, rows, stride;
        uint32_t br, bc;
        int dev;
        CUtensorMap map;
    };
    static E3 cache[64];
    static int used = 0, next = 0;
    if (inner % 64) return LORA_ERR_SHAPE;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < used; ++i) {
        const E3 &e = cache[i];
        if (e.base == base && e.inner == inner && e.rows == rows && e.stride == row_stride && e.br == box_rows &&
            e.bc == box_chunks && e.dev == dev) {
            *out = e.map;
            return LORA_OK;
        }
    }
    auto fn = encoder();
    if (!fn) return cuda_fail("cuTensorMapEncodeTiled: driver entry point not found");
    const cuuint64_t dims[3] = {64, rows, inner / 64};
    const cuuint64_t strides[2] = {row_stride * 2, 128};   // bytes: next row, next 64-column chunk
    const cuuint32_t box[3] = {64, box_rows, box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap m;
    const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail("cuTensorMapEncodeTiled failed");
    E3 &e = cache[used < 64 ? used++ : (next++ % 64)];
    e.base = base;
    e.inner = inner;
    e.rows = rows;
    e.stride = row_stride;
    e.br = box_rows;
    e.bc = box_chunks;
    e.dev = dev;
    e.map = m;
    *out = m;
    return LORA_OK;
}

}  // namespace lora
