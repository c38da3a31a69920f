// tensor_maps.cpp — TMA tensor maps over a paged cache, encoded through the
// driver entry point the runtime hands out (no libcuda link needed).
#include "tensor_maps.h"

#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

namespace pkv {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

}  // namespace

int encode_paged_map_16bit(CUtensorMap* map, const void* cache, pkv_dtype dtype, int head_dim,
                           int num_kv_heads, int block_size, int num_blocks,
                           int64_t block_stride, int box_halves) {
    auto fn = encoder();
    if (!fn) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    constexpr int kHalf = 64;  // dims per box row: 128 bytes
    const cuuint64_t dims[5] = {(cuuint64_t)kHalf, (cuuint64_t)num_kv_heads,
                                (cuuint64_t)block_size, (cuuint64_t)(head_dim / kHalf),
                                (cuuint64_t)num_blocks};
    const cuuint64_t strides[4] = {(cuuint64_t)head_dim * 2,
                                   (cuuint64_t)num_kv_heads * head_dim * 2,
                                   (cuuint64_t)kHalf * 2, (cuuint64_t)block_stride * 2};
    const cuuint32_t halves = box_halves > 0 ? (cuuint32_t)box_halves : (cuuint32_t)(head_dim / kHalf);
    const cuuint32_t box[5] = {kHalf, 1, 16, halves, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType ty = dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(map, ty, 5, const_cast<void*>(cache), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PKV_OK;
}

}  // namespace pkv
