// copy_blocks.cu — copy-on-write block copy ("PagedAttention 动态内存分页"
// page, 写时复制与内存共享: a block shared by several sequences is copied when
// one of them needs to write into it).
//
// A block of one cache is bs * Hkv * D contiguous elements, so each (src,
// dst) pair is two contiguous copies (K and V).  Each CTA moves one chunk of
// one pair with 16-byte vectors and several loads in flight per thread; the
// grid covers pairs x chunks.  Bound: HBM (read + write of whole blocks).
#include "common.cuh"

namespace pkv {
namespace {

constexpr int kThreads = 256;
constexpr int kVecsPerThread = 4;
constexpr int kChunkVecs = kThreads * kVecsPerThread;  // 16 KiB per CTA

__global__ void __launch_bounds__(kThreads)
copy_blocks_kernel(uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                   const int32_t* __restrict__ block_pairs, int num_pairs, int num_blocks,
                   int64_t block_vecs, int64_t block_stride_vecs, int chunks_per_cache,
                   int32_t* __restrict__ dev_error) {
    const int64_t item = blockIdx.x;
    const int per_pair = 2 * chunks_per_cache;
    const int pair = (int)(item / per_pair);
    const int r = (int)(item - (int64_t)pair * per_pair);
    const bool is_v = r >= chunks_per_cache;
    const int chunk = is_v ? r - chunks_per_cache : r;
    const int32_t src = __ldg(block_pairs + 2 * pair);
    const int32_t dst = __ldg(block_pairs + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (r == 0 && threadIdx.x == 0) report_error(dev_error, PKV_DEVERR_PAIR, pair);
        return;
    }
    uint4* cache = is_v ? value_cache : key_cache;
    const uint4* s = cache + (int64_t)src * block_stride_vecs;
    uint4* d = cache + (int64_t)dst * block_stride_vecs;
    const int64_t base = (int64_t)chunk * kChunkVecs + threadIdx.x;
    uint4 buf[kVecsPerThread];
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j) {
        const int64_t v = base + (int64_t)j * kThreads;
        if (v < block_vecs) buf[j] = __ldg(s + v);
    }
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j) {
        const int64_t v = base + (int64_t)j * kThreads;
        if (v < block_vecs) d[v] = buf[j];
    }
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_copy_blocks(void* key_cache, void* value_cache, const int32_t* block_pairs,
                               int num_pairs, int num_blocks, int block_size, int num_kv_heads,
                               int head_dim, int64_t block_stride, pkv_dtype dtype,
                               int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_copy_blocks");
    using namespace pkv;
    PKV_REQUIRE(dtype == PKV_F16 || dtype == PKV_BF16, PKV_ERR_UNSUPPORTED,
                "pkv_copy_blocks: dtype %d", (int)dtype);
    PKV_REQUIRE(num_pairs >= 0 && num_blocks >= 0 && block_size > 0 && num_kv_heads > 0 &&
                    head_dim > 0,
                PKV_ERR_INVALID, "pkv_copy_blocks: bad sizes");
    const int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    PKV_REQUIRE(block_elems % 8 == 0, PKV_ERR_INVALID,
                "pkv_copy_blocks: block_size * num_kv_heads * head_dim must be a multiple of 8");
    PKV_REQUIRE(block_stride >= block_elems && block_stride % 8 == 0, PKV_ERR_INVALID,
                "pkv_copy_blocks: block_stride %lld", (long long)block_stride);
    if (num_pairs == 0) return PKV_OK;
    PKV_REQUIRE(key_cache && value_cache && block_pairs, PKV_ERR_INVALID,
                "pkv_copy_blocks: NULL pointer");
    PKV_REQUIRE(aligned16(key_cache) && aligned16(value_cache), PKV_ERR_INVALID,
                "pkv_copy_blocks: caches must be 16-byte aligned");
    DeviceGuard guard(stream, key_cache);
    const int64_t block_vecs = block_elems / 8;
    const int64_t chunks = (block_vecs + kChunkVecs - 1) / kChunkVecs;
    const int64_t grid = (int64_t)num_pairs * 2 * chunks;
    PKV_REQUIRE(grid < (1ll << 31), PKV_ERR_INVALID, "pkv_copy_blocks: too many pairs");
    copy_blocks_kernel<<<(unsigned)grid, kThreads, 0, stream>>>(
        static_cast<uint4*>(key_cache), static_cast<uint4*>(value_cache), block_pairs,
        num_pairs, num_blocks, block_vecs, block_stride / 8, (int)chunks, dev_error);
    return launch_status("pkv_copy_blocks");
}

// ---------------------------------------------------------------------------
// Copy-on-write for FP8 (e4m3) caches: the block's bytes (the kernel above,
// in 16-byte vectors) and its per-KV-head scales.
// ---------------------------------------------------------------------------
namespace pkv {
namespace {

__global__ void copy_scales_kernel(float* __restrict__ k_scale, float* __restrict__ v_scale,
                                   const int32_t* __restrict__ block_pairs, int num_pairs,
                                   int num_blocks, int num_kv_heads) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)num_pairs * num_kv_heads) return;
    const int pair = (int)(i / num_kv_heads), h = (int)(i % num_kv_heads);
    const int32_t src = __ldg(block_pairs + 2 * pair), dst = __ldg(block_pairs + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return;  // reported above
    k_scale[(int64_t)dst * num_kv_heads + h] = k_scale[(int64_t)src * num_kv_heads + h];
    v_scale[(int64_t)dst * num_kv_heads + h] = v_scale[(int64_t)src * num_kv_heads + h];
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_copy_blocks_fp8(void* key_cache, void* value_cache, float* k_scale,
                                   float* v_scale, const int32_t* block_pairs, int num_pairs,
                                   int num_blocks, int block_size, int num_kv_heads,
                                   int head_dim, int64_t block_stride, int32_t* dev_error,
                                   cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_copy_blocks_fp8");
    using namespace pkv;
    PKV_REQUIRE(num_pairs >= 0 && num_blocks >= 0 && block_size > 0 && num_kv_heads > 0 &&
                    head_dim > 0,
                PKV_ERR_INVALID, "pkv_copy_blocks_fp8: bad sizes");
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim;
    PKV_REQUIRE(block_bytes % 16 == 0 && block_stride >= block_bytes && block_stride % 16 == 0,
                PKV_ERR_INVALID,
                "pkv_copy_blocks_fp8: block of %lld bytes, stride %lld (multiples of 16)",
                (long long)block_bytes, (long long)block_stride);
    if (num_pairs == 0) return PKV_OK;
    PKV_REQUIRE(key_cache && value_cache && k_scale && v_scale && block_pairs, PKV_ERR_INVALID,
                "pkv_copy_blocks_fp8: NULL pointer");
    PKV_REQUIRE(aligned16(key_cache) && aligned16(value_cache), PKV_ERR_INVALID,
                "pkv_copy_blocks_fp8: caches must be 16-byte aligned");
    DeviceGuard guard(stream, key_cache);
    const int64_t block_vecs = block_bytes / 16;
    const int64_t chunks = (block_vecs + kChunkVecs - 1) / kChunkVecs;
    const int64_t grid = (int64_t)num_pairs * 2 * chunks;
    PKV_REQUIRE(grid < (1ll << 31), PKV_ERR_INVALID, "pkv_copy_blocks_fp8: too many pairs");
    copy_blocks_kernel<<<(unsigned)grid, kThreads, 0, stream>>>(
        static_cast<uint4*>(key_cache), static_cast<uint4*>(value_cache), block_pairs,
        num_pairs, num_blocks, block_vecs, block_stride / 16, (int)chunks, dev_error);
    int st = launch_status("pkv_copy_blocks_fp8");
    if (st != PKV_OK) return st;
    const int64_t n = (int64_t)num_pairs * num_kv_heads;
    copy_scales_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
        k_scale, v_scale, block_pairs, num_pairs, num_blocks, num_kv_heads);
    return launch_status("pkv_copy_blocks_fp8 (scales)");
}

// ---------------------------------------------------------------------------
// Copy-on-write over every layer of a multi-layer cache in one launch: a
// physical block id names the block in all layers ("Paged KV" wiki page,
// 初始化阶段: one block holds K and V of every layer), so the pool's pairs
// apply to each layer's caches.  Grid: pairs x layers x {K, V} x chunks.
// ---------------------------------------------------------------------------
namespace pkv {
namespace {

__global__ void __launch_bounds__(kThreads)
copy_blocks_layers_kernel(uint4* const* __restrict__ key_caches,
                          uint4* const* __restrict__ value_caches, int num_layers,
                          const int32_t* __restrict__ block_pairs, int num_pairs, int num_blocks,
                          int64_t block_vecs, int64_t block_stride_vecs, int chunks_per_cache,
                          int32_t* __restrict__ dev_error) {
    const int64_t item = blockIdx.x;
    const int per_layer = 2 * chunks_per_cache;
    const int64_t per_pair = (int64_t)num_layers * per_layer;
    const int pair = (int)(item / per_pair);
    const int64_t rem = item - (int64_t)pair * per_pair;
    const int layer = (int)(rem / per_layer);
    const int r = (int)(rem - (int64_t)layer * per_layer);
    const bool is_v = r >= chunks_per_cache;
    const int chunk = is_v ? r - chunks_per_cache : r;
    const int32_t src = __ldg(block_pairs + 2 * pair);
    const int32_t dst = __ldg(block_pairs + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (rem == 0 && threadIdx.x == 0) report_error(dev_error, PKV_DEVERR_PAIR, pair);
        return;
    }
    uint4* cache = is_v ? value_caches[layer] : key_caches[layer];
    const uint4* s = cache + (int64_t)src * block_stride_vecs;
    uint4* d = cache + (int64_t)dst * block_stride_vecs;
    const int64_t base = (int64_t)chunk * kChunkVecs + threadIdx.x;
    uint4 buf[kVecsPerThread];
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j) {
        const int64_t v = base + (int64_t)j * kThreads;
        if (v < block_vecs) buf[j] = __ldg(s + v);
    }
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j) {
        const int64_t v = base + (int64_t)j * kThreads;
        if (v < block_vecs) d[v] = buf[j];
    }
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_copy_blocks_layers(void* const* key_caches, void* const* value_caches,
                                      int num_layers, const int32_t* block_pairs, int num_pairs,
                                      int num_blocks, int64_t block_bytes,
                                      int64_t block_stride_bytes, int32_t* dev_error,
                                      cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_copy_blocks_layers");
    using namespace pkv;
    PKV_REQUIRE(num_layers >= 0 && num_pairs >= 0 && num_blocks >= 0 && block_bytes > 0,
                PKV_ERR_INVALID, "pkv_copy_blocks_layers: bad sizes");
    PKV_REQUIRE(block_bytes % 16 == 0 && block_stride_bytes >= block_bytes &&
                    block_stride_bytes % 16 == 0,
                PKV_ERR_INVALID,
                "pkv_copy_blocks_layers: block of %lld bytes, stride %lld (multiples of 16)",
                (long long)block_bytes, (long long)block_stride_bytes);
    if (num_pairs == 0 || num_layers == 0) return PKV_OK;
    PKV_REQUIRE(key_caches && value_caches && block_pairs, PKV_ERR_INVALID,
                "pkv_copy_blocks_layers: NULL pointer");
    DeviceGuard guard(stream, block_pairs);
    const int64_t block_vecs = block_bytes / 16;
    const int64_t chunks = (block_vecs + kChunkVecs - 1) / kChunkVecs;
    const int64_t grid = (int64_t)num_pairs * num_layers * 2 * chunks;
    PKV_REQUIRE(grid < (1ll << 31), PKV_ERR_INVALID, "pkv_copy_blocks_layers: too many pairs");
    copy_blocks_layers_kernel<<<(unsigned)grid, kThreads, 0, stream>>>(
        reinterpret_cast<uint4* const*>(key_caches), reinterpret_cast<uint4* const*>(value_caches),
        num_layers, block_pairs, num_pairs, num_blocks, block_vecs, block_stride_bytes / 16,
        (int)chunks, dev_error);
    return launch_status("pkv_copy_blocks_layers");
}
