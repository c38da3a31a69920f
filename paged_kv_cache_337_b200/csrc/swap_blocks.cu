// swap_blocks.cu — block swap between the GPU pool and a pool in pinned host
// memory ("PagedAttention 动态内存分页" page, 动态块分配与回收: when GPU memory
// runs short, a sequence's KV blocks move to CPU memory and come back when
// it runs again; 性能监控要点 names the swap bandwidth as the figure to watch).
//
// One launch moves every pair: each CTA copies one chunk of one block of K
// or V with several vectors in flight per thread.  The host side is reached
// through its device mapping, so the kernel's loads (swap-in) or stores
// (swap-out) cross the host link directly, with no staging copy.  Bound: the
// host link.
#include "common.cuh"

namespace pkv {
namespace {

constexpr int kThreads = 256;
constexpr int kVecsPerThread = 4;

template <typename V>
__global__ void __launch_bounds__(kThreads)
swap_blocks_kernel(const V* __restrict__ src_key, const V* __restrict__ src_value,
                   V* __restrict__ dst_key, V* __restrict__ dst_value,
                   const int32_t* __restrict__ block_pairs, int num_pairs, int src_num_blocks,
                   int dst_num_blocks, int64_t block_vecs, int64_t src_stride_vecs,
                   int64_t dst_stride_vecs, int chunks_per_block, int32_t* __restrict__ dev_error) {
    constexpr int kChunk = kThreads * kVecsPerThread;
    const int planes = src_value != nullptr ? 2 : 1;  // K and V, or one pool
    const int64_t item = blockIdx.x;
    const int per_pair = planes * chunks_per_block;
    const int pair = (int)(item / per_pair);
    const int r = (int)(item - (int64_t)pair * per_pair);
    const bool is_v = r >= chunks_per_block;
    const int chunk = is_v ? r - chunks_per_block : r;
    const int32_t src = block_pairs[2 * pair];
    const int32_t dst = block_pairs[2 * pair + 1];
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
        if (r == 0 && threadIdx.x == 0) report_error(dev_error, PKV_DEVERR_PAIR, pair);
        return;
    }
    const V* s = (is_v ? src_value : src_key) + (int64_t)src * src_stride_vecs;
    V* d = (is_v ? dst_value : dst_key) + (int64_t)dst * dst_stride_vecs;
    const int64_t base = (int64_t)chunk * kChunk + threadIdx.x;
    V buf[kVecsPerThread];
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j) {
        const int64_t v = base + (int64_t)j * kThreads;
        if (v < block_vecs) buf[j] = s[v];
    }
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j) {
        const int64_t v = base + (int64_t)j * kThreads;
        if (v < block_vecs) d[v] = buf[j];
    }
}

// The address a kernel on the current device may dereference for p: device
// (or managed) memory as it is, pinned host memory through its device
// mapping.  Pageable host memory, or host memory without a mapping, is an
// error: the kernel must never touch an address it cannot reach.
int device_address(const void* p, const char* what, const void** out) {
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(PKV_ERR_INVALID, "pkv_swap_blocks: %s: %s", what, cudaGetErrorString(e));
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged ||
        a.type == cudaMemoryTypeHost) {
        if (a.devicePointer == nullptr)
            return fail(PKV_ERR_INVALID,
                        "pkv_swap_blocks: %s is host memory with no device mapping", what);
        *out = a.devicePointer;
        return PKV_OK;
    }
    return fail(PKV_ERR_INVALID,
                "pkv_swap_blocks: %s is pageable host memory (pin it: cudaHostAlloc)", what);
}

template <typename V>
int launch_swap(const void* sk, const void* sv, void* dk, void* dv, const int32_t* pairs,
                int num_pairs, int src_nb, int dst_nb, int64_t block_bytes, int64_t src_stride,
                int64_t dst_stride, int32_t* dev_error, cudaStream_t stream) {
    constexpr int64_t kChunk = (int64_t)kThreads * kVecsPerThread;
    const int64_t block_vecs = block_bytes / (int64_t)sizeof(V);
    const int64_t chunks = (block_vecs + kChunk - 1) / kChunk;
    const int64_t grid = (int64_t)num_pairs * (sv ? 2 : 1) * chunks;
    PKV_REQUIRE(grid < (1ll << 31), PKV_ERR_INVALID, "pkv_swap_blocks: too many pairs");
    swap_blocks_kernel<V><<<(unsigned)grid, kThreads, 0, stream>>>(
        static_cast<const V*>(sk), static_cast<const V*>(sv), static_cast<V*>(dk),
        static_cast<V*>(dv), pairs, num_pairs, src_nb, dst_nb, block_vecs,
        src_stride / (int64_t)sizeof(V), dst_stride / (int64_t)sizeof(V), (int)chunks,
        dev_error);
    return launch_status("pkv_swap_blocks");
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_swap_blocks(const void* src_key, const void* src_value, void* dst_key,
                               void* dst_value, const int32_t* block_pairs, int num_pairs,
                               int src_num_blocks, int dst_num_blocks, int64_t block_bytes,
                               int64_t src_block_stride, int64_t dst_block_stride,
                               int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_swap_blocks");
    using namespace pkv;
    PKV_REQUIRE(num_pairs >= 0 && src_num_blocks >= 0 && dst_num_blocks >= 0 &&
                    block_bytes > 0 && block_bytes % 4 == 0,
                PKV_ERR_INVALID, "pkv_swap_blocks: bad sizes (block_bytes %lld)",
                (long long)block_bytes);
    PKV_REQUIRE(src_block_stride >= block_bytes && dst_block_stride >= block_bytes &&
                    src_block_stride % 4 == 0 && dst_block_stride % 4 == 0,
                PKV_ERR_INVALID, "pkv_swap_blocks: block strides %lld, %lld",
                (long long)src_block_stride, (long long)dst_block_stride);
    PKV_REQUIRE((src_value == nullptr) == (dst_value == nullptr), PKV_ERR_INVALID,
                "pkv_swap_blocks: src_value and dst_value must both be given or both NULL");
    if (num_pairs == 0) return PKV_OK;
    PKV_REQUIRE(src_key && dst_key && block_pairs, PKV_ERR_INVALID,
                "pkv_swap_blocks: NULL pointer");
    DeviceGuard guard(stream, block_pairs);
    const void *sk, *sv = nullptr, *dk, *dv = nullptr, *pairs;
    int st;
    if ((st = device_address(src_key, "src_key", &sk)) != PKV_OK) return st;
    if ((st = device_address(dst_key, "dst_key", &dk)) != PKV_OK) return st;
    if ((st = device_address(block_pairs, "block_pairs", &pairs)) != PKV_OK) return st;
    if (src_value) {
        if ((st = device_address(src_value, "src_value", &sv)) != PKV_OK) return st;
        if ((st = device_address(dst_value, "dst_value", &dv)) != PKV_OK) return st;
    }
    auto all_aligned = [&](uintptr_t a) {
        bool ok = (uintptr_t)sk % a == 0 && (uintptr_t)dk % a == 0 &&
                  block_bytes % (int64_t)a == 0 && src_block_stride % (int64_t)a == 0 &&
                  dst_block_stride % (int64_t)a == 0;
        if (sv) ok = ok && (uintptr_t)sv % a == 0 && (uintptr_t)dv % a == 0;
        return ok;
    };
    const int32_t* pp = static_cast<const int32_t*>(pairs);
    if (all_aligned(16))
        return launch_swap<uint4>(sk, sv, const_cast<void*>(dk), const_cast<void*>(dv), pp,
                                  num_pairs, src_num_blocks, dst_num_blocks, block_bytes,
                                  src_block_stride, dst_block_stride, dev_error, stream);
    PKV_REQUIRE(all_aligned(4), PKV_ERR_INVALID,
                "pkv_swap_blocks: pools must be 4-byte aligned");
    return launch_swap<uint32_t>(sk, sv, const_cast<void*>(dk), const_cast<void*>(dv), pp,
                                 num_pairs, src_num_blocks, dst_num_blocks, block_bytes,
                                 src_block_stride, dst_block_stride, dev_error, stream);
}
