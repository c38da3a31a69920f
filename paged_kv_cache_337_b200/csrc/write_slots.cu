// write_slots.cu — the slot-mapped scatter of new tokens' K/V rows into the
// paged cache ("Paged KV" wiki page, 实现原理 / 运行阶段: a decoded token is
// written to the next slot of its sequence's current block; prefill fills
// the blocks it took, in order).
//
// A token's row for all KV heads, [num_kv_heads, head_dim], is contiguous in
// the source and, inside its block, in the cache, so the kernel is a gather
// of 16-byte vectors: one thread per vector, K and V in one launch, slots
// read once per vector from L1.  Bound: HBM (read + write of the rows).
// The two divisions per vector (vector -> token, slot -> block) run in
// 32-bit arithmetic whenever the launch's vector and slot counts allow: a
// 64-bit division is a long instruction sequence, and with two per 16-byte
// vector it made a prompt-sized write issue-bound.
#include "common.cuh"

namespace pkv {
namespace {

constexpr int kThreads = 256;

// I: the type of the vector, token and slot indexes (uint32_t when every
// one of them, and the grid stride past the last, fits; else int64_t).
// Addresses are formed in 64 bits either way.
template <typename I>
__global__ void __launch_bounds__(kThreads)
write_slots_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                   uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                   const int64_t* __restrict__ slot_mapping, int num_tokens,
                   int64_t num_slots, int block_size, I row_vecs,
                   int64_t block_stride_vecs, int32_t* __restrict__ dev_error) {
    // work item i: token i / (2 * row_vecs), K (first half) or V, vector
    const I per_token = 2 * row_vecs;
    const I total = (I)num_tokens * per_token;
    const I bs = (I)block_size;
    for (I i = (I)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (I)gridDim.x * blockDim.x) {
        const I t = i / per_token;
        const I r = i - t * per_token;
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;  // padding token
        if (slot >= num_slots) {
            if (r == 0) report_error(dev_error, PKV_DEVERR_SLOT, (int)t);
            continue;
        }
        const I blk = (I)slot / bs;
        const I off = (I)slot - blk * bs;
        const bool is_v = r >= row_vecs;
        const I v = is_v ? r - row_vecs : r;
        const int64_t dst = (int64_t)blk * block_stride_vecs + (int64_t)off * row_vecs + v;
        const int64_t src = (int64_t)t * row_vecs + v;
        if (is_v)
            value_cache[dst] = __ldg(value + src);
        else
            key_cache[dst] = __ldg(key + src);
    }
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_write_slots(const void* key, const void* value, void* key_cache,
                               void* value_cache, const int64_t* slot_mapping,
                               int num_tokens, int num_blocks, int block_size,
                               int num_kv_heads, int head_dim, int64_t block_stride,
                               pkv_dtype dtype, int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_write_slots");
    using namespace pkv;
    PKV_REQUIRE(dtype == PKV_F16 || dtype == PKV_BF16, PKV_ERR_UNSUPPORTED,
                "pkv_write_slots: dtype %d", (int)dtype);
    PKV_REQUIRE(num_tokens >= 0 && num_blocks >= 0 && block_size > 0 && num_kv_heads > 0 &&
                    head_dim > 0,
                PKV_ERR_INVALID, "pkv_write_slots: bad sizes");
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    PKV_REQUIRE(row % 8 == 0, PKV_ERR_INVALID,
                "pkv_write_slots: num_kv_heads * head_dim must be a multiple of 8");
    PKV_REQUIRE(block_stride >= (int64_t)block_size * row && block_stride % 8 == 0,
                PKV_ERR_INVALID, "pkv_write_slots: block_stride %lld", (long long)block_stride);
    if (num_tokens == 0) return PKV_OK;
    PKV_REQUIRE(key && value && key_cache && value_cache && slot_mapping, PKV_ERR_INVALID,
                "pkv_write_slots: NULL pointer");
    PKV_REQUIRE(aligned16(key) && aligned16(value) && aligned16(key_cache) &&
                    aligned16(value_cache),
                PKV_ERR_INVALID, "pkv_write_slots: pointers must be 16-byte aligned");
    DeviceGuard guard(stream, key_cache);
    const int64_t row_vecs = row / 8;
    const int64_t total = (int64_t)num_tokens * 2 * row_vecs;
    const int64_t num_slots = (int64_t)num_blocks * block_size;
    int64_t grid = (total + kThreads - 1) / kThreads;
    if (grid > 148 * 64) grid = 148 * 64;  // grid-stride beyond 64 CTAs per SM
    const auto* k = static_cast<const uint4*>(key);
    const auto* v = static_cast<const uint4*>(value);
    auto* kc = static_cast<uint4*>(key_cache);
    auto* vc = static_cast<uint4*>(value_cache);
    // 32-bit indexes: the vectors, the slots and the grid stride past the
    // last vector all below 2^31
    if (total + grid * kThreads < (int64_t(1) << 31) && num_slots < (int64_t(1) << 31))
        write_slots_kernel<uint32_t><<<(unsigned)grid, kThreads, 0, stream>>>(
            k, v, kc, vc, slot_mapping, num_tokens, num_slots, block_size, (uint32_t)row_vecs,
            block_stride / 8, dev_error);
    else
        write_slots_kernel<int64_t><<<(unsigned)grid, kThreads, 0, stream>>>(
            k, v, kc, vc, slot_mapping, num_tokens, num_slots, block_size, row_vecs,
            block_stride / 8, dev_error);
    return launch_status("pkv_write_slots");
}

// ---------------------------------------------------------------------------
// Slot write into FP8 (e4m3) caches with a float32 scale per (block, KV
// head): each value is stored as the e4m3 code nearest to x / scale
// (round to nearest even, saturating at 448) — the quantised layout of the
// "Paged KV" wiki page's 局限性 section ("KV FP8 with scaling per block").
// One thread per 8 values of one (token, KV head) row.
// ---------------------------------------------------------------------------
namespace pkv {
namespace {

template <typename T>
__global__ void __launch_bounds__(kThreads)
write_slots_fp8_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                       uint2* __restrict__ key_cache, uint2* __restrict__ value_cache,
                       const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                       const int64_t* __restrict__ slot_mapping, int num_tokens,
                       int64_t num_slots, int block_size, int num_kv_heads, int head_dim,
                       int64_t block_stride, int32_t* __restrict__ dev_error) {
    const int64_t row_vecs = (int64_t)num_kv_heads * head_dim / 8;  // 8 values per thread
    const int64_t per_token = 2 * row_vecs;
    const int64_t total = (int64_t)num_tokens * per_token;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_token;
        const int64_t r = i - t * per_token;
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (r == 0) report_error(dev_error, PKV_DEVERR_SLOT, (int)t);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        const bool is_v = r >= row_vecs;
        const int64_t v = is_v ? r - row_vecs : r;
        const int h = (int)(v * 8 / head_dim);
        const float sc = __ldg((is_v ? v_scale : k_scale) + blk * num_kv_heads + h);
        const uint4 x = __ldg((is_v ? value : key) + t * row_vecs + v);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint16_t q[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = Storage<T>::to_float2(w[j]);
            q[j] = f32x2_to_e4m3x2(__fdiv_rn(f.x, sc), __fdiv_rn(f.y, sc));
        }
        uint2 out;
        out.x = (uint32_t)q[0] | ((uint32_t)q[1] << 16);
        out.y = (uint32_t)q[2] | ((uint32_t)q[3] << 16);
        // 8 bytes per thread: block_stride and rows in bytes, /8 for uint2
        const int64_t dst = (blk * block_stride + off * (int64_t)num_kv_heads * head_dim) / 8 + v;
        (is_v ? value_cache : key_cache)[dst] = out;
    }
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_write_slots_fp8(const void* key, const void* value, void* key_cache,
                                   void* value_cache, const float* k_scale,
                                   const float* v_scale, const int64_t* slot_mapping,
                                   int num_tokens, int num_blocks, int block_size,
                                   int num_kv_heads, int head_dim, int64_t block_stride,
                                   pkv_dtype dtype, int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_write_slots_fp8");
    using namespace pkv;
    PKV_REQUIRE(dtype == PKV_F16 || dtype == PKV_BF16, PKV_ERR_UNSUPPORTED,
                "pkv_write_slots_fp8: dtype %d of the new rows", (int)dtype);
    PKV_REQUIRE(num_tokens >= 0 && num_blocks >= 0 && block_size > 0 && num_kv_heads > 0 &&
                    head_dim > 0 && head_dim % 8 == 0,
                PKV_ERR_INVALID, "pkv_write_slots_fp8: bad sizes");
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    PKV_REQUIRE(block_stride >= (int64_t)block_size * row && block_stride % 16 == 0,
                PKV_ERR_INVALID, "pkv_write_slots_fp8: block_stride %lld (bytes, multiple of 16)",
                (long long)block_stride);
    if (num_tokens == 0) return PKV_OK;
    PKV_REQUIRE(key && value && key_cache && value_cache && k_scale && v_scale && slot_mapping,
                PKV_ERR_INVALID, "pkv_write_slots_fp8: NULL pointer");
    PKV_REQUIRE(aligned16(key) && aligned16(value) && aligned16(key_cache) &&
                    aligned16(value_cache),
                PKV_ERR_INVALID, "pkv_write_slots_fp8: pointers must be 16-byte aligned");
    DeviceGuard guard(stream, key_cache);
    const int64_t total = (int64_t)num_tokens * 2 * (row / 8);
    int64_t grid = (total + kThreads - 1) / kThreads;
    if (grid > 148 * 64) grid = 148 * 64;
    if (dtype == PKV_BF16)
        write_slots_fp8_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, 0, stream>>>(
            static_cast<const uint4*>(key), static_cast<const uint4*>(value),
            static_cast<uint2*>(key_cache), static_cast<uint2*>(value_cache), k_scale, v_scale,
            slot_mapping, num_tokens, (int64_t)num_blocks * block_size, block_size,
            num_kv_heads, head_dim, block_stride, dev_error);
    else
        write_slots_fp8_kernel<__half><<<(unsigned)grid, kThreads, 0, stream>>>(
            static_cast<const uint4*>(key), static_cast<const uint4*>(value),
            static_cast<uint2*>(key_cache), static_cast<uint2*>(value_cache), k_scale, v_scale,
            slot_mapping, num_tokens, (int64_t)num_blocks * block_size, block_size,
            num_kv_heads, head_dim, block_stride, dev_error);
    return launch_status("pkv_write_slots_fp8");
}
