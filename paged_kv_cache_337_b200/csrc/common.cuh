// common.cuh — device-side building blocks for the sm_100a kernels:
// 16-bit storage traits, the device error record, bounded mbarrier waits,
// TMA tensor loads, ldmatrix / movmatrix / mma.sync wrappers, and the host
// guard that makes the stream's device current for a launch.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace pkv {

// ---------------------------------------------------------------------------
// storage types
// ---------------------------------------------------------------------------
template <typename T>
struct Storage;

template <>
struct Storage<__half> {
    static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    __device__ static __forceinline__ float2 to_float2(uint32_t w) {
        __half2 h;
        memcpy(&h, &w, 4);
        return __half22float2(h);
    }
    __device__ static __forceinline__ uint32_t from_float2(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);  // a -> low half
        uint32_t w;
        memcpy(&w, &h, 4);
        return w;
    }
    __device__ static __forceinline__ __half from_float(float a) { return __float2half_rn(a); }
};

template <>
struct Storage<__nv_bfloat16> {
    static constexpr CUtensorMapDataType kTmaType = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    __device__ static __forceinline__ float2 to_float2(uint32_t w) {
        // bf16 is the upper half of an fp32: widening is a shift
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    __device__ static __forceinline__ uint32_t from_float2(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // a -> low half
        uint32_t w;
        memcpy(&w, &h, 4);
        return w;
    }
    __device__ static __forceinline__ __nv_bfloat16 from_float(float a) {
        return __float2bfloat16_rn(a);
    }
};

// ---------------------------------------------------------------------------
// device error record {code, index}; first writer wins
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report_error(int32_t* err, int code, int index) {
    if (err != nullptr && atomicCAS(err, 0, code) == 0) {
        atomicExch(err + 1, index);
    }
}

// ---------------------------------------------------------------------------
// shared-memory addresses, mbarriers and TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Makes mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wall-clock limit of one bounded wait.  A TMA copy completes in
// microseconds; a wait this long means something is broken.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// Waits for the phase with the given parity to complete, for at most
// limit_ns nanoseconds.  Returns false when the limit ran out.  The elapsed
// time is a signed difference, so a global timer that steps back does not
// end the wait (it lengthens it by the step).  The loop is kept this short
// on purpose: waiting warps poll it, and every instruction it adds takes an
// issue slot from the warps that work.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((int64_t)(global_timer_ns() - t0) > (int64_t)limit_ns) return false;
    }
}

// 4-D tiled TMA load into shared memory, completing on `bar` (no multicast).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
        : "memory");
}

// 5-D tiled TMA load into shared memory, completing on `bar` (no multicast).
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3), "r"(c4)
        : "memory");
}

// L2 cache policies (createpolicy): evict_first for data read or written
// once, evict_last for data that later accesses re-read.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// tma_load_5d with an L2 cache policy for the bytes it reads.
__device__ __forceinline__ void tma_load_5d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int c0, int c1, int c2, int c3, int c4,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3), "r"(c4), "l"(policy)
        : "memory");
}

// 16-byte global store with an L2 cache policy.
__device__ __forceinline__ void st_global_v4_hint(void* dst, uint4 v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;"
                 ::"l"(reinterpret_cast<uint64_t>(dst)), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w),
                 "l"(policy)
                 : "memory");
}

// Untiled bulk copy of `bytes` (a multiple of 16) from global memory into
// shared memory, completing on `bar`; both addresses 16-byte aligned.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes),
        "r"(smem_addr(bar))
        : "memory");
}

// ---------------------------------------------------------------------------
// FP8 (e4m3) conversions, by the hardware cvt instructions
// ---------------------------------------------------------------------------
// Two e4m3 codes (low byte first) to two halves (low half first); exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t codes) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(codes));
    return r;
}

// Two floats to two e4m3 codes (lo in the low byte), round to nearest even,
// magnitudes beyond 448 saturating to 448.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}


__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// warp-level matrix helpers (16-bit operands, fp32 accumulators)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

// Two 16x16 matrices of bytes, transposed: lanes 0-15 give the 16 row
// addresses of the first, lanes 16-31 of the second.  Lane t receives, per
// matrix, rows 4(t%4) .. 4(t%4)+3 of column t/4 (one register, lowest row
// in the low byte) and of column t/4 + 8 (the next register).
__device__ __forceinline__ void ldmatrix_b8_x2_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

// Transposes an 8x8 matrix of 16-bit values held one row-pair per lane.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

template <typename T>
struct Mma;

template <>
struct Mma<__nv_bfloat16> {
    __device__ static __forceinline__ void m16n8k16(float (&c)[4], const uint32_t (&a)[4],
                                                    uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
            "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

template <>
struct Mma<__half> {
    __device__ static __forceinline__ void m16n8k16(float (&c)[4], const uint32_t (&a)[4],
                                                    uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
            "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

}  // namespace pkv

// ---------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------
namespace pkv {

// Makes the stream's device current for the lifetime of the guard, so that
// launches from a process driving several GPUs land where the caller's
// stream lives.
class DeviceGuard {
   public:
    // The device is the stream's; for the legacy default stream (NULL),
    // the device that holds `ptr`.
    DeviceGuard(cudaStream_t stream, const void* ptr) {
        int want = -1;
        if (cudaGetDevice(&prev_) != cudaSuccess) {
            prev_ = -1;
            return;
        }
        if (stream != nullptr) {
            if (cudaStreamGetDevice(stream, &want) != cudaSuccess) want = -1;
        } else if (ptr != nullptr) {
            cudaPointerAttributes a;
            if (cudaPointerGetAttributes(&a, ptr) == cudaSuccess && a.type == cudaMemoryTypeDevice)
                want = a.device;
            else
                cudaGetLastError();  // clear a non-sticky error from the query
        }
        if (want >= 0 && want != prev_ && cudaSetDevice(want) == cudaSuccess) switched_ = true;
    }
    ~DeviceGuard() {
        if (switched_) cudaSetDevice(prev_);
    }
    DeviceGuard(const DeviceGuard&) = delete;
    DeviceGuard& operator=(const DeviceGuard&) = delete;

   private:
    int prev_ = -1;
    bool switched_ = false;
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(PKV_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return PKV_OK;
}

}  // namespace pkv
