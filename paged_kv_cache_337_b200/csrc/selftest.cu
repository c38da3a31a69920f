// selftest.cu — a check of the kernels' failure path.  Every wait of the
// library's kernels on an mbarrier is bounded; when the limit runs out the
// kernel records PKV_DEVERR_TIMEOUT and returns instead of hanging.  This
// entry point runs that exact wait on a barrier nothing will ever complete,
// so a test can watch the limit expire and the error be reported, with the
// context left usable.  A second entry point applies the prefill softmax's
// FMA-pipe 2^x (ex2_poly2) to an array, so that a test can hold it to its
// error bound against the exact power of two.
#include "common.cuh"
#include "packed_f32.cuh"

namespace pkv {
namespace {

__global__ void bounded_wait_kernel(int32_t* dev_error, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none will come
        fence_barrier_init();
    }
    __syncthreads();
    if (!mbar_wait_bounded(&bar, 0, limit_ns) && threadIdx.x == 0)
        report_error(dev_error, PKV_DEVERR_TIMEOUT, 0);
}

// y[i] = ex2_poly2(x[i]), two elements per thread (an odd tail pairs with 0)
__global__ void ex2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const bool two = i + 1 < n;
    const float2 r = ex2_poly2(make_float2(x[i], two ? x[i + 1] : 0.f));
    y[i] = r.x;
    if (two) y[i + 1] = r.y;
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_selftest_bounded_wait(int32_t* dev_error, int limit_us, cudaStream_t stream) {
    using namespace pkv;
    PKV_REQUIRE(dev_error != nullptr && aligned16(dev_error), PKV_ERR_INVALID,
                "pkv_selftest_bounded_wait: dev_error must be a 16-byte aligned device pointer");
    PKV_REQUIRE(limit_us > 0 && limit_us <= 1000000, PKV_ERR_INVALID,
                "pkv_selftest_bounded_wait: limit %d us (1 .. 1000000)", limit_us);
    DeviceGuard guard(stream, dev_error);
    bounded_wait_kernel<<<1, 32, 0, stream>>>(dev_error, (uint64_t)limit_us * 1000ull);
    return launch_status("pkv_selftest_bounded_wait");
}

extern "C" int pkv_selftest_ex2_poly(const float* x, float* y, int n, cudaStream_t stream) {
    using namespace pkv;
    PKV_REQUIRE(n >= 0 && n <= (1 << 28), PKV_ERR_INVALID,
                "pkv_selftest_ex2_poly: n = %d (0 .. 2^28)", n);
    if (n == 0) return PKV_OK;
    PKV_REQUIRE(x != nullptr && y != nullptr, PKV_ERR_INVALID,
                "pkv_selftest_ex2_poly: null pointer");
    DeviceGuard guard(stream, y);
    constexpr int kThreads = 256;
    const int pairs = (n + 1) / 2;
    ex2_poly_kernel<<<(unsigned)((pairs + kThreads - 1) / kThreads), kThreads, 0, stream>>>(x, y,
                                                                                          n);
    return launch_status("pkv_selftest_ex2_poly");
}
