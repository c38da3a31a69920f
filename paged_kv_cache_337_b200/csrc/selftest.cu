// selftest.cu — a check of the kernels' failure path.  Every wait of the
// library's kernels on an mbarrier is bounded; when the limit runs out the
// kernel records PKV_DEVERR_TIMEOUT and returns instead of hanging.  This
// entry point runs that exact wait on a barrier nothing will ever complete,
// so a test can watch the limit expire and the error be reported, with the
// context left usable.
#include "common.cuh"

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
