// internal.h — host-side helpers shared by the library's translation units:
// the thread-local last-error message and argument-check macros.
#pragma once
#include <cstdarg>
#include <cstdint>

#include "pkv.h"

namespace pkv {

// Records a printf-style message for pkv_last_error() and returns `status`.
int fail(int status, const char* fmt, ...);
// Clears the calling thread's last-error message.
void clear_error();

// An NVTX range named after an entry point, open for the call's host-side
// duration (its launches show under it on a profiler's timeline).  Emitted
// only when the environment has PKV_NVTX=1; otherwise the constructor and
// destructor test one cached flag and do nothing else.
class NvtxRange {
  public:
    explicit NvtxRange(const char* name);
    ~NvtxRange();
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;

  private:
    bool on_;
};

// The partitions of a decode launch: the partition length actually used
// and the number of partitions of the grid.  One pass (the longest context
// rounded up to the 16-token tile) when partition_size is 0 or covers
// max_context_len.
inline void plan_partitions(int max_context_len, int partition_size, int* P, int* NP) {
    constexpr int kTile = 16;
    if (partition_size <= 0 || partition_size >= max_context_len) {
        const int ctx = max_context_len > 0 ? max_context_len : 1;
        *P = (ctx + kTile - 1) / kTile * kTile;
        *NP = 1;
    } else {
        *P = partition_size;
        *NP = (max_context_len + partition_size - 1) / partition_size;
    }
}

}  // namespace pkv

#define PKV_NVTX_RANGE(name) ::pkv::NvtxRange pkv_nvtx_range_(name)

#define PKV_REQUIRE(cond, status, ...)              \
    do {                                            \
        if (!(cond)) return ::pkv::fail((status), __VA_ARGS__); \
    } while (0)
