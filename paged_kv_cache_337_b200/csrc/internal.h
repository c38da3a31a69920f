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

}  // namespace pkv

#define PKV_NVTX_RANGE(name) ::pkv::NvtxRange pkv_nvtx_range_(name)

#define PKV_REQUIRE(cond, status, ...)              \
    do {                                            \
        if (!(cond)) return ::pkv::fail((status), __VA_ARGS__); \
    } while (0)
