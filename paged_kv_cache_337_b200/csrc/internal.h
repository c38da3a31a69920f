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

}  // namespace pkv

#define PKV_REQUIRE(cond, status, ...)              \
    do {                                            \
        if (!(cond)) return ::pkv::fail((status), __VA_ARGS__); \
    } while (0)
