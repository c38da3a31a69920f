// status.cpp — status strings, the thread-local last-error message, sizing.
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"

namespace pkv {

static thread_local char g_last_error[512] = "";

int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return status;
}

void clear_error() { g_last_error[0] = '\0'; }

static bool nvtx_enabled() {
    static const bool on = [] {
        const char* v = std::getenv("PKV_NVTX");
        return v != nullptr && std::strcmp(v, "1") == 0;
    }();
    return on;
}

NvtxRange::NvtxRange(const char* name) : on_(nvtx_enabled()) {
    if (on_) nvtxRangePushA(name);
}

NvtxRange::~NvtxRange() {
    if (on_) nvtxRangePop();
}

}  // namespace pkv

extern "C" const char* pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
        case PKV_ERR_CUDA: return "CUDA error";
        case PKV_ERR_OOM: return "block pool exhausted";
        case PKV_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

extern "C" const char* pkv_last_error(void) { return pkv::g_last_error; }

extern "C" int pkv_version(void) { return 100; }

// Bytes of one physical block: [block_size, num_kv_heads, head_dim] for K and
// for V, for every layer ("Paged KV" wiki page, 初始化阶段).
extern "C" int64_t pkv_block_bytes(int block_size, int num_kv_heads,
                                   int head_dim, int num_layers,
                                   int dtype_bytes) {
    if (block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_layers <= 0 || dtype_bytes <= 0)
        return pkv::fail(PKV_ERR_INVALID, "pkv_block_bytes: sizes must be positive");
    return (int64_t)block_size * num_kv_heads * head_dim * 2 * num_layers *
           dtype_bytes;
}
