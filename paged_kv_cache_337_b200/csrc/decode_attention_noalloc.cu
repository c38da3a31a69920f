// decode_attention_noalloc.cu — pkv_decode_attention for callers that cannot
// allocate device memory (a host framework that owns the whole device and
// forbids plug-ins from calling cudaMalloc, a loop that must not pay for an
// allocation).  The split-K scratch is a device array built into the
// library instead of a caller-provided workspace; everything else is the
// ordinary entry point.  This file holds the array, the per-device lookup of
// its address and the entry point, and nothing else.  With lazy module
// loading (CUDA's default) a device holds the array only once this entry
// point has run there; with CUDA_MODULE_LOADING=EAGER every context that
// loads the library holds it.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace pkv {
namespace {

// Shared by every call on a device; kept until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_workspace[PKV_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_lookup_mutex;
struct Lookup {
    CUcontext context;  // the context the address belongs to
    void* addr;         // device address of the array in it
};
Lookup g_lookup[kMaxDevices];

// The calling thread's current CUDA context, through the driver entry
// point the runtime exposes (no link against the driver library).
CUcontext current_context() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    });
    CUcontext ctx = nullptr;
    if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

// Device address of the array on `device`, which must be current.  In host
// code `g_noalloc_workspace` names a host-side stand-in, not device memory,
// so the address is looked up (cudaGetSymbolAddress) at the first call on
// the device and kept.  It is looked up again when the device's context is
// not the one it was found in (after cudaDeviceReset, the module and the
// array are loaded anew).
int workspace_address(int device, void** addr) {
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_lookup_mutex);
    Lookup& l = g_lookup[device];
    if (l.addr == nullptr || l.context != ctx) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
        if (e != cudaSuccess || p == nullptr)
            return fail(PKV_ERR_CUDA,
                        "pkv_decode_attention_noalloc: cudaGetSymbolAddress failed on device "
                        "%d: %s",
                        device, cudaGetErrorString(e));
        l.context = ctx;
        l.addr = p;
    }
    *addr = l.addr;
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_decode_attention_noalloc(void* out, const void* query, const void* key_cache,
                                            const void* value_cache,
                                            const int32_t* block_tables,
                                            int max_blocks_per_seq,
                                            const int32_t* context_lens, int num_seqs,
                                            int max_context_len, int num_q_heads,
                                            int num_kv_heads, int head_dim, int num_blocks,
                                            int block_size, int64_t block_stride, float scale,
                                            int partition_size, pkv_dtype dtype,
                                            int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_decode_attention_noalloc");
    using namespace pkv;
    const size_t need = pkv_decode_workspace_bytes(num_seqs, num_q_heads, max_context_len,
                                                   partition_size, head_dim);
    PKV_REQUIRE(need <= (size_t)PKV_NOALLOC_WORKSPACE_BYTES, PKV_ERR_WORKSPACE,
                "pkv_decode_attention_noalloc: these sizes need %zu bytes of split-K scratch, "
                "more than the %u built into the library; use a larger partition_size or "
                "pkv_decode_attention with a workspace",
                need, (unsigned)PKV_NOALLOC_WORKSPACE_BYTES);
    void* ws = nullptr;
    // any call with sequences finds the array (so a first, single-pass call
    // made before a stream capture has done the set-up for a later split-K
    // call inside it); the array is handed on only when partitions need it
    if (num_seqs > 0 && key_cache != nullptr) {
        DeviceGuard guard(stream, key_cache);
        int device = -1;
        cudaError_t e = cudaGetDevice(&device);
        if (e != cudaSuccess)
            return fail(PKV_ERR_CUDA, "pkv_decode_attention_noalloc: cudaGetDevice: %s",
                        cudaGetErrorString(e));
        PKV_REQUIRE(device >= 0 && device < kMaxDevices, PKV_ERR_UNSUPPORTED,
                    "pkv_decode_attention_noalloc: device %d", device);
        int st = workspace_address(device, &ws);
        if (st != PKV_OK) return st;
        if (need == 0) ws = nullptr;
    }
    return pkv_decode_attention(out, query, key_cache, value_cache, block_tables,
                                max_blocks_per_seq, context_lens, num_seqs, max_context_len,
                                num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                                block_stride, scale, partition_size, ws,
                                need > 0 ? (size_t)PKV_NOALLOC_WORKSPACE_BYTES : 0, dtype,
                                dev_error, stream);
}
