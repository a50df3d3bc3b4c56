// la_prefill_noalloc: la_prefill for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: code running under an
// allocator-free runtime or a fixed memory budget that must not grow, hooks
// called from inside another library's memory manager, or hosts where the
// one-off cudaMalloc of a large buffer is not allowed on the serving path.
// This entry point needs no workspace argument: its scratch is one static
// device array of LA_NOALLOC_SCRATCH_BYTES, created with the module on every
// GPU that loads the library and kept until the process exits. The caller
// still owns q, k, v, o, cu_seqlens and init_state.
//
// The array's name in host code is only a host-side stand-in for the device
// symbol, not a device address, so it is never passed to a kernel. The first
// call on each device (with that device current) asks the runtime for the real
// device address once, with cudaGetSymbolAddress, and caches it; that first
// call should therefore happen before any stream capture. Every later call on
// the device reuses the cached address. Nothing here calls cudaMalloc,
// cudaFree or any allocating routine. Two limits follow from the cache: the
// scratch is the current device's copy, so the caller's stream must belong to
// the current device; and the cached address does not survive a
// cudaDeviceReset of that device, after which this entry point may not be
// called on it again.
//
// All calls on a device share the one array, which keeps whatever the last
// call left in it: la_prefill rebuilds every part of its workspace that must
// start from a known value (block table, flags) at the start of each call, so
// no clearing is needed here. Calls whose executions overlap on the GPU
// (different streams, or different host threads without ordering) race on the
// shared scratch and produce undefined results.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>

#include "lightning_attention.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array (set up once per device).
la_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return LA_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return LA_OK;
}

}  // namespace

extern "C" la_status la_prefill_noalloc(const void* q, const void* k, const void* v, void* o,
                                        const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens,
                                        int heads, int d, int B, la_dtype dtype, const float* init_state,
                                        void* stream) {
    const size_t need = la_prefill_workspace_size(total_tokens, num_seqs, heads, d, B, dtype);
    if (need == 0 || total_tokens == 0)   // unsupported or empty: la_prefill reports it without scratch
        return la_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state,
                          nullptr, 0, stream);
    if (need > (size_t)LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_WORKSPACE_TOO_SMALL;
    void* scratch = nullptr;
    const la_status s = scratch_address(&scratch);
    if (s != LA_OK) return s;
    return la_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state, scratch,
                      (size_t)LA_NOALLOC_SCRATCH_BYTES, stream);
}
