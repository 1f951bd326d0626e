// kvq_decode_attention_noalloc: the decode step with library-owned scratch.
//
// kvq_decode_attention needs a caller-owned workspace (per-split softmax states and
// the query sketches).  Some callers cannot provide one: code embedded in a host
// engine whose device memory is entirely reserved up front by that engine's own
// allocator, or code on a latency-critical path where a device allocation (which can
// synchronise the device) is not acceptable, and which has no spare buffer to lend.
// For them this entry point runs the same kernels with a fixed scratch area that
// lives in the library's own device image: a file-scope __device__ array, created when
// the library's module is loaded on a GPU and kept by every GPU that loads it until
// the process exits.  Nothing here calls cudaMalloc, cudaFree or any allocating
// routine.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>

#include "kvq.h"

#define KVQ_API extern "C" __attribute__((visibility("default")))

namespace {

// The largest workspace this entry point can serve.  The 7B-shaped and long-context
// GQA decode steps need about 0.23 MB and 1.2 MB.
constexpr size_t kScratchBytes = (size_t)8 << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  In host code the name
// g_decode_scratch only stands for the symbol; its device address has to be looked up
// once per device, with that device current.
kvq_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return KVQ_ERR_CUDA;
    if (dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
            return KVQ_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KVQ_OK;
}

}  // namespace

KVQ_API size_t kvq_decode_noalloc_max_workspace_bytes(void) { return kScratchBytes; }

KVQ_API kvq_status kvq_decode_attention_noalloc(const kvq_decode_args* a, kvq_stream_t stream) {
    if (!a) return KVQ_ERR_INVALID_ARG;
    kvq_decode_args local = *a;
    local.workspace = nullptr;
    local.workspace_bytes = 0;
    const size_t need = kvq_decode_workspace_bytes(&local);
    if (need > kScratchBytes) return KVQ_ERR_WORKSPACE;  // larger than the built-in scratch
    void* scratch = nullptr;
    if (need > 0) {
        const kvq_status st = scratch_for_current_device(&scratch);
        if (st != KVQ_OK) return st;
    }
    local.workspace = scratch;
    local.workspace_bytes = kScratchBytes;
    return kvq_decode_attention(&local, stream);
}
