// noalloc.cu -- pha_attn_fwd_noalloc: the attention forward with its scratch memory in a fixed
// array owned by the library, for callers that cannot allocate device memory.
//
// pha_attn_fwd needs a caller-provided workspace for the varlen work list. Some callers have no
// way to provide one: a plug-in that is handed only its input and output buffers by a host
// framework that owns all device memory, or latency-critical code that must not call
// cudaMalloc (which can synchronise the whole device). This entry point takes the same
// arguments minus the workspace and uses a file-scope device array instead.
//
// The array is kNoAllocScratchBytes (1 MiB) per GPU and is held by every GPU that loads the
// library until the process exits. Problems whose work list needs more than that are rejected.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pha.h"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(1) << 20;
constexpr int kMaxDevices = 64;

// In host code this name is only a stand-in for the symbol, not a device address; the address
// comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of g_noalloc_scratch per device, once set up

// Device address of the scratch array on the calling thread's current device. The first call
// on a device resolves it (with that device current) and remembers it.
pha_status scratch_on_current_device(void** addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PHA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PHA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return PHA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return PHA_OK;
}

}  // namespace

extern "C" pha_status pha_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                           const int32_t* cu_seqlens, int batch, int max_len,
                                           int total_tokens, int n_heads, int n_kv_heads,
                                           int head_dim, pha_dtype dtype, int causal, int window,
                                           int paired, float scale, void* o, float* lse,
                                           pha_stream_t stream) {
    if (dtype == PHA_BF16) {
        const size_t need = pha_attn_workspace_bytes(batch, max_len, n_heads, head_dim, paired);
        if (need == 0) return PHA_ERR_INVALID;
        if (need > kNoAllocScratchBytes) return PHA_ERR_WORKSPACE;  // beyond the built-in 1 MiB
    }
    void* scratch = nullptr;
    const pha_status st = scratch_on_current_device(&scratch);
    if (st != PHA_OK) return st;
    // Nothing in the scratch has to start at zero: the scheduler kernel writes the header, the
    // per-document offsets and every work item the attention kernel then reads.
    return pha_attn_fwd(q, k, v, cu_seqlens, batch, max_len, total_tokens, n_heads, n_kv_heads,
                        head_dim, dtype, causal, window, paired, scale, o, lse, scratch,
                        kNoAllocScratchBytes, stream);
}
