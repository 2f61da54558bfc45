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
#include <cuda.h>
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

// Per device: the CUDA context in which the address was looked up, and the address. A new
// context on the device (after cudaDeviceReset, or once the primary context has been released
// and created again) loads the module afresh, so the address is looked up again.
struct ScratchSlot {
    CUcontext ctx;
    void* addr;
};
std::mutex g_setup_mutex;
ScratchSlot g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn get_ctx_fn() {
    // Resolved through the runtime so that the library does not link libcuda directly.
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(fn);
}

// Device address of the scratch array in the calling thread's current device and context.
// The first call in a context resolves it (with that device current) and remembers it.
pha_status scratch_on_current_device(void** addr) {
    static CtxGetCurrentFn ctx_get = get_ctx_fn();
    if (!ctx_get) return PHA_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PHA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PHA_ERR_UNSUPPORTED;
    CUcontext ctx = nullptr;  // NULL while no context is current on this thread yet
    if (ctx_get(&ctx) != CUDA_SUCCESS) return PHA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchSlot& slot = g_scratch[dev];
    if (ctx == nullptr || slot.addr == nullptr || slot.ctx != ctx) {
        // the lookup makes the device's primary context current when none is
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return PHA_ERR_CUDA;
        if (ctx == nullptr && (ctx_get(&ctx) != CUDA_SUCCESS || ctx == nullptr))
            return PHA_ERR_CUDA;
        slot.ctx = ctx;
        slot.addr = p;
    }
    *addr = slot.addr;
    return PHA_OK;
}

}  // namespace

extern "C" pha_status pha_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                           const int32_t* cu_seqlens, int batch, int max_len,
                                           int total_tokens, int n_heads, int n_kv_heads,
                                           int head_dim, pha_dtype dtype, int causal, int window,
                                           int paired, float scale, void* o, float* lse,
                                           pha_stream_t stream) {
    void* scratch = nullptr;
    const pha_status st = scratch_on_current_device(&scratch);
    if (st != PHA_OK) return st;
    // pha_attn_fwd checks the arguments first, then rejects a work list larger than the array
    // with PHA_ERR_WORKSPACE, before any launch. Nothing in the scratch has to start at zero:
    // the scheduler kernel writes the header, the per-document offsets and every work item the
    // attention kernel then reads.
    return pha_attn_fwd(q, k, v, cu_seqlens, batch, max_len, total_tokens, n_heads, n_kv_heads,
                        head_dim, dtype, causal, window, paired, scale, o, lse, scratch,
                        kNoAllocScratchBytes, stream);
}
