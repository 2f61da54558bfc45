// schedule.cu -- varlen tile scheduler: cu_seqlens -> list of (query tile, head) work items.
//
// Paired path: document boundaries and max_len are doubled ("modded-nanogpt Paired Head
// Attention record" page, section "sequence length and window handling") while the window stays
// as given. For each query tile of 128 slots [q0, q0+n) of a document [a, b) the key range is
//   causal:      [max(a, q0 - window + 1), q0 + n)   (window <= 0: from a)
//   non-causal:  [a, b)
// so key tiles that the causal mask or the window hide entirely are never scheduled. Key tiles
// start at the range's first slot (not at a multiple of 128): with a window of w the range of a
// full query tile is 127 + w slots wide, i.e. ceil((127 + w) / 128) key tiles.
//
// Items are ordered longest first (counting sort on the number of key tiles) so that a static
// round-robin over persistent CTAs balances; the heads of one query tile are adjacent so that
// CTAs sharing a kv head (GQA) run close together in time and share K/V through L2.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.cuh"

namespace pha {

constexpr int kSchedThreads = 1024;
constexpr int kSchedBuckets = 4096;  // cost classes; costs above the last share one class

__device__ __forceinline__ void tile_range(const AttnProblem& p, int64_t a, int64_t b, int64_t q0,
                                           int64_t& n_q, int64_t& kv_lo, int64_t& kv_hi) {
    n_q = b - q0 < kBlockM ? b - q0 : kBlockM;
    if (p.causal) {
        kv_hi = q0 + n_q;
        kv_lo = a;
        if (p.window > 0 && q0 - p.window + 1 > a) kv_lo = q0 - p.window + 1;
    } else {
        kv_lo = a;
        kv_hi = b;
    }
}

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(AttnProblem p, int capacity,
                                                                 int4* __restrict__ items,
                                                                 WorkspaceHeader* hdr) {
    __shared__ int hist[kSchedBuckets];
    __shared__ int bad;
    const int tid = threadIdx.x;
    for (int c = tid; c < kSchedBuckets; c += kSchedThreads) hist[c] = 0;
    if (tid == 0) bad = 0;
    __syncthreads();

    const int64_t mult = p.slot_mult;
    // validation + histogram of per-tile costs
    for (int d = tid; d < p.batch; d += kSchedThreads) {
        const int64_t a0 = p.cu_seqlens[d], b0 = p.cu_seqlens[d + 1];
        if (a0 < 0 || b0 < a0 || b0 > p.total_tokens || b0 - a0 > p.max_len) {
            atomicOr(&bad, 1);
            continue;
        }
        const int64_t a = a0 * mult, b = b0 * mult;
        for (int64_t q0 = a; q0 < b; q0 += kBlockM) {
            int64_t n_q, lo, hi;
            tile_range(p, a, b, q0, n_q, lo, hi);
            int64_t cost = (hi - lo + kBlockN - 1) / kBlockN;
            if (cost >= kSchedBuckets) cost = kSchedBuckets - 1;
            atomicAdd(&hist[cost], 1);
        }
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            hdr->n_items = 0;
            hdr->status = DEV_BAD_SEQLENS;
        }
        return;
    }
    // exclusive scan in descending cost order (one thread; 4096 entries)
    __shared__ int total_tiles;
    if (tid == 0) {
        int acc = 0;
        for (int c = kSchedBuckets - 1; c >= 0; --c) {
            const int n = hist[c];
            hist[c] = acc;
            acc += n;
        }
        total_tiles = acc;
    }
    __syncthreads();
    const int64_t n_items = static_cast<int64_t>(total_tiles) * p.heads;
    if (n_items > capacity) {
        if (tid == 0) {
            hdr->n_items = 0;
            hdr->status = DEV_OVERFLOW;
        }
        return;
    }
    for (int d = tid; d < p.batch; d += kSchedThreads) {
        const int64_t a = static_cast<int64_t>(p.cu_seqlens[d]) * mult;
        const int64_t b = static_cast<int64_t>(p.cu_seqlens[d + 1]) * mult;
        for (int64_t q0 = a; q0 < b; q0 += kBlockM) {
            int64_t n_q, lo, hi;
            tile_range(p, a, b, q0, n_q, lo, hi);
            int64_t cost = (hi - lo + kBlockN - 1) / kBlockN;
            if (cost >= kSchedBuckets) cost = kSchedBuckets - 1;
            const int slot = atomicAdd(&hist[cost], 1);
            for (int h = 0; h < p.heads; ++h)
                items[static_cast<int64_t>(slot) * p.heads + h] =
                    make_int4(static_cast<int>(q0), (h << 16) | static_cast<int>(n_q),
                              static_cast<int>(lo), static_cast<int>(hi));
        }
    }
    if (tid == 0) {
        hdr->n_items = static_cast<int>(n_items);
        hdr->status = DEV_OK;
    }
}

cudaError_t launch_schedule(const AttnProblem& p, int capacity, int4* items, WorkspaceHeader* hdr,
                            cudaStream_t stream) {
    schedule_kernel<<<1, kSchedThreads, 0, stream>>>(p, capacity, items, hdr);
    return cudaGetLastError();
}

}  // namespace pha
