// schedule.cu -- varlen tile scheduler: cu_seqlens -> list of (query block, head) work items.
//
// Paired path: document boundaries and max_len are doubled ("modded-nanogpt Paired Head
// Attention record" page, section "sequence length and window handling") while the window stays
// as given. Two item shapes, one per attention kernel:
//
// Block items (attn_tc.cu): a block of up to kItemRows = 256 query slots [q0, q0+n) of one
// document [a, b) and one head; its key range is
//   causal:      [max(a, q0 - window + 1), q0 + n)   (window <= 0: from a)
//   non-causal:  [a, b)
// so key tiles that the causal mask or the window hide from the whole block are never scheduled
// (the attention kernel further skips, per 128-row half of the block, the tiles that half cannot
// see). Key tiles start at the range's first slot, not at a multiple of 128.
//
// Band items (attn_band.cu, causal with 1 <= window <= 128): a run of up to kBandTiles query
// tiles of 128 slots, tile u = [q0 + 128u, q0 + 128u + 128) of one document and one head, tiles
// counted from the document start. Such a query tile sees at most the key tile at its own start
// and the one before it, so the run streams key tiles from q0 - 128 (q0 - 128 >= a, "has
// previous") or q0, one per step, each shared by two consecutive query tiles.
//
// Tile items (the tensor-core backward outside the band case): one 128-slot tile of one document
// and head, with the document's start; dQ lists are ordered by the key tiles the query tile sees,
// dK / dV lists by the query tiles that see the key tile.
//
// Items are ordered longest first (counting sort on the number of key tiles) so that a static
// round-robin over persistent CTAs balances; the heads of one block are adjacent so that CTAs
// sharing a kv head (GQA) run close together in time and share K/V through L2.
//
// One CTA of 1024 threads: (1) per-document validation and block counts, (2) an exclusive scan
// over documents, (3) a cost histogram over all blocks, (4) a scan of the histogram in descending
// cost order, (5) emission, one thread per block. Before that, (0): when the workspace holds the
// list of an earlier call with the same inputs (header key, the copy of cu_seqlens kept in the
// per-document scratch, and the items' checksum all match) the kernel keeps it and returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.cuh"

namespace pha {

constexpr int kSchedThreads = 1024;

// Exclusive scan of one value per thread across the CTA; returns the thread's prefix and writes
// the total to *total. Needs kSchedThreads / 32 ints of shared scratch.
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < kSchedThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        warp_sums[lane] = s;  // inclusive prefix of warp totals
    }
    __syncthreads();
    const int before = warp > 0 ? warp_sums[warp - 1] : 0;
    const int t = warp_sums[kSchedThreads / 32 - 1];
    __syncthreads();  // warp_sums may be reused by the caller's next scan
    *total = t;
    return before + x - v;
}

// Checksum term of work item i (a multiply-xorshift mix of its words and index); the list's
// checksum is the XOR over its items.
__device__ __forceinline__ uint32_t item_hash(int4 it, uint32_t i) {
    uint32_t a = static_cast<uint32_t>(it.x) ^ (i * 0x85EBCA6Bu);
    a = a * 0x9E3779B1u + static_cast<uint32_t>(it.y);
    a ^= a >> 15;
    a = a * 0xC2B2AE35u + static_cast<uint32_t>(it.z);
    a ^= a >> 13;
    a = a * 0x27D4EB2Fu + static_cast<uint32_t>(it.w);
    a ^= a >> 16;
    return a;
}

// XOR of item_hash over items [0, n), across the CTA (every thread gets it).
__device__ uint32_t items_checksum(const int4* items, int n, uint32_t* warp_x) {
    uint32_t x = 0;
    for (int i = threadIdx.x; i < n; i += kSchedThreads) x ^= item_hash(items[i], static_cast<uint32_t>(i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x ^= __shfl_xor_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0) warp_x[threadIdx.x >> 5] = x;
    __syncthreads();
    uint32_t t = 0;
#pragma unroll 8
    for (int w = 0; w < kSchedThreads / 32; ++w) t ^= warp_x[w];
    __syncthreads();
    return t;
}

struct BlockRange {
    int4 item;  // the encoded work item (head field left 0)
    int cost;   // key tiles streamed, clamped to the last bucket
};

__device__ __forceinline__ int mode_rows(int mode) {
    return mode == kSchedBlock ? kItemRows : (mode == kSchedBand ? kBandRows : kBlockM);
}

__device__ __forceinline__ BlockRange block_range(const AttnProblem& p, int64_t a, int64_t b,
                                                  int blk, int n_buckets, int mode) {
    BlockRange r;
    const int rows = mode_rows(mode);
    const int64_t q0 = a + static_cast<int64_t>(blk) * rows;
    const int64_t n_q = b - q0 < rows ? b - q0 : rows;
    int64_t cost;
    if (mode == kSchedTilesQ || mode == kSchedTilesK) {
        // tile j = blk of the document's 128-slot tiles
        const int64_t last = (b - a - 1) / kBlockN;  // index of the document's last tile
        int64_t lo = 0, hi = last;
        if (mode == kSchedTilesQ) {  // key tiles this query tile sees
            if (p.causal) {
                hi = blk;
                if (p.window > 0 && q0 - p.window + 1 > a) lo = (q0 - p.window + 1 - a) / kBlockN;
            }
        } else if (p.causal) {       // query tiles that see this key tile
            lo = blk;
            if (p.window > 0) {
                // the last query that sees a key of this tile, inside the document
                const int64_t q_last = q0 + n_q - 1 + p.window - 1;
                hi = ((q_last < b ? q_last : b - 1) - a) / kBlockN;
            }
        }
        cost = hi - lo + 1;
        r.item = make_int4(static_cast<int>(q0), ((blk > 0 ? 1 : 0) << 15) | 1, static_cast<int>(b),
                           static_cast<int>(a));
    } else if (mode == kSchedBand) {
        const int n_qt = static_cast<int>((n_q + kBlockM - 1) / kBlockM);
        const int hp = blk > 0 ? 1 : 0;
        cost = n_qt + hp;
        r.item = make_int4(static_cast<int>(q0), (hp << 15) | n_qt, static_cast<int>(b),
                           static_cast<int>(a));
    } else {
        int64_t lo = a, hi = b;
        if (p.causal) {
            hi = q0 + n_q;
            if (p.window > 0 && q0 - p.window + 1 > a) lo = q0 - p.window + 1;
        }
        cost = (hi - lo + kBlockN - 1) / kBlockN;
        r.item = make_int4(static_cast<int>(q0), static_cast<int>(n_q), static_cast<int>(lo),
                           static_cast<int>(hi));
    }
    r.cost = static_cast<int>(cost >= n_buckets ? n_buckets - 1 : cost);
    return r;
}

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(AttnProblem p, int capacity,
                                                                 int n_buckets, int mode,
                                                                 int* __restrict__ doc_blocks,
                                                                 int4* __restrict__ items,
                                                                 WorkspaceHeader* hdr) {
    __shared__ int hist[kMaxCostBuckets];
    __shared__ int warp_sums[kSchedThreads / 32];
    __shared__ int bad;
    __shared__ int same;
    // the attention kernel may start its prologue (barriers, tensor memory, descriptor prefetch)
    // now; it waits for this grid's completion before it reads the work list
    grid_dep_launch();
    const int tid = threadIdx.x;
    const int64_t mult = p.slot_mult;
    const int rows = mode_rows(mode);
    const int key[10] = {mode, p.batch, p.max_len, p.total_tokens, p.slot_mult, p.heads,
                         p.causal, p.window, capacity, n_buckets};

    // (0) the list of an earlier call with the same inputs is kept
    if (tid == 0) {
        int ok = hdr->magic == kScheduleMagic && hdr->status == DEV_OK && hdr->n_items >= 0 &&
                 hdr->n_items <= capacity;
        for (int j = 0; j < 10; ++j) ok &= hdr->key[j] == key[j];
        same = ok;
    }
    __syncthreads();
    if (same) {
        for (int d = tid; d <= p.batch; d += kSchedThreads)
            if (p.cu_seqlens[d] != doc_blocks[d]) same = 0;
        const uint32_t sum = items_checksum(items, hdr->n_items, reinterpret_cast<uint32_t*>(warp_sums));
        if (sum != hdr->checksum) same = 0;  // (every thread computes the same sum)
        __syncthreads();
        if (same) {
            if (tid == 0) hdr->reused = 1;
            return;
        }
    }
    if (tid == 0) {
        hdr->magic = 0;
        hdr->reused = 0;
    }
    for (int c = tid; c < n_buckets; c += kSchedThreads) hist[c] = 0;
    if (tid == 0) bad = 0;
    __syncthreads();

    // (1) validation and blocks per document
    for (int d = tid; d < p.batch; d += kSchedThreads) {
        const int64_t a0 = p.cu_seqlens[d], b0 = p.cu_seqlens[d + 1];
        int nb = 0;
        if (a0 < 0 || b0 < a0 || b0 > p.total_tokens || b0 - a0 > p.max_len)
            atomicOr(&bad, 1);
        else
            nb = static_cast<int>(((b0 - a0) * mult + rows - 1) / rows);
        doc_blocks[d] = nb;
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            hdr->n_items = 0;
            hdr->status = DEV_BAD_SEQLENS;
        }
        return;
    }
    // (2) exclusive scan over documents (in place, chunks of kSchedThreads)
    int carry = 0;
    for (int base = 0; base < p.batch; base += kSchedThreads) {
        const int d = base + tid;
        const int v = d < p.batch ? doc_blocks[d] : 0;
        int total;
        const int ex = block_exclusive_scan(v, warp_sums, &total);
        if (d < p.batch) doc_blocks[d] = carry + ex;
        carry += total;
        __syncthreads();
    }
    const int n_blocks = carry;
    if (tid == 0) doc_blocks[p.batch] = n_blocks;
    __syncthreads();
    const int64_t n_items = static_cast<int64_t>(n_blocks) * p.heads;
    if (n_items > capacity) {
        if (tid == 0) {
            hdr->n_items = 0;
            hdr->status = DEV_OVERFLOW;
        }
        return;
    }

    auto doc_of = [&](int g) {  // last d with doc_blocks[d] <= g (skips empty documents)
        int lo = 0, hi = p.batch;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (doc_blocks[mid] <= g) lo = mid; else hi = mid;
        }
        return lo;
    };
    // (3) cost histogram
    for (int g = tid; g < n_blocks; g += kSchedThreads) {
        const int d = doc_of(g);
        const BlockRange r = block_range(p, p.cu_seqlens[d] * mult, p.cu_seqlens[d + 1] * mult,
                                         g - doc_blocks[d], n_buckets, mode);
        atomicAdd(&hist[r.cost], 1);
    }
    __syncthreads();
    // (4) exclusive scan in descending cost order: bucket c starts after all costlier buckets
    carry = 0;
    for (int base = 0; base < n_buckets; base += kSchedThreads) {
        const int c = n_buckets - 1 - (base + tid);
        const int v = c >= 0 ? hist[c] : 0;
        int total;
        const int ex = block_exclusive_scan(v, warp_sums, &total);
        if (c >= 0) hist[c] = carry + ex;
        carry += total;
        __syncthreads();
    }
    // (5) emission
    for (int g = tid; g < n_blocks; g += kSchedThreads) {
        const int d = doc_of(g);
        const BlockRange r = block_range(p, p.cu_seqlens[d] * mult, p.cu_seqlens[d + 1] * mult,
                                         g - doc_blocks[d], n_buckets, mode);
        const int slot = atomicAdd(&hist[r.cost], 1);
        int4* dst = items + static_cast<int64_t>(slot) * p.heads;
        for (int h = 0; h < p.heads; ++h)
            dst[h] = make_int4(r.item.x, (h << 16) | r.item.y, r.item.z, r.item.w);
    }
    // the cache record: the copy of cu_seqlens replaces the per-document scratch, then the key,
    // the items' checksum and the magic
    __syncthreads();
    for (int d = tid; d <= p.batch; d += kSchedThreads) doc_blocks[d] = p.cu_seqlens[d];
    const uint32_t sum = items_checksum(items, static_cast<int>(n_items),
                                        reinterpret_cast<uint32_t*>(warp_sums));
    if (tid == 0) {
        hdr->n_items = static_cast<int>(n_items);
        hdr->status = DEV_OK;
        for (int j = 0; j < 10; ++j) hdr->key[j] = key[j];
        hdr->checksum = sum;
        __threadfence_block();
        hdr->magic = kScheduleMagic;
    }
}

int schedule_buckets(const AttnProblem& p, int mode) {
    if (mode == kSchedBand) return kBandTiles + 2;
    if (mode == kSchedTilesQ || mode == kSchedTilesK) {
        const int64_t tiles = (static_cast<int64_t>(p.max_len) * p.slot_mult + kBlockN - 1) / kBlockN + 2;
        return static_cast<int>(tiles < kMaxCostBuckets ? tiles : kMaxCostBuckets);
    }
    const int64_t slots = static_cast<int64_t>(p.max_len) * p.slot_mult;
    const int64_t nb = (slots + kItemRows) / kBlockN + 2;
    return static_cast<int>(nb < kMaxCostBuckets ? nb : kMaxCostBuckets);
}

cudaError_t launch_schedule(const AttnProblem& p, ScheduleMode mode, int capacity, int* doc_blocks,
                            int4* items, WorkspaceHeader* hdr, cudaStream_t stream) {
    schedule_kernel<<<1, kSchedThreads, 0, stream>>>(p, capacity, schedule_buckets(p, mode),
                                                     static_cast<int>(mode), doc_blocks, items, hdr);
    return cudaGetLastError();
}

}  // namespace pha
