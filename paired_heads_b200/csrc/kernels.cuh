// kernels.cuh -- launchers shared between the kernel files and the C-ABI layer (pha_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace pha {

constexpr int kBlockM = 128;         // query rows per sub-tile (one softmax warpgroup)
constexpr int kBlockN = 128;         // key slots per tile
constexpr int kItemRows = 2 * kBlockM;  // query slots per block work item (attn_tc)
constexpr int kBandTiles = 8;            // query tiles per band work item (attn_band)
constexpr int kBandRows = kBandTiles * kBlockM;
static_assert(kBandRows >= kItemRows, "band items must not outnumber block items");
constexpr int kMaxCostBuckets = 4096;   // scheduler cost classes (longest-first ordering)

// Workspace: header (bytes [0, 256)), per-document scratch (int32[batch + 1], padded to 16
// bytes), then int4 work items.
// Work-list cache: after a build the scheduler leaves a copy of cu_seqlens in the per-document
// scratch and records in the header what else the list depends on (key) and a checksum of the
// items; a later call whose inputs and items match reuses the list instead of rebuilding it.
struct WorkspaceHeader {
    int n_items;
    int status;
    uint32_t magic;     // kScheduleMagic while the fields below describe a valid list
    int key[10];        // mode, batch, max_len, total_tokens, slot_mult, heads, causal, window,
                        // capacity, n_buckets
    uint32_t checksum;  // of the items, in order
    int reused;         // 1 when the last scheduler call kept the list (read by tests)
};
constexpr uint32_t kScheduleMagic = 0x50484153u;
static_assert(sizeof(WorkspaceHeader) <= 256, "the header must fit its 256 bytes");
constexpr size_t kWorkspaceHeaderBytes = 256;

inline size_t workspace_doc_bytes(int batch) {
    return (static_cast<size_t>(batch + 1) * sizeof(int) + 15) & ~static_cast<size_t>(15);
}

// Block work item (attn_tc) = one block of up to kItemRows query slots of one head:
//   x = first query slot, y = (head << 16) | valid query rows, z = first key slot, w = key end.
// Keys [z, w) are streamed in tiles of kBlockN starting at z.
// Band work item (attn_band) = a run of up to kBandTiles query tiles of one head:
//   x = first query slot q0, y = (head << 16) | (has_prev << 15) | query tiles, z = document end,
//   w = document start. Key tiles start at q0 - kBlockN (has_prev) or q0, one per step.
// Tile work item (the tensor-core backward outside the band case): the band item format with a
// single tile, the 128-slot tile at q0 of one head of a document [w, z).

// Work-list shapes of the scheduler: block items (attn_tc), band items (attn_band and the band
// backward), and tile items ordered by the number of key tiles a query tile sees (dQ) or of query
// tiles that see a key tile (dK / dV).
enum ScheduleMode : int { kSchedBlock = 0, kSchedBand = 1, kSchedTilesQ = 2, kSchedTilesK = 3 };

struct AttnProblem {
    const void* q;
    const void* k;
    const void* v;
    const int32_t* cu_seqlens;  // tokens, not doubled
    int batch;
    int max_len;          // tokens
    int total_tokens;
    int slot_mult;        // 2 when paired (slots = 2 * tokens), else 1
    int heads;            // H' (heads of the slot view)
    int kv_heads;         // Hkv'
    int head_dim;
    int causal;
    int window;
    float scale;
    void* o;
    float* lse;
    // Value embedding (pha_attn_fwd_aux_v): added to v, with v's layout, before attention;
    // nullptr: none.
    const void* v_aux;
    // Failure-detection test hook (band kernel): > 0 makes the softmax warps first wait up to this
    // many microseconds on a barrier that nothing signals; 0 in every normal call.
    int test_stall_us;
    // FP8 inputs (pha_attn_fwd_fp8): q, k, v hold e4m3 codes standing for qk / v scale times
    // their values; the block kernel folds qk_scale (= q_scale * k_scale) into the logit scale
    // and v_scale into the epilogue. 1 / 1 otherwise.
    float qk_scale;
    float v_scale;
};

cudaError_t launch_rope_tables(float* cos_tab, float* sin_tab, int rows, int head_dim, int paired,
                               double base, cudaStream_t stream);

// Factored rotary tables: kRopeLoRows fine rows and rope_hi_rows(rows) coarse rows of float64
// (cos, sin) pairs (layout in rope.cu).
constexpr int kRopeLoRows = 16;
__host__ __device__ inline int rope_hi_rows(int rows) {
    return (rows + kRopeLoRows - 1) / kRopeLoRows;
}
inline size_t rope_factor_bytes(int rows, int head_dim, int paired) {
    const size_t a_width = paired ? head_dim : head_dim / 2;
    return (static_cast<size_t>(kRopeLoRows) * a_width +
            static_cast<size_t>(rope_hi_rows(rows)) * (head_dim / 2)) * 2 * sizeof(double);
}
cudaError_t launch_rope_factor_tables(double2* fac, int rows, int head_dim, int paired, double base,
                                      cudaStream_t stream);

// RoPE (norm: QK RMS-norm first; neg: the backward, rotation by -angle) with factored tables.
cudaError_t launch_rope_factored(void* q, void* k, const double2* fac, int rows,
                                 const int32_t* positions, int total_tokens, int n_heads,
                                 int n_kv_heads, int head_dim, int is_bf16, int paired,
                                 int stagger_offset, bool norm, bool neg, const float* q_weight,
                                 const float* k_weight, float eps, cudaStream_t stream);

cudaError_t launch_rope(void* q, void* k, const float* cos_tab, const float* sin_tab, int tab_rows,
                        int tab_width, const int32_t* positions, int total_tokens, int n_heads,
                        int n_kv_heads, int head_dim, int is_bf16, int paired, int stagger_offset,
                        cudaStream_t stream);

// Backward of RoPE: the rotation by -angle, in place on the gradients of q and k.
cudaError_t launch_rope_bwd(void* dq, void* dk, const float* cos_tab, const float* sin_tab,
                            int tab_rows, int tab_width, const int32_t* positions, int total_tokens,
                            int n_heads, int n_kv_heads, int head_dim, int is_bf16, int paired,
                            int stagger_offset, cudaStream_t stream);

// Backward of attention, D_i = dO_i . O_i into dsum (float[slots][heads]), from the forward's
// output o and the upstream gradient dout (both laid out like q).
cudaError_t launch_attn_bwd_dsum(const AttnProblem& p, const void* o, const void* dout,
                                 float* dsum, int is_bf16, cudaStream_t stream);

// Backward of attention on CUDA cores (any shape): dq, dk, dv (same layouts and dtype as q, k, v)
// for dout, from D in dsum. Needs p.lse. Rows outside every document get zeros.
cudaError_t launch_attn_bwd(const AttnProblem& p, const void* dout, const float* dsum, void* dq,
                            void* dk, void* dv, int is_bf16, cudaStream_t stream);

// Zeros the rows of dq, dk, dv (bf16) outside every document.
cudaError_t launch_attn_bwd_zero_outside(const AttnProblem& p, void* dq, void* dk, void* dv,
                                         cudaStream_t stream);

// Backward of attention on the tensor cores (bf16, head_dim 64 / 128). tm_do is a map over dout
// like tm_q; tm_dq a map over dq like tm_q with a 64 x 32 box, tm_dk / tm_dv maps over dk / dv
// like tm_k with a 64 x 16 box (the epilogues' TMA stores). Writes the rows inside the documents
// only. which: 1 = the dQ kernel, 2 = the dK / dV kernel, 3 = both. Band case (band_applies):
// band work list; otherwise tile work lists (kSchedTilesQ for dQ, kSchedTilesK for dK / dV).
cudaError_t launch_attn_bwd_tc(const AttnProblem& p, const CUtensorMap& tm_q,
                               const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                               const CUtensorMap& tm_do, const CUtensorMap& tm_dq,
                               const CUtensorMap& tm_dk, const CUtensorMap& tm_dv,
                               const float* dsum, void* dq, void* dk, void* dv, const int4* items,
                               WorkspaceHeader* hdr, int which, cudaStream_t stream);

// RoPE preceded by the QK RMS-norm of every head row (weights may be NULL = ones).
cudaError_t launch_qk_norm_rope(void* q, void* k, const float* q_weight, const float* k_weight,
                                float eps, const float* cos_tab, const float* sin_tab,
                                int tab_rows, int tab_width, const int32_t* positions,
                                int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                                int is_bf16, int paired, int stagger_offset, cudaStream_t stream);

cudaError_t launch_attn_f32(const AttnProblem& p, cudaStream_t stream);

// Builds the varlen work list of the given shape into `items` (capacity entries) and the header;
// doc_blocks is int32[batch + 1] scratch.
cudaError_t launch_schedule(const AttnProblem& p, ScheduleMode mode, int capacity, int* doc_blocks,
                            int4* items, WorkspaceHeader* hdr, cudaStream_t stream);

// tcgen05 attention over a scheduled work list. tm_q / tm_k / tm_v are 2-D bf16 tensor maps
// over the slot view ([slots][heads * head_dim] and [slots][kv_heads * head_dim]) with a
// 64 x 128 box and 128-byte swizzle.
// fp8: q, k, v are e4m3; tm_q / tm_k are 2-D uint8 maps with a head_dim x 128 box (128-byte
// swizzle at head_dim 128, 64-byte at 64) and tm_v the same box without swizzle.
cudaError_t launch_attn_tc(const AttnProblem& p, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, const int4* items, WorkspaceHeader* hdr,
                           cudaStream_t stream, bool fp8 = false);

// True when the band kernel covers the problem: causal, 1 <= window <= kBlockN.
inline bool band_applies(const AttnProblem& p) {
    return p.causal && p.window >= 1 && p.window <= kBlockN;
}

// tcgen05 attention over a band work list (same tensor maps as launch_attn_tc, plus tm_o: a map
// over o like tm_q but with a 64 x 32 box, for the epilogue's stores).
cudaError_t launch_attn_band(const AttnProblem& p, const CUtensorMap& tm_q,
                             const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_o, const int4* items, WorkspaceHeader* hdr,
                             cudaStream_t stream);

}  // namespace pha
