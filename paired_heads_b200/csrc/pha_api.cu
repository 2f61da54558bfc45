// pha_api.cu -- the extern "C" boundary of libpha (declared in include/pha.h).
//
// Validates every argument before any launch, builds the TMA tensor maps for the slot view of
// the caller's buffers, and queues the kernels on the caller's stream. Allocates nothing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include "../../include/pha.h"
#include "kernels.cuh"

using namespace pha;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    // Resolved through the runtime so that the library does not link libcuda directly.
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// 2-D bf16 map over [rows][width] elements, box 64 x box_rows, 128-byte swizzle, zero fill
// outside.
bool encode_slot_map(CUtensorMap* map, const void* base, uint64_t width, uint64_t rows,
                     uint32_t box_rows = 128) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
    if (!encode) return false;
    cuuint64_t dims[2] = {width, rows};
    cuuint64_t strides[1] = {width * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D uint8 map over [rows][width] bytes for e4m3 tiles: box box_inner x 128, swizzled to match
// the box width (128-byte rows: 128-byte swizzle; 64-byte rows: 64-byte swizzle) or unswizzled.
bool encode_u8_map(CUtensorMap* map, const void* base, uint64_t width, uint64_t rows,
                   uint32_t box_inner, bool swizzle) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
    if (!encode) return false;
    cuuint64_t dims[2] = {width, rows};
    cuuint64_t strides[1] = {width};
    cuuint32_t box[2] = {box_inner, 128};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = !swizzle ? CU_TENSOR_MAP_SWIZZLE_NONE
                                  : box_inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                     : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int64_t div_up(int64_t a, int64_t b) { return (a + b - 1) / b; }

int64_t max_work_items(int batch, int max_len, int n_heads, int paired) {
    const int64_t slots = static_cast<int64_t>(max_len) * (paired ? 2 : 1);
    const int64_t heads = paired ? n_heads / 2 : n_heads;
    return static_cast<int64_t>(batch) * div_up(slots, kItemRows) * heads;
}

}  // namespace

extern "C" {

const char* pha_status_string(pha_status s) {
    switch (s) {
        case PHA_OK: return "ok";
        case PHA_ERR_INVALID: return "invalid argument";
        case PHA_ERR_UNSUPPORTED: return "unsupported configuration";
        case PHA_ERR_WORKSPACE: return "workspace missing or too small";
        case PHA_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

pha_status pha_rope_tables(float* cos_tab, float* sin_tab, int rows, int head_dim, int paired,
                           double base, pha_stream_t stream) {
    if (!cos_tab || !sin_tab || !aligned16(cos_tab) || !aligned16(sin_tab) || rows < 0 ||
        head_dim <= 0 || (head_dim & 1) || !(base > 0.0) || (paired != 0 && paired != 1))
        return PHA_ERR_INVALID;
    return launch_rope_tables(cos_tab, sin_tab, rows, head_dim, paired, base, stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

pha_status pha_rope(void* q, void* k, const float* cos_tab, const float* sin_tab, int tab_rows,
                    int tab_width, const int32_t* positions, int total_tokens, int n_heads,
                    int n_kv_heads, int head_dim, pha_dtype dtype, int paired, int stagger_offset,
                    pha_stream_t stream) {
    if (dtype != PHA_BF16 && dtype != PHA_F32) return PHA_ERR_INVALID;
    const int span = dtype == PHA_BF16 ? 16 : 8;
    if (tab_rows < 0 || total_tokens < 0 || n_heads <= 0 || n_kv_heads < 0 || head_dim <= 0 ||
        head_dim % span != 0 || (paired != 0 && paired != 1))
        return PHA_ERR_INVALID;
    // With no tokens there is nothing to read or write; the buffers may be empty (NULL).
    if (total_tokens > 0 &&
        (!q || !aligned16(q) || (n_kv_heads > 0 && (!k || !aligned16(k))) || !cos_tab ||
         !sin_tab || !aligned16(cos_tab) || !aligned16(sin_tab) || !positions))
        return PHA_ERR_INVALID;
    if (!paired && (tab_width != head_dim || stagger_offset != 0)) return PHA_ERR_INVALID;
    if (paired && (tab_width != 2 * head_dim ||
                   (stagger_offset != 0 && stagger_offset != head_dim)))
        return PHA_ERR_INVALID;
    if (total_tokens == 0) return PHA_OK;
    return launch_rope(q, k, cos_tab, sin_tab, tab_rows, tab_width, positions, total_tokens,
                       n_heads, n_kv_heads, head_dim, dtype == PHA_BF16, paired, stagger_offset,
                       stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

pha_status pha_qk_norm_rope(void* q, void* k, const float* q_weight, const float* k_weight,
                            float eps, const float* cos_tab, const float* sin_tab, int tab_rows,
                            int tab_width, const int32_t* positions, int total_tokens,
                            int n_heads, int n_kv_heads, int head_dim, pha_dtype dtype,
                            int paired, int stagger_offset, pha_stream_t stream) {
    if (dtype != PHA_BF16 && dtype != PHA_F32) return PHA_ERR_INVALID;
    const int span = dtype == PHA_BF16 ? 16 : 8;
    if (tab_rows < 0 || total_tokens < 0 || n_heads <= 0 || n_kv_heads < 0 || head_dim <= 0 ||
        head_dim % span != 0 || (paired != 0 && paired != 1) || !(eps >= 0.f) || !(eps < INFINITY))
        return PHA_ERR_INVALID;
    if (total_tokens > 0 &&
        (!q || !aligned16(q) || (n_kv_heads > 0 && (!k || !aligned16(k))) || !cos_tab ||
         !sin_tab || !aligned16(cos_tab) || !aligned16(sin_tab) || !positions))
        return PHA_ERR_INVALID;
    if ((q_weight && !aligned16(q_weight)) || (k_weight && !aligned16(k_weight)))
        return PHA_ERR_INVALID;
    if (!paired && (tab_width != head_dim || stagger_offset != 0)) return PHA_ERR_INVALID;
    if (paired && (tab_width != 2 * head_dim ||
                   (stagger_offset != 0 && stagger_offset != head_dim)))
        return PHA_ERR_INVALID;
    // the 16-byte chunks of one head row must sit on a power-of-two group of lanes of a warp
    const int cph = head_dim / (dtype == PHA_BF16 ? 8 : 4);
    if (32 % cph != 0) return PHA_ERR_UNSUPPORTED;
    if (total_tokens == 0) return PHA_OK;
    return launch_qk_norm_rope(q, k, q_weight, k_weight, eps, cos_tab, sin_tab, tab_rows, tab_width,
                               positions, total_tokens, n_heads, n_kv_heads, head_dim,
                               dtype == PHA_BF16, paired, stagger_offset, stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

pha_status pha_rope_bwd(void* dq, void* dk, const float* cos_tab, const float* sin_tab,
                        int tab_rows, int tab_width, const int32_t* positions, int total_tokens,
                        int n_heads, int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                        int stagger_offset, pha_stream_t stream) {
    // the same arguments and checks as pha_rope
    if (dtype != PHA_BF16 && dtype != PHA_F32) return PHA_ERR_INVALID;
    const int span = dtype == PHA_BF16 ? 16 : 8;
    if (tab_rows < 0 || total_tokens < 0 || n_heads <= 0 || n_kv_heads < 0 || head_dim <= 0 ||
        head_dim % span != 0 || (paired != 0 && paired != 1))
        return PHA_ERR_INVALID;
    if (total_tokens > 0 &&
        (!dq || !aligned16(dq) || (n_kv_heads > 0 && (!dk || !aligned16(dk))) || !cos_tab ||
         !sin_tab || !aligned16(cos_tab) || !aligned16(sin_tab) || !positions))
        return PHA_ERR_INVALID;
    if (!paired && (tab_width != head_dim || stagger_offset != 0)) return PHA_ERR_INVALID;
    if (paired && (tab_width != 2 * head_dim ||
                   (stagger_offset != 0 && stagger_offset != head_dim)))
        return PHA_ERR_INVALID;
    if (total_tokens == 0) return PHA_OK;
    return launch_rope_bwd(dq, dk, cos_tab, sin_tab, tab_rows, tab_width, positions, total_tokens,
                           n_heads, n_kv_heads, head_dim, dtype == PHA_BF16, paired, stagger_offset,
                           stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

size_t pha_rope_factor_bytes(int rows, int head_dim, int paired) {
    if (rows < 0 || head_dim <= 0 || (head_dim & 1) || (paired != 0 && paired != 1)) return 0;
    return rope_factor_bytes(rows, head_dim, paired);
}

pha_status pha_rope_factor_tables(void* factors, size_t bytes, int rows, int head_dim, int paired,
                                  double base, pha_stream_t stream) {
    if (!factors || !aligned16(factors) || rows < 0 || head_dim <= 0 || (head_dim & 1) ||
        !(base > 0.0) || (paired != 0 && paired != 1))
        return PHA_ERR_INVALID;
    if (bytes < rope_factor_bytes(rows, head_dim, paired)) return PHA_ERR_INVALID;
    return launch_rope_factor_tables(static_cast<double2*>(factors), rows, head_dim, paired, base,
                                     stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

// Argument checks shared by the factored RoPE calls (those of pha_rope, with the factored tables
// in place of the stored ones).
static pha_status rope_factored_args(const void* q, const void* k, const void* factors, int rows,
                                     const int32_t* positions, int total_tokens, int n_heads,
                                     int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                                     int stagger_offset) {
    if (dtype != PHA_BF16 && dtype != PHA_F32) return PHA_ERR_INVALID;
    const int span = dtype == PHA_BF16 ? 16 : 8;
    if (rows < 0 || total_tokens < 0 || n_heads <= 0 || n_kv_heads < 0 || head_dim <= 0 ||
        head_dim % span != 0 || (paired != 0 && paired != 1))
        return PHA_ERR_INVALID;
    if (total_tokens > 0 && (!q || !aligned16(q) || (n_kv_heads > 0 && (!k || !aligned16(k))) ||
                             !factors || !aligned16(factors) || !positions))
        return PHA_ERR_INVALID;
    if (!paired && stagger_offset != 0) return PHA_ERR_INVALID;
    if (paired && stagger_offset != 0 && stagger_offset != head_dim) return PHA_ERR_INVALID;
    return PHA_OK;
}

pha_status pha_rope_factored(void* q, void* k, const void* factors, int rows,
                             const int32_t* positions, int total_tokens, int n_heads,
                             int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                             int stagger_offset, pha_stream_t stream) {
    const pha_status st = rope_factored_args(q, k, factors, rows, positions, total_tokens, n_heads,
                                             n_kv_heads, head_dim, dtype, paired, stagger_offset);
    if (st != PHA_OK || total_tokens == 0) return st;
    return launch_rope_factored(q, k, static_cast<const double2*>(factors), rows, positions,
                                total_tokens, n_heads, n_kv_heads, head_dim, dtype == PHA_BF16,
                                paired, stagger_offset, false, false, nullptr, nullptr, 0.f,
                                stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

pha_status pha_qk_norm_rope_factored(void* q, void* k, const float* q_weight,
                                     const float* k_weight, float eps, const void* factors,
                                     int rows, const int32_t* positions, int total_tokens,
                                     int n_heads, int n_kv_heads, int head_dim, pha_dtype dtype,
                                     int paired, int stagger_offset, pha_stream_t stream) {
    const pha_status st = rope_factored_args(q, k, factors, rows, positions, total_tokens, n_heads,
                                             n_kv_heads, head_dim, dtype, paired, stagger_offset);
    if (st != PHA_OK) return st;
    if (!(eps >= 0.f) || !(eps < INFINITY)) return PHA_ERR_INVALID;
    if ((q_weight && !aligned16(q_weight)) || (k_weight && !aligned16(k_weight)))
        return PHA_ERR_INVALID;
    const int cph = head_dim / (dtype == PHA_BF16 ? 8 : 4);
    if (32 % cph != 0) return PHA_ERR_UNSUPPORTED;
    if (total_tokens == 0) return PHA_OK;
    return launch_rope_factored(q, k, static_cast<const double2*>(factors), rows, positions,
                                total_tokens, n_heads, n_kv_heads, head_dim, dtype == PHA_BF16,
                                paired, stagger_offset, true, false, q_weight, k_weight, eps,
                                stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

pha_status pha_rope_bwd_factored(void* dq, void* dk, const void* factors, int rows,
                                 const int32_t* positions, int total_tokens, int n_heads,
                                 int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                                 int stagger_offset, pha_stream_t stream) {
    const pha_status st = rope_factored_args(dq, dk, factors, rows, positions, total_tokens,
                                             n_heads, n_kv_heads, head_dim, dtype, paired,
                                             stagger_offset);
    if (st != PHA_OK || total_tokens == 0) return st;
    return launch_rope_factored(dq, dk, static_cast<const double2*>(factors), rows, positions,
                                total_tokens, n_heads, n_kv_heads, head_dim, dtype == PHA_BF16,
                                paired, stagger_offset, false, true, nullptr, nullptr, 0.f,
                                stream) == cudaSuccess
               ? PHA_OK
               : PHA_ERR_CUDA;
}

// Scheduling area of the backward: header, per-document offsets and the largest of its work
// lists, the tile lists (one item per 128-slot tile and head), rounded up to 256 bytes.
static size_t bwd_sched_bytes(int batch, int max_len, int n_heads, int paired) {
    if (pha_attn_workspace_bytes(batch, max_len, n_heads, 64, paired) == 0) return 0;
    const int64_t slots = static_cast<int64_t>(max_len) * (paired ? 2 : 1);
    const int64_t heads = paired ? n_heads / 2 : n_heads;
    const size_t items = static_cast<size_t>(batch) * div_up(slots, kBlockM) * heads;
    const size_t bytes = kWorkspaceHeaderBytes + workspace_doc_bytes(batch) + items * sizeof(int4);
    return (bytes + 255) & ~static_cast<size_t>(255);
}

size_t pha_attn_bwd_workspace_bytes(int batch, int max_len, int total_tokens, int n_heads,
                                    int head_dim, int paired) {
    (void)head_dim;
    if (total_tokens < 0) return 0;
    const size_t sched = bwd_sched_bytes(batch, max_len, n_heads, paired);
    if (sched == 0) return 0;
    return sched + ((static_cast<size_t>(total_tokens) * n_heads * sizeof(float) + 255) &
                    ~static_cast<size_t>(255));
}

pha_status pha_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, const int32_t* cu_seqlens, int batch,
                        int max_len, int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                        pha_dtype dtype, int causal, int window, int paired, float scale, void* dq,
                        void* dk, void* dv, void* workspace, size_t workspace_bytes,
                        pha_stream_t stream) {
    if (dtype != PHA_BF16 && dtype != PHA_F32) return PHA_ERR_INVALID;
    const bool have = total_tokens > 0;
    if ((have && (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !aligned16(q) ||
                  !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
                  !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
                  (reinterpret_cast<uintptr_t>(lse) & 3u))) ||
        !cu_seqlens || batch <= 0 || max_len < 0 || total_tokens < 0 ||
        total_tokens > (1 << 29) || n_heads <= 0 || n_kv_heads <= 0 || n_heads > 4096 ||
        n_heads % n_kv_heads != 0 || head_dim <= 0 || (causal != 0 && causal != 1) ||
        (paired != 0 && paired != 1) || !(scale == scale))
        return PHA_ERR_INVALID;
    if (paired && ((n_heads & 1) || (n_kv_heads & 1))) return PHA_ERR_INVALID;
    if (!causal && window > 0) return PHA_ERR_UNSUPPORTED;
    if (head_dim > 128) return PHA_ERR_UNSUPPORTED;
    if (!have) return PHA_OK;  // nothing to do (no launch, the workspace is not touched)
    const size_t need =
        pha_attn_bwd_workspace_bytes(batch, max_len, total_tokens, n_heads, head_dim, paired);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return PHA_ERR_WORKSPACE;
    AttnProblem p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.cu_seqlens = cu_seqlens;
    p.batch = batch;
    p.max_len = max_len;
    p.total_tokens = total_tokens;
    p.slot_mult = paired ? 2 : 1;
    p.heads = paired ? n_heads / 2 : n_heads;
    p.kv_heads = paired ? n_kv_heads / 2 : n_kv_heads;
    p.head_dim = head_dim;
    p.causal = causal;
    p.window = window > 0 ? window : 0;
    p.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(head_dim));
    p.lse = const_cast<float*>(lse);

    // Workspace: the scheduling area (header, document offsets, work items), then D.
    const size_t sched = bwd_sched_bytes(batch, max_len, n_heads, paired);
    auto* base = static_cast<uint8_t*>(workspace);
    auto* hdr = reinterpret_cast<WorkspaceHeader*>(base);
    auto* doc_blocks = reinterpret_cast<int*>(base + kWorkspaceHeaderBytes);
    const size_t fixed = kWorkspaceHeaderBytes + workspace_doc_bytes(batch);
    auto* items = reinterpret_cast<int4*>(base + fixed);
    const int64_t cap64 = static_cast<int64_t>((sched - fixed) / sizeof(int4));
    const int capacity = cap64 > 0x7FFFFFFF ? 0x7FFFFFFF : static_cast<int>(cap64);
    float* dsum = reinterpret_cast<float*>(base + sched);

    // Tensor cores for bf16 with head_dim 64 / 128 (band work lists for causal windows <= 128,
    // tile lists otherwise); CUDA cores for the rest. The scheduler also checks cu_seqlens
    // (pha_attn_status).
    const bool tc = dtype == PHA_BF16 && (head_dim == 64 || head_dim == 128);
    const bool band = band_applies(p);
    const ScheduleMode mode = !tc ? kSchedBlock : (band ? kSchedBand : kSchedTilesQ);
    if (launch_schedule(p, mode, capacity, doc_blocks, items, hdr, stream) != cudaSuccess)
        return PHA_ERR_CUDA;
    if (launch_attn_bwd_dsum(p, o, dout, dsum, dtype == PHA_BF16, stream) != cudaSuccess)
        return PHA_ERR_CUDA;
    if (!tc)
        return launch_attn_bwd(p, dout, dsum, dq, dk, dv, dtype == PHA_BF16, stream) == cudaSuccess
                   ? PHA_OK
                   : PHA_ERR_CUDA;
    const uint64_t rows = static_cast<uint64_t>(total_tokens) * p.slot_mult;
    CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
    if (!encode_slot_map(&tq, q, static_cast<uint64_t>(p.heads) * head_dim, rows) ||
        !encode_slot_map(&tk, k, static_cast<uint64_t>(p.kv_heads) * head_dim, rows) ||
        !encode_slot_map(&tv, v, static_cast<uint64_t>(p.kv_heads) * head_dim, rows) ||
        !encode_slot_map(&tdo, dout, static_cast<uint64_t>(p.heads) * head_dim, rows) ||
        !encode_slot_map(&tdq, dq, static_cast<uint64_t>(p.heads) * head_dim, rows, 32) ||
        !encode_slot_map(&tdk, dk, static_cast<uint64_t>(p.kv_heads) * head_dim, rows, 16) ||
        !encode_slot_map(&tdv, dv, static_cast<uint64_t>(p.kv_heads) * head_dim, rows, 16))
        return PHA_ERR_CUDA;
    if (launch_attn_bwd_zero_outside(p, dq, dk, dv, stream) != cudaSuccess) return PHA_ERR_CUDA;
    if (band)
        return launch_attn_bwd_tc(p, tq, tk, tv, tdo, tdq, tdk, tdv, dsum, dq, dk, dv, items, hdr, 3,
                                  stream) == cudaSuccess
                   ? PHA_OK
                   : PHA_ERR_CUDA;
    // tile lists: the dQ kernel over query tiles, then the list rebuilt over key tiles (ordered by
    // their own cost) for the dK / dV kernel
    if (launch_attn_bwd_tc(p, tq, tk, tv, tdo, tdq, tdk, tdv, dsum, dq, dk, dv, items, hdr, 1,
                           stream) != cudaSuccess ||
        launch_schedule(p, kSchedTilesK, capacity, doc_blocks, items, hdr, stream) != cudaSuccess ||
        launch_attn_bwd_tc(p, tq, tk, tv, tdo, tdq, tdk, tdv, dsum, dq, dk, dv, items, hdr, 2,
                           stream) != cudaSuccess)
        return PHA_ERR_CUDA;
    return PHA_OK;
}

size_t pha_attn_workspace_bytes(int batch, int max_len, int n_heads, int head_dim, int paired) {
    (void)head_dim;
    if (batch <= 0 || max_len < 0 || n_heads <= 0 || (paired && (n_heads & 1))) return 0;
    return kWorkspaceHeaderBytes + workspace_doc_bytes(batch) +
           static_cast<size_t>(max_work_items(batch, max_len, n_heads, paired)) * sizeof(int4);
}

}  // extern "C"

namespace {

pha_status attn_fwd_impl(const void* q, const void* k, const void* v, const void* v_aux,
                         const int32_t* cu_seqlens, int batch, int max_len, int total_tokens,
                         int n_heads, int n_kv_heads, int head_dim, pha_dtype dtype, int causal,
                         int window, int paired, float scale, void* o, float* lse, void* workspace,
                         size_t workspace_bytes, pha_stream_t stream, int test_stall_us = 0) {
    if (dtype != PHA_BF16 && dtype != PHA_F32) return PHA_ERR_INVALID;
    // With no tokens the q / k / v / o / lse buffers may be empty (NULL); cu_seqlens is still read.
    const bool have = total_tokens > 0;
    if ((have && (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
                  !aligned16(o))) ||
        !cu_seqlens || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || batch <= 0 ||
        max_len < 0 || total_tokens < 0 || total_tokens > (1 << 29) || n_heads <= 0 ||
        n_kv_heads <= 0 || n_heads > 4096 || n_heads % n_kv_heads != 0 || head_dim <= 0 ||
        (causal != 0 && causal != 1) || (paired != 0 && paired != 1) || !(scale == scale))
        return PHA_ERR_INVALID;
    if (paired && ((n_heads & 1) || (n_kv_heads & 1))) return PHA_ERR_INVALID;
    if (!causal && window > 0) return PHA_ERR_UNSUPPORTED;
    if (dtype == PHA_BF16 && head_dim != 64 && head_dim != 128) return PHA_ERR_UNSUPPORTED;
    if (dtype == PHA_F32 && head_dim > 128) return PHA_ERR_UNSUPPORTED;

    AttnProblem p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.cu_seqlens = cu_seqlens;
    p.batch = batch;
    p.max_len = max_len;
    p.total_tokens = total_tokens;
    p.slot_mult = paired ? 2 : 1;
    p.heads = paired ? n_heads / 2 : n_heads;
    p.kv_heads = paired ? n_kv_heads / 2 : n_kv_heads;
    p.head_dim = head_dim;
    p.causal = causal;
    p.window = window > 0 ? window : 0;
    p.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(head_dim));
    p.o = o;
    p.lse = lse;
    p.qk_scale = 1.0f;
    p.v_scale = 1.0f;
    if (test_stall_us != 0) {
        // the failure-detection hook exists in the band kernel only
        if (dtype != PHA_BF16 || !band_applies(p)) return PHA_ERR_UNSUPPORTED;
        if (test_stall_us < 1 || test_stall_us > 100000) return PHA_ERR_INVALID;
        p.test_stall_us = test_stall_us;
    }
    if (v_aux) {
        // value embedding: the bf16 tensor-core kernels (band and block)
        if (dtype != PHA_BF16) return PHA_ERR_UNSUPPORTED;
        if (!aligned16(v_aux)) return PHA_ERR_INVALID;
        p.v_aux = v_aux;
    }

    if (dtype == PHA_F32) {
        if (total_tokens == 0) return PHA_OK;
        return launch_attn_f32(p, stream) == cudaSuccess ? PHA_OK : PHA_ERR_CUDA;
    }

    const size_t need = pha_attn_workspace_bytes(batch, max_len, n_heads, head_dim, paired);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return PHA_ERR_WORKSPACE;
    const size_t fixed = kWorkspaceHeaderBytes + workspace_doc_bytes(batch);
    const int64_t cap64 = static_cast<int64_t>((workspace_bytes - fixed) / sizeof(int4));
    const int capacity = cap64 > 0x7FFFFFFF ? 0x7FFFFFFF : static_cast<int>(cap64);
    auto* base = static_cast<uint8_t*>(workspace);
    auto* hdr = reinterpret_cast<WorkspaceHeader*>(base);
    auto* doc_blocks = reinterpret_cast<int*>(base + kWorkspaceHeaderBytes);
    auto* items = reinterpret_cast<int4*>(base + fixed);

    // Causal windows of at most one key tile run on the band kernel, everything else on the block
    // kernel; the scheduler emits the matching item shape.
    const bool band = band_applies(p);
    if (launch_schedule(p, band ? kSchedBand : kSchedBlock, capacity, doc_blocks, items, hdr,
                        stream) != cudaSuccess)
        return PHA_ERR_CUDA;
    if (total_tokens == 0) return PHA_OK;

    const uint64_t rows = static_cast<uint64_t>(total_tokens) * p.slot_mult;
    CUtensorMap tq, tk, tv;
    if (!encode_slot_map(&tq, q, static_cast<uint64_t>(p.heads) * head_dim, rows) ||
        !encode_slot_map(&tk, k, static_cast<uint64_t>(p.kv_heads) * head_dim, rows) ||
        !encode_slot_map(&tv, v, static_cast<uint64_t>(p.kv_heads) * head_dim, rows))
        return PHA_ERR_CUDA;
    // the band kernel stores O with one 32-row box per warp
    CUtensorMap to;
    if (band && !encode_slot_map(&to, o, static_cast<uint64_t>(p.heads) * head_dim, rows, 32))
        return PHA_ERR_CUDA;
    const cudaError_t e = band ? launch_attn_band(p, tq, tk, tv, to, items, hdr, stream)
                               : launch_attn_tc(p, tq, tk, tv, items, hdr, stream);
    return e == cudaSuccess ? PHA_OK : PHA_ERR_CUDA;
}

}  // namespace

extern "C" {

pha_status pha_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                        int batch, int max_len, int total_tokens, int n_heads, int n_kv_heads,
                        int head_dim, pha_dtype dtype, int causal, int window, int paired,
                        float scale, void* o, float* lse, void* workspace, size_t workspace_bytes,
                        pha_stream_t stream) {
    return attn_fwd_impl(q, k, v, nullptr, cu_seqlens, batch, max_len, total_tokens, n_heads,
                         n_kv_heads, head_dim, dtype, causal, window, paired, scale, o, lse,
                         workspace, workspace_bytes, stream);
}

pha_status pha_attn_fwd_aux_v(const void* q, const void* k, const void* v, const void* aux_v,
                              const int32_t* cu_seqlens, int batch, int max_len,
                              int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                              pha_dtype dtype, int causal, int window, int paired, float scale,
                              void* o, float* lse, void* workspace, size_t workspace_bytes,
                              pha_stream_t stream) {
    if (total_tokens > 0 && !aux_v) return PHA_ERR_INVALID;
    return attn_fwd_impl(q, k, v, total_tokens > 0 ? aux_v : nullptr, cu_seqlens, batch, max_len,
                         total_tokens, n_heads, n_kv_heads, head_dim, dtype, causal, window,
                         paired, scale, o, lse, workspace, workspace_bytes, stream);
}

pha_status pha_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_scale,
                            float k_scale, float v_scale, const int32_t* cu_seqlens, int batch,
                            int max_len, int total_tokens, int n_heads, int n_kv_heads,
                            int head_dim, int causal, int window, int paired, float scale, void* o,
                            float* lse, void* workspace, size_t workspace_bytes,
                            pha_stream_t stream) {
    const bool have = total_tokens > 0;
    if ((have && (!q8 || !k8 || !v8 || !o || !aligned16(q8) || !aligned16(k8) || !aligned16(v8) ||
                  !aligned16(o))) ||
        !cu_seqlens || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || batch <= 0 ||
        max_len < 0 || total_tokens < 0 || total_tokens > (1 << 29) || n_heads <= 0 ||
        n_kv_heads <= 0 || n_heads > 4096 || n_heads % n_kv_heads != 0 || head_dim <= 0 ||
        (causal != 0 && causal != 1) || (paired != 0 && paired != 1) || !(scale == scale) ||
        !(q_scale > 0.f) || !(k_scale > 0.f) || !(v_scale > 0.f) || !(q_scale < INFINITY) ||
        !(k_scale < INFINITY) || !(v_scale < INFINITY))
        return PHA_ERR_INVALID;
    if (paired && ((n_heads & 1) || (n_kv_heads & 1))) return PHA_ERR_INVALID;
    if (!causal && window > 0) return PHA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PHA_ERR_UNSUPPORTED;

    AttnProblem p{};
    p.q = q8;
    p.k = k8;
    p.v = v8;
    p.cu_seqlens = cu_seqlens;
    p.batch = batch;
    p.max_len = max_len;
    p.total_tokens = total_tokens;
    p.slot_mult = paired ? 2 : 1;
    p.heads = paired ? n_heads / 2 : n_heads;
    p.kv_heads = paired ? n_kv_heads / 2 : n_kv_heads;
    p.head_dim = head_dim;
    p.causal = causal;
    p.window = window > 0 ? window : 0;
    p.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(head_dim));
    p.o = o;
    p.lse = lse;
    p.qk_scale = q_scale * k_scale;
    p.v_scale = v_scale;

    const size_t need = pha_attn_workspace_bytes(batch, max_len, n_heads, head_dim, paired);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return PHA_ERR_WORKSPACE;
    const size_t fixed = kWorkspaceHeaderBytes + workspace_doc_bytes(batch);
    const int64_t cap64 = static_cast<int64_t>((workspace_bytes - fixed) / sizeof(int4));
    const int capacity = cap64 > 0x7FFFFFFF ? 0x7FFFFFFF : static_cast<int>(cap64);
    auto* base = static_cast<uint8_t*>(workspace);
    auto* hdr = reinterpret_cast<WorkspaceHeader*>(base);
    auto* doc_blocks = reinterpret_cast<int*>(base + kWorkspaceHeaderBytes);
    auto* items = reinterpret_cast<int4*>(base + fixed);
    // every window runs on the block kernel (its FP8 variant)
    if (launch_schedule(p, kSchedBlock, capacity, doc_blocks, items, hdr, stream) != cudaSuccess)
        return PHA_ERR_CUDA;
    if (total_tokens == 0) return PHA_OK;
    const uint64_t rows = static_cast<uint64_t>(total_tokens) * p.slot_mult;
    CUtensorMap tq, tk, tv;
    if (!encode_u8_map(&tq, q8, static_cast<uint64_t>(p.heads) * head_dim, rows, head_dim, true) ||
        !encode_u8_map(&tk, k8, static_cast<uint64_t>(p.kv_heads) * head_dim, rows, head_dim, true) ||
        !encode_u8_map(&tv, v8, static_cast<uint64_t>(p.kv_heads) * head_dim, rows, head_dim, false))
        return PHA_ERR_CUDA;
    return launch_attn_tc(p, tq, tk, tv, items, hdr, stream, true) == cudaSuccess ? PHA_OK
                                                                                   : PHA_ERR_CUDA;
}

pha_status pha_test_attn_fwd_stalled(const void* q, const void* k, const void* v,
                                     const int32_t* cu_seqlens, int batch, int max_len,
                                     int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                                     pha_dtype dtype, int causal, int window, int paired,
                                     float scale, void* o, float* lse, void* workspace,
                                     size_t workspace_bytes, int stall_us, pha_stream_t stream) {
    if (stall_us == 0) return PHA_ERR_INVALID;
    return attn_fwd_impl(q, k, v, nullptr, cu_seqlens, batch, max_len, total_tokens, n_heads,
                         n_kv_heads, head_dim, dtype, causal, window, paired, scale, o, lse,
                         workspace, workspace_bytes, stream, stall_us);
}

pha_status pha_attn_status(const void* workspace, int* status, int* n_items, pha_stream_t stream) {
    if (!workspace || !status) return PHA_ERR_INVALID;
    WorkspaceHeader h{};
    if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return PHA_ERR_CUDA;
    *status = h.status;
    if (n_items) *n_items = h.n_items;
    return PHA_OK;
}

}  // extern "C"
