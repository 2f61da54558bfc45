/*
 * pha.h -- C ABI of libpha: B200 (sm_100a) forward pass of causal, rotary-embedded, varlen
 * multi-head attention, including the paired-head variant.
 *
 * Method: the "modded-nanogpt Paired Head Attention record" page (hncyxsy.com/news/170276).
 * In the paired variant the two heads h and h + H/2 of every token are interleaved by position
 * into a sequence of twice the length with half the heads: token t, head h lands at slot
 * 2t + h / (H/2), head h % (H/2) (sections "core idea" and "4. interleave index in the Triton
 * kernel"). For a contiguous [tokens][H][head_dim] buffer this is a pure reinterpretation as
 * [2*tokens][H/2][head_dim] (section "zero-copy RoPE and delayed reshape"), so no entry point
 * ever copies data to interleave it. Rotary tables for the paired path pack positions 2p and
 * 2p+1 side by side in one row; odd heads read the second half ("staggered rotary",
 * "2. building the paired rotary table"). Sequence lengths and max_len double on the paired
 * path while the window stays the same ("sequence length and window handling").
 *
 * Conventions shared by all entry points:
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless stated otherwise.
 *     The library allocates no memory and keeps no mutable global state; calls on different
 *     streams may run concurrently as long as they do not share output or workspace buffers.
 *   - All work is queued on `stream` (a cudaStream_t; NULL = the legacy default stream) and is
 *     asynchronous: a return of PHA_OK means "arguments accepted and kernels launched".
 *   - Argument errors are detected before any launch and return a negative pha_status with
 *     nothing launched and no memory touched. Launch failures return PHA_ERR_CUDA.
 *   - Tensors are contiguous, row-major. "bf16" is IEEE bfloat16, "f32" IEEE binary32.
 */
#ifndef PHA_H
#define PHA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* pha_stream_t; /* same type as cudaStream_t */

typedef enum {
    PHA_OK = 0,
    PHA_ERR_INVALID = -1,     /* bad pointer, size, shape or alignment */
    PHA_ERR_UNSUPPORTED = -2, /* well-formed but outside what the kernels implement */
    PHA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than pha_attn_workspace_bytes() */
    PHA_ERR_CUDA = -4         /* a CUDA runtime call or kernel launch failed */
} pha_status;

typedef enum { PHA_BF16 = 0, PHA_F32 = 1 } pha_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* pha_status_string(pha_status s);

/*
 * pha_rope_tables -- fill rotary tables on the device.
 *   Frequencies f_i = base^(-2i/head_dim), i = 0 .. head_dim/2 - 1 (the "Training an LLM from
 *   scratch (part 2)" page, section "2. RoPE"); angles and their cosines and sines are computed
 *   in float64 and rounded to float32.
 *   paired = 0: width = head_dim; cos_tab[p][j] = cos(p * f_{j/2}), sin_tab likewise.
 *   paired = 1: width = 2*head_dim; columns [0, head_dim) hold angles 2p * f_{j/2}, columns
 *               [head_dim, 2*head_dim) hold (2p+1) * f_{(j-head_dim)/2} (the paired table of the
 *               record page, section "2. building the paired rotary table").
 *   cos_tab, sin_tab: float[rows][width], 16-byte aligned, written.
 *   Errors: PHA_ERR_INVALID if a pointer is NULL or misaligned, rows < 0, head_dim odd or
 *   <= 0, base <= 0.
 */
pha_status pha_rope_tables(float* cos_tab, float* sin_tab, int rows, int head_dim, int paired,
                           double base, pha_stream_t stream);

/*
 * pha_rope -- in-place rotary embedding of q and k (record page, sections "zero-copy RoPE and
 * delayed reshape", "staggered rotary", "4. interleave index in the Triton kernel").
 *   q: [total_tokens][n_heads][head_dim], k: [total_tokens][n_kv_heads][head_dim], dtype
 *      `dtype`, 16-byte aligned, read and overwritten. k may be NULL when n_kv_heads == 0.
 *   cos_tab, sin_tab: float[tab_rows][tab_width] as written by pha_rope_tables, 16-byte aligned.
 *   positions: int32[total_tokens], the table row of each token.
 *   For token t, head h, pair i (columns 2i, 2i+1) with c = cos_tab[positions[t]][col0 + 2i],
 *   s = sin_tab[...][col0 + 2i]:  y[2i] = x[2i] c - x[2i+1] s,  y[2i+1] = x[2i] s + x[2i+1] c,
 *   where col0 = 0, or col0 = stagger_offset for odd h when paired = 1.
 *   paired = 0: tab_width must equal head_dim and stagger_offset must be 0.
 *   paired = 1: tab_width must equal 2*head_dim; stagger_offset is head_dim (the page's
 *               staggered rotary: odd heads take phase 2p+1) or 0 (both heads take 2p).
 *   A token whose position lies outside [0, tab_rows) is left unchanged; this is not reported.
 *   The rotation is computed in float64 (exact products) and rounded once to the dtype, so the
 *   result is the correctly rounded rotation with the tables' float32 values.
 *   total_tokens = 0 is a no-op and then q, k, the tables and positions may be NULL.
 *   Errors: PHA_ERR_INVALID for NULL/misaligned pointers, negative sizes, n_heads <= 0,
 *   head_dim not a positive multiple of 16 (bf16) or 8 (f32), or table width / stagger_offset
 *   not as above.
 */
pha_status pha_rope(void* q, void* k, const float* cos_tab, const float* sin_tab, int tab_rows,
                    int tab_width, const int32_t* positions, int total_tokens, int n_heads,
                    int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                    int stagger_offset, pha_stream_t stream);

/*
 * pha_qk_norm_rope -- the QK RMS-norm of every head row, then pha_rope, in one pass (in place).
 *   The paired-head page's rotary kernel also applies the QK RMS-norm ("modded-nanogpt Paired Head
 *   Attention record", section "4. interleave index in the Triton kernel"); RMSNorm is
 *   y = x / sqrt(mean(x^2) + eps) * weight over the last dimension ("Training an LLM from scratch
 *   (part 2)", section "1. RMSNorm"). Each (token, head) row of q and of k is normalised over
 *   head_dim in float32 and multiplied by q_weight / k_weight (float[head_dim], 16-byte aligned, or
 *   NULL for ones), then rotated as pha_rope rotates, with one rounding to dtype at the end.
 *   Tokens whose position lies outside [0, tab_rows) are normalised but not rotated.
 *   eps: >= 0, finite. Other arguments, layouts and errors: as pha_rope.
 *   Supported head_dim: those whose row of 16-byte chunks (head_dim/8 for bf16, head_dim/4 for f32)
 *   divides 32; others return PHA_ERR_UNSUPPORTED.
 */
pha_status pha_qk_norm_rope(void* q, void* k, const float* q_weight, const float* k_weight,
                            float eps, const float* cos_tab, const float* sin_tab, int tab_rows,
                            int tab_width, const int32_t* positions, int total_tokens,
                            int n_heads, int n_kv_heads, int head_dim, pha_dtype dtype,
                            int paired, int stagger_offset, pha_stream_t stream);

/*
 * pha_rope_factor_bytes -- size in bytes of the factored rotary tables (pha_rope_factor_tables)
 *   for table rows [0, rows), head_dim and paired; 0 for invalid arguments (rows < 0, head_dim
 *   odd or <= 0, paired not 0/1).
 */
size_t pha_rope_factor_bytes(int rows, int head_dim, int paired);

/*
 * pha_rope_factor_tables -- fill factored rotary tables on the device. They stand for the
 *   pha_rope_tables of the same rows, head_dim, paired and base (same frequencies, same float64
 *   angles), in two small float64 tables that stay in L1 / L2 instead of a float32 row per
 *   position: table row p = 16 r + l splits each angle into a coarse part (row 16 r; for a paired
 *   row its even position 32 r) and a fine part (row l), whose cosines and sines are stored.
 *   The factored RoPE calls form cos(a + b) = cos a cos b - sin a sin b and
 *   sin(a + b) = sin a cos b + cos a sin b in float64 and round each once to float32 (the
 *   "modded-nanogpt Paired Head Attention record" page, section "2. building the paired rotary
 *   table", keeps precomputed factor tables; this is a compact form of the same values).
 *   Layout, pairs (cos, sin) of float64: 16 fine rows of A entries (A = head_dim/2, or head_dim
 *   when paired), entry a of fine row l holding position l (standard) or 2l + a / (head_dim/2)
 *   (paired) at frequency i = a % (head_dim/2); then ceil(rows/16) coarse rows of head_dim/2
 *   entries, entry i of coarse row r holding position 16 r (standard) or 32 r (paired) at
 *   frequency i. Frequencies f_i = base^(-2i/head_dim) as in pha_rope_tables.
 *   factors: device buffer of `bytes` >= pha_rope_factor_bytes(rows, head_dim, paired) bytes,
 *   16-byte aligned, written.
 *   Errors: PHA_ERR_INVALID for a NULL or misaligned buffer, bytes too small, rows < 0, head_dim
 *   odd or <= 0, base <= 0, paired not 0/1.
 */
pha_status pha_rope_factor_tables(void* factors, size_t bytes, int rows, int head_dim, int paired,
                                  double base, pha_stream_t stream);

/*
 * pha_rope_factored -- pha_rope with factored tables (pha_rope_factor_tables) in place of
 *   cos_tab / sin_tab: the rotation reads only q and k from HBM.
 *   factors: as written by pha_rope_factor_tables for `rows` rows and the same head_dim and
 *   paired, 16-byte aligned, read only. positions index rows [0, rows); a token outside is left
 *   unchanged. Each cosine and sine equals the stored table's float32 value, or differs from it
 *   by one unit in the last place next to a float32 rounding midpoint, or, for values very close
 *   to zero, by the float64 angles' own difference (the two forms round their angles differently:
 *   at most about 5e-11 at angles of 1.4e5). With these values the rotation is correctly rounded
 *   as in pha_rope (bf16: compensated float32 arithmetic, float64 next to a rounding midpoint).
 *   Other arguments, layouts and errors: as pha_rope (there is no tab_width; stagger_offset is 0,
 *   or head_dim when paired).
 */
pha_status pha_rope_factored(void* q, void* k, const void* factors, int rows,
                             const int32_t* positions, int total_tokens, int n_heads,
                             int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                             int stagger_offset, pha_stream_t stream);

/* pha_qk_norm_rope_factored -- pha_qk_norm_rope with factored tables, as pha_rope_factored. */
pha_status pha_qk_norm_rope_factored(void* q, void* k, const float* q_weight,
                                     const float* k_weight, float eps, const void* factors,
                                     int rows, const int32_t* positions, int total_tokens,
                                     int n_heads, int n_kv_heads, int head_dim, pha_dtype dtype,
                                     int paired, int stagger_offset, pha_stream_t stream);

/*
 * pha_attn_workspace_bytes -- device workspace that pha_attn_fwd needs: a 256-byte header,
 * int32[batch + 1] of per-document scratch (padded to 16 bytes) and the varlen work list, 16
 * bytes for each of at most batch * ceil(L/256) * H' (query block, head) items (L = max_len,
 * doubled when paired; H' = n_heads, halved when paired). Returns 0 for invalid arguments.
 */
size_t pha_attn_workspace_bytes(int batch, int max_len, int n_heads, int head_dim, int paired);

/*
 * pha_attn_fwd -- varlen attention forward: O and the per-row log-sum-exp.
 *   q: [total_tokens][n_heads][head_dim]; k, v: [total_tokens][n_kv_heads][head_dim]; dtype
 *      `dtype`; 16-byte aligned; read only.
 *   cu_seqlens: int32[batch+1], document boundaries in TOKENS (not doubled), non-decreasing,
 *      cu_seqlens[0] >= 0, cu_seqlens[batch] <= total_tokens; every document at most max_len
 *      tokens long. When paired = 1 the library itself doubles the boundaries and max_len.
 *   Sequence seen by the kernels: standard -- slots = tokens, H' = n_heads, Hkv' = n_kv_heads;
 *      paired -- the same buffers read as [2*total_tokens][n_heads/2][head_dim] (slot 2t+h/(H/2)).
 *   Query slot i of the document spanning slots [a, b) attends key slot j iff a <= j < b,
 *      j <= i when causal, and i - j < window when window > 0 (window counts key slots,
 *      including the query's own; it is NOT doubled on the paired path). Query head h' uses
 *      kv head h' / (H'/Hkv') (GQA).
 *   scale: logit multiplier; scale <= 0 selects 1/sqrt(head_dim).
 *   o: same shape, dtype and layout as q, written (16-byte aligned).
 *   lse: float[total_tokens][n_heads] (paired: the same bytes as [2*total_tokens][n_heads/2]),
 *      lse = ln sum_j exp(scale * q.k_j) over visible keys; may be NULL (then not written).
 *   workspace: device scratch of at least pha_attn_workspace_bytes(...) bytes, 16-byte aligned;
 *      its contents need not be initialised. The scheduler kernel writes the work list into it
 *      and records in its first 8 bytes the number of work items and a device-side status
 *      (see pha_attn_status). May be NULL for PHA_F32, which does not use it.
 *      The list stays in the workspace after the call, with a copy of cu_seqlens, the shape it
 *      was built for and a checksum of its items. A later call on the same workspace whose
 *      cu_seqlens values, shape (batch, max_len, total_tokens, heads, causal, window, paired,
 *      kernel) and workspace size match, and whose items are intact, keeps the list instead of
 *      rebuilding it (the scheduler kernel then only compares; the usual case when every layer
 *      of a model attends over the same documents). Anything else rebuilds it, so the caller may
 *      still use the workspace as scratch between calls.
 *   total_tokens = 0: q, k, v, o, lse may be NULL; the scheduler still records 0 work items.
 *   Slots that lie outside every document (cu_seqlens[batch] < total_tokens) are not written.
 *   Supported: bf16 with head_dim in {64, 128} (tcgen05 tensor-core kernel); f32 with
 *      1 <= head_dim <= 128 (exact float32 CUDA-core kernel).
 *   Errors (before launch): PHA_ERR_INVALID for NULL/misaligned pointers, non-positive sizes,
 *      n_heads % n_kv_heads != 0, paired with odd n_heads or n_kv_heads;
 *      PHA_ERR_UNSUPPORTED for causal = 0 with window > 0 and for unsupported dtype/head_dim;
 *      PHA_ERR_WORKSPACE when the workspace is NULL or too small for the bf16 path.
 *   Errors found on the device (cu_seqlens not as stated): no output row is written and the
 *      status word in the workspace is set; read it with pha_attn_status.
 */
pha_status pha_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                        int batch, int max_len, int total_tokens, int n_heads, int n_kv_heads,
                        int head_dim, pha_dtype dtype, int causal, int window, int paired,
                        float scale, void* o, float* lse, void* workspace, size_t workspace_bytes,
                        pha_stream_t stream);

/*
 * pha_attn_fwd_aux_v -- pha_attn_fwd with a value embedding added to v on the way in:
 *   attention over (q, k, v + aux_v), with v + aux_v rounded to dtype as a tensor addition in
 *   dtype rounds it ("modded-nanogpt Paired Head Attention record" page, section "3. the paired
 *   branch of the forward pass": v = v + aux_v, reshaped like v on the paired path). aux_v has v's
 *   shape, dtype and layout ([total_tokens][n_kv_heads][head_dim], 16-byte aligned); neither v nor
 *   aux_v is modified (the sum is formed tile by tile in shared memory).
 *   Other arguments, results and errors: as pha_attn_fwd.
 *   Supported: bf16 with head_dim in {64, 128}, every window and causal setting (the band kernel
 *      for causal windows <= 128, the block kernel otherwise); f32 returns PHA_ERR_UNSUPPORTED
 *      before any launch. aux_v NULL with total_tokens > 0: PHA_ERR_INVALID.
 */
pha_status pha_attn_fwd_aux_v(const void* q, const void* k, const void* v, const void* aux_v,
                              const int32_t* cu_seqlens, int batch, int max_len,
                              int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                              pha_dtype dtype, int causal, int window, int paired, float scale,
                              void* o, float* lse, void* workspace, size_t workspace_bytes,
                              pha_stream_t stream);

/*
 * pha_attn_fwd_fp8 -- pha_attn_fwd over FP8 (e4m3) q, k, v with per-tensor scales.
 *   The packed FP8 QKV projection of the record page produces Q, K and V in 8-bit floating point
 *   ("modded-nanogpt Paired Head Attention record", section "5. interactions with other
 *   mechanisms"); this entry point consumes them without widening them in HBM.
 *   q8: [total_tokens][n_heads][head_dim], k8, v8: [total_tokens][n_kv_heads][head_dim], one byte
 *      per element in the OCP FP8 E4M3 format (torch.float8_e4m3fn: bias 7, no infinities, NaN
 *      codes 0x7F / 0xFF, largest finite 448); 16-byte aligned; read only. The paired slot view,
 *      cu_seqlens, masks, GQA mapping and errors are those of pha_attn_fwd.
 *   q_scale, k_scale, v_scale: positive finite float32; the tensors stand for
 *      q = q_scale * value(q8), k = k_scale * value(k8), v = v_scale * value(v8).
 *   Result: O and LSE of attention over those q, k, v, exactly as pha_attn_fwd defines them
 *      (scale <= 0 selects 1/sqrt(head_dim)); o is bf16 ([total_tokens][n_heads][head_dim]),
 *      lse float32 [total_tokens][n_heads] (may be NULL).
 *   Arithmetic: S = Q K^T on the tensor cores in kind::f8f6f4 (products of e4m3 values are exact
 *      in the float32 accumulator), scaled by scale * q_scale * k_scale; P rounded to f16; V
 *      widened exactly to f16 in shared memory; O += P V in kind::f16 with float32 accumulation;
 *      O multiplied by v_scale / l; bf16 output.
 *   Supported: head_dim 64 or 128, any causal window or none, causal or not (block kernel).
 *   workspace: as pha_attn_fwd (pha_attn_workspace_bytes with the same arguments).
 *   Errors: as pha_attn_fwd; PHA_ERR_INVALID also for a scale that is not positive and finite;
 *      PHA_ERR_UNSUPPORTED for head_dim other than 64 / 128.
 */
pha_status pha_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_scale,
                            float k_scale, float v_scale, const int32_t* cu_seqlens, int batch,
                            int max_len, int total_tokens, int n_heads, int n_kv_heads,
                            int head_dim, int causal, int window, int paired, float scale, void* o,
                            float* lse, void* workspace, size_t workspace_bytes,
                            pha_stream_t stream);

/*
 * pha_rope_bwd -- backward of pha_rope: the gradients with respect to the unrotated q and k, from
 *   the gradients with respect to the rotated ones (in place). The rotation of each pair is
 *   orthogonal, so its gradient is the transposed rotation, i.e. the rotation by -angle
 *   (the paired-head page's note that the backward of its rotary kernel uses the same PAIRED
 *   index branch: "modded-nanogpt Paired Head Attention record", section "4. interleave index in
 *   the Triton kernel"). Arguments, layouts, rounding and errors: as pha_rope, with dq, dk in place
 *   of q, k. Tokens whose position lies outside the table are left unchanged.
 */
pha_status pha_rope_bwd(void* dq, void* dk, const float* cos_tab, const float* sin_tab,
                        int tab_rows, int tab_width, const int32_t* positions, int total_tokens,
                        int n_heads, int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                        int stagger_offset, pha_stream_t stream);

/* pha_rope_bwd_factored -- pha_rope_bwd with factored tables, as pha_rope_factored. */
pha_status pha_rope_bwd_factored(void* dq, void* dk, const void* factors, int rows,
                                 const int32_t* positions, int total_tokens, int n_heads,
                                 int n_kv_heads, int head_dim, pha_dtype dtype, int paired,
                                 int stagger_offset, pha_stream_t stream);

/*
 * pha_attn_bwd_workspace_bytes -- device scratch pha_attn_bwd needs: a scheduling area (a 256-byte
 *   header, which pha_attn_status reads, int32[batch + 1] padded to 16 bytes, and 16 bytes for
 *   each of at most batch * ceil(L/128) * H' (128-slot tile, head) work items, L and H' as for
 *   pha_attn_workspace_bytes; rounded up to 256 bytes) followed by float[total_tokens][n_heads]
 *   (the row sums D_i), rounded up to 256 bytes. head_dim does not enter. 0 for invalid arguments.
 */
size_t pha_attn_bwd_workspace_bytes(int batch, int max_len, int total_tokens, int n_heads,
                                    int head_dim, int paired);

/*
 * pha_attn_bwd -- backward of pha_attn_fwd: dq, dk, dv for the upstream gradient dout.
 *   With P the forward's attention weights, P_ij = exp(scale q_i.k_j - lse_i) over the visible
 *   keys (recomputed from q, k and the forward's lse; no score matrix is saved):
 *     dP_ij = dout_i . v_j,  D_i = sum_j P_ij dP_ij = dout_i . o_i,  dS_ij = P_ij (dP_ij - D_i),
 *     dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dout_i
 *   (FlashAttention's backward; "Training an LLM from scratch (part 2)", section "4. GQA &
 *   FlashAttention"). D is taken from the forward's output o, as stored (bf16 or f32).
 *   q, k, v, cu_seqlens, batch, max_len, total_tokens, heads, head_dim, dtype, causal, window,
 *   paired, scale: exactly as given to the forward (the paired path uses the same slot view and
 *   doubled documents). o, lse: the forward's outputs (lse float[total_tokens][n_heads]; both
 *   required). dout: like o. dq: like q; dk, dv: like k, v (all written; rows outside every
 *   document get zeros). workspace: at least pha_attn_bwd_workspace_bytes(...), 16-byte aligned;
 *   pha_attn_status(workspace) reports the device status afterwards (malformed cu_seqlens, a
 *   kernel wait that gave up).
 *   Arithmetic: bf16 with head_dim 64 or 128: the tensor cores (tcgen05, bf16 operands with P and
 *   dS rounded to bf16, float32 accumulation in TMEM), one kernel for dq and one for dk, dv (band
 *   work lists for causal windows <= 128, per-tile work lists otherwise); other head_dims and f32
 *   run in float32 on CUDA cores (head_dim <= 128). No atomics on any path.
 *   Errors: as pha_attn_fwd (PHA_ERR_INVALID, PHA_ERR_UNSUPPORTED for head_dim > 128 and for
 *   non-causal windows, PHA_ERR_WORKSPACE); o or lse NULL with total_tokens > 0: PHA_ERR_INVALID.
 *   With total_tokens == 0 the call returns PHA_OK after checking its arguments, launching nothing.
 */
pha_status pha_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, const int32_t* cu_seqlens, int batch,
                        int max_len, int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                        pha_dtype dtype, int causal, int window, int paired, float scale, void* dq,
                        void* dk, void* dv, void* workspace, size_t workspace_bytes,
                        pha_stream_t stream);

/*
 * pha_attn_status -- synchronise `stream` and read the device-side status that the last
 * pha_attn_fwd on this workspace recorded: 0 = fine; 1 = cu_seqlens malformed (decreasing,
 * negative start, beyond total_tokens, or a document longer than max_len); 2 = more work
 * items than the workspace holds; 3 = a kernel wait exceeded its time limit and the kernel
 * gave up. *n_items receives the number of scheduled work items (may be NULL).
 * Host pointers: status, n_items. Errors: PHA_ERR_INVALID for NULL workspace/status,
 * PHA_ERR_CUDA if the copy fails.
 */
pha_status pha_attn_status(const void* workspace, int* status, int* n_items, pha_stream_t stream);

/*
 * pha_test_attn_fwd_stalled -- failure-detection test hook; not for production use.
 *   Runs pha_attn_fwd (same arguments, same checks) with one change in the band kernel: its
 *   softmax warps first wait up to stall_us microseconds on a barrier that nothing signals. The
 *   wait runs out, the kernel records device status 3 (read it with pha_attn_status), every role
 *   of each CTA winds down (the producer waits for its copies in flight, the MMA thread for its
 *   MMAs, tensor memory is freed) and no output row is written. The GPU context stays usable: a
 *   later call on the same workspace and stream runs normally. This is how a kernel wait that
 *   gives up is exercised without faulting or hanging a GPU.
 *   stall_us: 1 .. 100000, else PHA_ERR_INVALID. Only the band kernel has the hook (bf16, causal,
 *   1 <= window <= 128); other shapes return PHA_ERR_UNSUPPORTED.
 */
pha_status pha_test_attn_fwd_stalled(const void* q, const void* k, const void* v,
                                     const int32_t* cu_seqlens, int batch, int max_len,
                                     int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                                     pha_dtype dtype, int causal, int window, int paired,
                                     float scale, void* o, float* lse, void* workspace,
                                     size_t workspace_bytes, int stall_us, pha_stream_t stream);

/*
 * pha_attn_fwd_noalloc -- pha_attn_fwd without a caller-provided workspace.
 *   The pages describe nothing like it: it exists for callers that cannot allocate device
 *   memory, such as a plug-in that receives only its input and output buffers from a host
 *   framework that owns all device memory, or latency-critical code that must not call
 *   cudaMalloc because it can synchronise the whole device.
 *   Arguments and results are those of pha_attn_fwd, minus workspace / workspace_bytes. The
 *   scratch is a 1 MiB array inside the library, one per GPU, held by every GPU that loads the
 *   library until the process exits. The call itself allocates nothing.
 *   Limit: problems whose pha_attn_workspace_bytes(...) exceeds 1 MiB are rejected with
 *   PHA_ERR_WORKSPACE before any launch, after the argument checks of pha_attn_fwd (PHA_F32 uses
 *   no scratch and has no such limit).
 *   Set-up: the first call in a CUDA context on a device looks up the array's device address,
 *   with the calling thread's current device; that device must be the one `stream` belongs to.
 *   Make that first call before any stream capture. A new context on the device (after
 *   cudaDeviceReset, or after the primary context was released and created again) loads the
 *   library's device code afresh; the next call notices the new context and looks the address
 *   up again, so that first call should also come before any capture.
 *   Sharing: every call uses the same array, which keeps the last call's contents. Nothing in it
 *   needs to start at zero (each call rewrites what it reads). Calls whose kernels can run at the
 *   same time on one GPU (unordered streams, several host threads) race on the array; order them
 *   on one stream or with events. The device-side status that pha_attn_status reports lives in
 *   this array and cannot be read through this entry point.
 *   Errors: as pha_attn_fwd; PHA_ERR_UNSUPPORTED for a device index >= 64; PHA_ERR_CUDA if the
 *   address lookup fails.
 */
pha_status pha_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens, int batch, int max_len,
                                int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                                pha_dtype dtype, int causal, int window, int paired, float scale,
                                void* o, float* lse, pha_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PHA_H */
