// attn_bwd.cu -- backward of the varlen (paired-head) attention forward on CUDA cores in float32
// (every shape), and the two small kernels both backward paths share.
//
// The gradients through the row softmax (with P the attention weights of the forward,
// P_ij = exp(scale q_i . k_j - lse_i) over the visible keys):
//   dP_ij = dO_i . v_j,  D_i = sum_j P_ij dP_ij,  dS_ij = P_ij (dP_ij - D_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dO_i.
// P is recomputed from q, k and the forward's lse (FlashAttention's recomputation: "Training an
// LLM from scratch (part 2)", section "4. GQA & FlashAttention" -- no score matrix is stored), and
// D_i = sum_j P_ij (dO_i . v_j) = dO_i . O_i is taken from the forward's output O (one pass over
// O and dO, attn_bwd_dsum_kernel). The paired-head variant is the same slot view of the buffers
// and the same doubled documents as the forward ("modded-nanogpt Paired Head Attention record"
// page, sections "3. the paired branch of the forward pass" and "sequence length and window
// handling").
//
// CUDA-core path: two kernels, no atomics, each on blocks of 32 consecutive rows of one head:
//   dq   (query-major): 32 query slots of one head; the keys they see are staged 32 at a time in
//        shared memory (float32), accumulating dq_i.
//   dkdv (key-major):   32 key slots of one kv head; for each query head of the group the queries
//        that see them are staged 32 at a time (q, dO, lse, D), accumulating dk_j and dv_j.
// Eight consecutive lanes share a row. Lane r of the eight holds the float4 chunks r, r + 8, ... of
// the row (rows padded with zeros to HP = 32, 64 or 128 elements), so the eight lanes read a staged
// row as contiguous 128-byte pieces and the four row groups of a warp share (broadcast) them. The
// two dot products of a (query, key) pair are reduced over the eight lanes with three 64-bit
// shuffles. Staged chunks that no row of a warp can see are skipped by that warp.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <limits.h>
#include <math.h>
#include <stdint.h>

#include "kernels.cuh"

namespace pha {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kLanesPerRow = 8;
constexpr int kRowsPerBlock = kBwdThreads / kLanesPerRow;  // 32
constexpr int kStage = 32;                                // rows staged per chunk

template <typename T>
__device__ __forceinline__ float ld(const T* p);
template <>
__device__ __forceinline__ float ld<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(__ldg(p));
}

template <typename T>
__device__ __forceinline__ void st(T* p, float x);
template <>
__device__ __forceinline__ void st<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
}

// Sum of (a, b) over the eight lanes of a row group (both results in all eight).
__device__ __forceinline__ void group_sum2(float& a, float& b) {
#pragma unroll
    for (int o = 1; o < kLanesPerRow; o <<= 1) {
        const unsigned long long v =
            (static_cast<unsigned long long>(__float_as_uint(b)) << 32) | __float_as_uint(a);
        const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
        a += __uint_as_float(static_cast<uint32_t>(w));
        b += __uint_as_float(static_cast<uint32_t>(w >> 32));
    }
}

// [min, max) of per-row ranges over the four row groups of a warp.
__device__ __forceinline__ void warp_range(long long& a, long long& b) {
#pragma unroll
    for (int o = kLanesPerRow; o < 32; o <<= 1) {
        a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
        b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
    }
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b, float acc) {
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}

__device__ __forceinline__ void axpy4(float4& y, float a, const float4& x) {
    y.x = fmaf(a, x.x, y.x);
    y.y = fmaf(a, x.y, y.y);
    y.z = fmaf(a, x.z, y.z);
    y.w = fmaf(a, x.w, y.w);
}

// Document [lo, hi) (in slots) that contains slot s, or false when s lies outside every document.
__device__ __forceinline__ bool doc_of_slot(const AttnProblem& p, int64_t s, int64_t& lo,
                                            int64_t& hi) {
    int a = 0, b = p.batch;  // last d with cu[d] * mult <= s, among d in [0, batch)
    if (p.batch <= 0 || s < static_cast<int64_t>(p.cu_seqlens[0]) * p.slot_mult) return false;
    while (b - a > 1) {
        const int m = (a + b) >> 1;
        if (static_cast<int64_t>(p.cu_seqlens[m]) * p.slot_mult <= s) a = m; else b = m;
    }
    lo = static_cast<int64_t>(p.cu_seqlens[a]) * p.slot_mult;
    hi = static_cast<int64_t>(p.cu_seqlens[a + 1]) * p.slot_mult;
    return s < hi;
}

// Cooperative copy of rows first .. first + n - 1 (n <= kStage; row r at src + r * stride, hd
// elements) into dst[kStage][HP] as float32, zero past n rows and past hd elements.
template <int HP, typename T>
__device__ __forceinline__ void stage_rows(float* dst, const T* src, int64_t first, int n,
                                           int64_t stride, int hd) {
    for (int x = threadIdx.x; x < kStage * HP; x += kBwdThreads) {
        const int r = x / HP, e = x % HP;
        dst[x] = (r < n && e < hd) ? ld(src + (first + r) * stride + e) : 0.f;
    }
}

// The (zero-padded) row of hd elements at src, as this lane's NC float4 chunks.
template <int NC, typename T>
__device__ __forceinline__ void load_row(float4 (&x)[NC], const T* src, int hd, int r8, bool valid) {
#pragma unroll
    for (int t = 0; t < NC; ++t) {
        const int e = 4 * (r8 + kLanesPerRow * t);
        x[t].x = (valid && e + 0 < hd) ? ld(src + e + 0) : 0.f;
        x[t].y = (valid && e + 1 < hd) ? ld(src + e + 1) : 0.f;
        x[t].z = (valid && e + 2 < hd) ? ld(src + e + 2) : 0.f;
        x[t].w = (valid && e + 3 < hd) ? ld(src + e + 3) : 0.f;
    }
}

template <int NC, typename T>
__device__ __forceinline__ void store_row(T* dst, const float4 (&x)[NC], int hd, int r8) {
#pragma unroll
    for (int t = 0; t < NC; ++t) {
        const int e = 4 * (r8 + kLanesPerRow * t);
        if (e + 0 < hd) st(dst + e + 0, x[t].x);
        if (e + 1 < hd) st(dst + e + 1, x[t].y);
        if (e + 2 < hd) st(dst + e + 2, x[t].z);
        if (e + 3 < hd) st(dst + e + 3, x[t].w);
    }
}

template <int HP, typename T>
__global__ void __launch_bounds__(kBwdThreads) attn_bwd_dq_kernel(AttnProblem p,
                                                                   const T* __restrict__ dout,
                                                                   const float* __restrict__ dsum,
                                                                   T* __restrict__ dq) {
    constexpr int NC = HP / (4 * kLanesPerRow);
    extern __shared__ float4 bsm4[];
    float* ks = reinterpret_cast<float*>(bsm4);  // [kStage][HP]
    float* vs = ks + kStage * HP;                // [kStage][HP]
    __shared__ long long range[2];               // keys seen by the block's rows: [min, max)
    const int H = p.heads, Hkv = p.kv_heads, hd = p.head_dim, G = H / Hkv;
    const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
    const int h = blockIdx.y, g = h / G;
    const int r8 = threadIdx.x % kLanesPerRow;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kLanesPerRow;
    const float scale2 = p.scale * 1.4426950408889634f;
    int64_t lo = 0, hi = 0;
    const bool in_doc = i < slots && doc_of_slot(p, i, lo, hi);
    long long j0 = LLONG_MAX, j1 = LLONG_MIN;  // this row's visible keys [j0, j1)
    if (in_doc) {
        j0 = lo;
        j1 = hi;
        if (p.causal) {
            j1 = i + 1;
            if (p.window > 0 && i - p.window + 1 > j0) j0 = i - p.window + 1;
        }
    }
    if (threadIdx.x == 0) {
        range[0] = LLONG_MAX;
        range[1] = LLONG_MIN;
    }
    __syncthreads();
    if (in_doc && r8 == 0) {
        atomicMin(&range[0], j0);
        atomicMax(&range[1], j1);
    }
    const int64_t row = i * H + h;
    float4 qi[NC], gi[NC], acc[NC];
    load_row<NC>(qi, static_cast<const T*>(p.q) + row * hd, hd, r8, in_doc);
    load_row<NC>(gi, dout + row * hd, hd, r8, in_doc);
#pragma unroll
    for (int t = 0; t < NC; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
    const float lse2 = in_doc ? p.lse[row] * 1.4426950408889634f : 0.f;
    long long wj0 = j0, wj1 = j1;
    warp_range(wj0, wj1);
    __syncthreads();
    const long long J0 = range[0], J1 = range[1];
    const T* kg = static_cast<const T*>(p.k) + static_cast<int64_t>(g) * hd;
    const T* vg = static_cast<const T*>(p.v) + static_cast<int64_t>(g) * hd;
    const int64_t kstride = static_cast<int64_t>(Hkv) * hd;
    const float d = in_doc ? dsum[row] : 0.f;
    {
        for (long long c0 = J0; c0 < J1; c0 += kStage) {
            const int n = static_cast<int>(J1 - c0 < kStage ? J1 - c0 : kStage);
            __syncthreads();  // every warp is done with the previous chunk
            stage_rows<HP>(ks, kg, c0, n, kstride, hd);
            stage_rows<HP>(vs, vg, c0, n, kstride, hd);
            __syncthreads();
            if (c0 + n <= wj0 || c0 >= wj1) continue;  // warp-uniform
            for (int jj = 0; jj < n; ++jj) {
                const long long j = c0 + jj;
                const float4* kr = reinterpret_cast<const float4*>(ks + jj * HP);
                const float4* vr = reinterpret_cast<const float4*>(vs + jj * HP);
                float4 kk[NC];
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int t = 0; t < NC; ++t) {
                    kk[t] = kr[r8 + kLanesPerRow * t];
                    s = dot4(qi[t], kk[t], s);
                    dp = dot4(gi[t], vr[r8 + kLanesPerRow * t], dp);
                }
                group_sum2(s, dp);
                const float pij = (j >= j0 && j < j1) ? exp2f(fmaf(s, scale2, -lse2)) : 0.f;
                const float ds = pij * (dp - d) * p.scale;
#pragma unroll
                for (int t = 0; t < NC; ++t) axpy4(acc[t], ds, kk[t]);
            }
        }
    }
    if (i < slots) store_row<NC>(dq + row * hd, acc, hd, r8);
}

template <int HP, typename T>
__global__ void __launch_bounds__(kBwdThreads) attn_bwd_dkdv_kernel(AttnProblem p,
                                                                     const T* __restrict__ dout,
                                                                     const float* __restrict__ dsum,
                                                                     T* __restrict__ dk,
                                                                     T* __restrict__ dv) {
    constexpr int NC = HP / (4 * kLanesPerRow);
    extern __shared__ float4 bsm4[];
    float* qs = reinterpret_cast<float*>(bsm4);  // [kStage][HP]
    float* gs = qs + kStage * HP;                // [kStage][HP]
    float* ls = gs + kStage * HP;                // lse * log2(e) [kStage]
    float* dd = ls + kStage;                     // D [kStage]
    __shared__ long long range[2];               // queries that see the block's keys: [min, max)
    const int H = p.heads, Hkv = p.kv_heads, hd = p.head_dim, G = H / Hkv;
    const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
    const int g = blockIdx.y;
    const int r8 = threadIdx.x % kLanesPerRow;
    const int64_t j = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kLanesPerRow;
    const float scale2 = p.scale * 1.4426950408889634f;
    int64_t lo = 0, hi = 0;
    const bool in_doc = j < slots && doc_of_slot(p, j, lo, hi);
    long long i0 = LLONG_MAX, i1 = LLONG_MIN;  // queries that see key j: [i0, i1)
    if (in_doc) {
        i0 = lo;
        i1 = hi;
        if (p.causal) {
            i0 = j;
            if (p.window > 0 && j + p.window < i1) i1 = j + p.window;
        }
    }
    if (threadIdx.x == 0) {
        range[0] = LLONG_MAX;
        range[1] = LLONG_MIN;
    }
    __syncthreads();
    if (in_doc && r8 == 0) {
        atomicMin(&range[0], i0);
        atomicMax(&range[1], i1);
    }
    const int64_t krow = j * Hkv + g;
    float4 kj[NC], vj[NC], ak[NC], av[NC];
    load_row<NC>(kj, static_cast<const T*>(p.k) + krow * hd, hd, r8, in_doc);
    load_row<NC>(vj, static_cast<const T*>(p.v) + krow * hd, hd, r8, in_doc);
#pragma unroll
    for (int t = 0; t < NC; ++t) ak[t] = av[t] = make_float4(0.f, 0.f, 0.f, 0.f);
    long long wi0 = i0, wi1 = i1;
    warp_range(wi0, wi1);
    __syncthreads();
    const long long I0 = range[0], I1 = range[1];
    const int64_t qstride = static_cast<int64_t>(H) * hd;
    for (int h = g * G; h < (g + 1) * G; ++h) {
        const T* qh = static_cast<const T*>(p.q) + static_cast<int64_t>(h) * hd;
        const T* gh = dout + static_cast<int64_t>(h) * hd;
        for (long long c0 = I0; c0 < I1; c0 += kStage) {
            const int n = static_cast<int>(I1 - c0 < kStage ? I1 - c0 : kStage);
            __syncthreads();
            stage_rows<HP>(qs, qh, c0, n, qstride, hd);
            stage_rows<HP>(gs, gh, c0, n, qstride, hd);
            if (threadIdx.x < kStage) {
                const int r = threadIdx.x;
                ls[r] = r < n ? p.lse[(c0 + r) * H + h] * 1.4426950408889634f : 0.f;
                dd[r] = r < n ? dsum[(c0 + r) * H + h] : 0.f;
            }
            __syncthreads();
            if (c0 + n <= wi0 || c0 >= wi1) continue;  // warp-uniform
            for (int ii = 0; ii < n; ++ii) {
                const long long i = c0 + ii;
                const float4* qr = reinterpret_cast<const float4*>(qs + ii * HP);
                const float4* gr = reinterpret_cast<const float4*>(gs + ii * HP);
                float4 qq[NC], gg[NC];
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int t = 0; t < NC; ++t) {
                    qq[t] = qr[r8 + kLanesPerRow * t];
                    gg[t] = gr[r8 + kLanesPerRow * t];
                    s = dot4(kj[t], qq[t], s);
                    dp = dot4(vj[t], gg[t], dp);
                }
                group_sum2(s, dp);
                const float pij = (i >= i0 && i < i1) ? exp2f(fmaf(s, scale2, -ls[ii])) : 0.f;
                const float dsv = pij * (dp - dd[ii]) * p.scale;
#pragma unroll
                for (int t = 0; t < NC; ++t) {
                    axpy4(ak[t], dsv, qq[t]);
                    axpy4(av[t], pij, gg[t]);
                }
            }
        }
    }
    if (j < slots) {
        store_row<NC>(dk + krow * hd, ak, hd, r8);
        store_row<NC>(dv + krow * hd, av, hd, r8);
    }
}

// D_i = dO_i . O_i for every row (slot, head) of the slot view: 8 lanes per row, VEC elements per
// load (rows are 16-byte aligned when VEC > 1).
template <typename T, int VEC>
__global__ void __launch_bounds__(256) attn_bwd_dsum_kernel(const T* __restrict__ o,
                                                            const T* __restrict__ dout,
                                                            float* __restrict__ dsum, int64_t rows,
                                                            int hd) {
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t r = gid / kLanesPerRow;
    const int r8 = static_cast<int>(gid % kLanesPerRow);
    float acc = 0.f, acc2 = 0.f;
    if (r < rows) {
        const T* orow = o + r * hd;
        const T* grow = dout + r * hd;
        for (int e = r8 * VEC; e < hd; e += kLanesPerRow * VEC) {
            if (VEC == 1) {
                acc = fmaf(ld(orow + e), ld(grow + e), acc);
            } else {
                const uint4 a = __ldg(reinterpret_cast<const uint4*>(orow + e));
                const uint4 b = __ldg(reinterpret_cast<const uint4*>(grow + e));
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (sizeof(T) == 2) {
                        acc = fmaf(__uint_as_float(aw[w] << 16), __uint_as_float(bw[w] << 16), acc);
                        acc2 = fmaf(__uint_as_float(aw[w] & 0xFFFF0000u),
                                    __uint_as_float(bw[w] & 0xFFFF0000u), acc2);
                    } else {
                        acc = fmaf(__uint_as_float(aw[w]), __uint_as_float(bw[w]), acc);
                    }
                }
            }
        }
    }
    acc += acc2;
    float unused = 0.f;
    group_sum2(acc, unused);
    if (r < rows && r8 == 0) dsum[r] = acc;
}

// Zeros rows [0, cu[0] * mult) and [cu[batch] * mult, slots) (outside every document) of dq, dk,
// dv (bf16, row widths multiples of 8 elements).
__global__ void __launch_bounds__(256) attn_bwd_zero_outside_kernel(AttnProblem p,
                                                                    __nv_bfloat16* dq,
                                                                    __nv_bfloat16* dk,
                                                                    __nv_bfloat16* dv) {
    const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
    const int64_t head = min(static_cast<int64_t>(p.cu_seqlens[0]) * p.slot_mult, slots);
    const int64_t tail = max(min(static_cast<int64_t>(p.cu_seqlens[p.batch]) * p.slot_mult, slots),
                             head);
    const int64_t wq = static_cast<int64_t>(p.heads) * p.head_dim / 8;     // 16-byte units
    const int64_t wk = static_cast<int64_t>(p.kv_heads) * p.head_dim / 8;
    const int64_t rows = head + (slots - tail);
    const int64_t n = rows * (wq + 2 * wk);
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < n;
         x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t rr = x / (wq + 2 * wk), c = x % (wq + 2 * wk);
        const int64_t slot = rr < head ? rr : tail + (rr - head);
        if (c < wq) reinterpret_cast<uint4*>(dq)[slot * wq + c] = z;
        else if (c < wq + wk) reinterpret_cast<uint4*>(dk)[slot * wk + (c - wq)] = z;
        else reinterpret_cast<uint4*>(dv)[slot * wk + (c - wq - wk)] = z;
    }
}

template <int HP, typename T>
void launch_bwd_hp(const AttnProblem& p, const T* dout, const float* dsum, T* dq, T* dk, T* dv,
                   unsigned tiles, cudaStream_t stream) {
    const size_t smem_dq = 2 * static_cast<size_t>(kStage) * HP * sizeof(float);
    const size_t smem_kv = smem_dq + 2 * kStage * sizeof(float);
    attn_bwd_dq_kernel<HP, T><<<dim3(tiles, p.heads), kBwdThreads, smem_dq, stream>>>(p, dout, dsum, dq);
    attn_bwd_dkdv_kernel<HP, T><<<dim3(tiles, p.kv_heads), kBwdThreads, smem_kv, stream>>>(
        p, dout, dsum, dk, dv);
}

template <typename T>
void launch_bwd_t(const AttnProblem& p, const void* dout, const float* dsum, void* dq, void* dk, void* dv,
                  unsigned tiles, cudaStream_t stream) {
    const T* go = static_cast<const T*>(dout);
    T *a = static_cast<T*>(dq), *b = static_cast<T*>(dk), *c = static_cast<T*>(dv);
    if (p.head_dim <= 32) launch_bwd_hp<32>(p, go, dsum, a, b, c, tiles, stream);
    else if (p.head_dim <= 64) launch_bwd_hp<64>(p, go, dsum, a, b, c, tiles, stream);
    else launch_bwd_hp<128>(p, go, dsum, a, b, c, tiles, stream);
}

}  // namespace

cudaError_t launch_attn_bwd_dsum(const AttnProblem& p, const void* o, const void* dout,
                                 float* dsum, int is_bf16, cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(p.total_tokens) * p.slot_mult * p.heads;
    if (rows == 0) return cudaSuccess;
    const int hd = p.head_dim;
    const unsigned blocks = static_cast<unsigned>((rows * kLanesPerRow + 255) / 256);
    if (is_bf16) {
        const auto* a = static_cast<const __nv_bfloat16*>(o);
        const auto* b = static_cast<const __nv_bfloat16*>(dout);
        if (hd % 8 == 0) attn_bwd_dsum_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, stream>>>(a, b, dsum, rows, hd);
        else attn_bwd_dsum_kernel<__nv_bfloat16, 1><<<blocks, 256, 0, stream>>>(a, b, dsum, rows, hd);
    } else {
        const auto* a = static_cast<const float*>(o);
        const auto* b = static_cast<const float*>(dout);
        if (hd % 4 == 0) attn_bwd_dsum_kernel<float, 4><<<blocks, 256, 0, stream>>>(a, b, dsum, rows, hd);
        else attn_bwd_dsum_kernel<float, 1><<<blocks, 256, 0, stream>>>(a, b, dsum, rows, hd);
    }
    return cudaGetLastError();
}

cudaError_t launch_attn_bwd_zero_outside(const AttnProblem& p, void* dq, void* dk, void* dv,
                                         cudaStream_t stream) {
    if (p.total_tokens == 0) return cudaSuccess;
    attn_bwd_zero_outside_kernel<<<148, 256, 0, stream>>>(p, static_cast<__nv_bfloat16*>(dq),
                                                          static_cast<__nv_bfloat16*>(dk),
                                                          static_cast<__nv_bfloat16*>(dv));
    return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const AttnProblem& p, const void* dout, const float* dsum, void* dq,
                            void* dk, void* dv, int is_bf16, cudaStream_t stream) {
    const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
    if (slots == 0) return cudaSuccess;
    if (p.head_dim > 128) return cudaErrorInvalidValue;
    const unsigned tiles = static_cast<unsigned>((slots + kRowsPerBlock - 1) / kRowsPerBlock);
    if (is_bf16) launch_bwd_t<__nv_bfloat16>(p, dout, dsum, dq, dk, dv, tiles, stream);
    else launch_bwd_t<float>(p, dout, dsum, dq, dk, dv, tiles, stream);
    return cudaGetLastError();
}

}  // namespace pha
