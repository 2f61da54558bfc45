// attn_bwd.cu -- backward of the varlen (paired-head) attention forward: dq, dk, dv for an upstream
// gradient dO, on CUDA cores in float32.
//
// The gradients through the row softmax (with P the attention weights of the forward,
// P_ij = exp(scale q_i . k_j - lse_i) over the visible keys):
//   dP_ij = dO_i . v_j,  D_i = sum_j P_ij dP_ij,  dS_ij = P_ij (dP_ij - D_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dO_i.
// P is recomputed from q, k and the forward's lse (FlashAttention's recomputation: "Training an
// LLM from scratch (part 2)", section "4. GQA & FlashAttention" -- no score matrix is stored).
// The paired-head variant is the same slot view of the buffers and the same doubled documents as
// the forward ("modded-nanogpt Paired Head Attention record" page, sections "3. the paired branch
// of the forward pass" and "sequence length and window handling").
//
// Two kernels, no atomics:
//   dq   (query-major): one warp per (query slot, head). Pass 1 over the visible keys gives D_i,
//        pass 2 accumulates dq_i; D_i is stored for the second kernel.
//   dkdv (key-major):   one warp per (key slot, kv head), over the visible queries of every query
//        head of the kv group, accumulating dk_j and dv_j.
// Lane l holds elements l, l + 32, ... of a head row (any head_dim <= 128); the two dot products of
// a (query, key) pair are reduced together with one 64-bit shuffle per step.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.cuh"

namespace pha {

namespace {

constexpr int kBwdMaxE = 4;  // elements per lane: head_dim <= 128

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

// Sum of (a, b) over the warp (both results in every lane).
__device__ __forceinline__ void warp_sum2(float& a, float& b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long v =
            (static_cast<unsigned long long>(__float_as_uint(b)) << 32) | __float_as_uint(a);
        const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
        a += __uint_as_float(static_cast<uint32_t>(w));
        b += __uint_as_float(static_cast<uint32_t>(w >> 32));
    }
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

template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(AttnProblem p, const T* __restrict__ dout,
                                                           float* __restrict__ dsum,
                                                           T* __restrict__ dq) {
    const int lane = threadIdx.x & 31;
    const int H = p.heads, Hkv = p.kv_heads, hd = p.head_dim, G = H / Hkv;
    const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
    const int64_t n_rows = slots * H;
    const int64_t warp0 = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const T* q = static_cast<const T*>(p.q);
    const T* k = static_cast<const T*>(p.k);
    const T* v = static_cast<const T*>(p.v);
    const float scale = p.scale, log2e = 1.4426950408889634f;
    for (int64_t row = warp0; row < n_rows; row += n_warps) {
        const int64_t i = row / H;
        const int h = static_cast<int>(row - i * H), g = h / G;
        int64_t lo, hi;
        float qi[kBwdMaxE], gi[kBwdMaxE], acc[kBwdMaxE];
        const bool in_doc = doc_of_slot(p, i, lo, hi);
#pragma unroll
        for (int e = 0; e < kBwdMaxE; ++e) {
            const int c = lane + 32 * e;
            qi[e] = (in_doc && c < hd) ? ld(q + row * hd + c) : 0.f;
            gi[e] = (in_doc && c < hd) ? ld(dout + row * hd + c) : 0.f;
            acc[e] = 0.f;
        }
        float d = 0.f;
        if (in_doc) {
            const float lse2 = p.lse[row] * log2e;
            int64_t j0 = lo, j1 = hi;  // visible keys [j0, j1)
            if (p.causal) {
                j1 = i + 1;
                if (p.window > 0 && i - p.window + 1 > j0) j0 = i - p.window + 1;
            }
            // pass 1: D_i = sum_j P_ij dP_ij
            for (int64_t j = j0; j < j1; ++j) {
                const T* kj = k + (j * Hkv + g) * hd;
                const T* vj = v + (j * Hkv + g) * hd;
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int e = 0; e < kBwdMaxE; ++e) {
                    const int c = lane + 32 * e;
                    if (c < hd) {
                        s = fmaf(qi[e], ld(kj + c), s);
                        dp = fmaf(gi[e], ld(vj + c), dp);
                    }
                }
                warp_sum2(s, dp);
                d = fmaf(exp2f(s * scale * log2e - lse2), dp, d);
            }
            // pass 2: dq_i = scale sum_j P_ij (dP_ij - D_i) k_j
            for (int64_t j = j0; j < j1; ++j) {
                const T* kj = k + (j * Hkv + g) * hd;
                const T* vj = v + (j * Hkv + g) * hd;
                float kv[kBwdMaxE];
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int e = 0; e < kBwdMaxE; ++e) {
                    const int c = lane + 32 * e;
                    kv[e] = c < hd ? ld(kj + c) : 0.f;
                    s = fmaf(qi[e], kv[e], s);
                    dp = fmaf(gi[e], c < hd ? ld(vj + c) : 0.f, dp);
                }
                warp_sum2(s, dp);
                const float ds = exp2f(s * scale * log2e - lse2) * (dp - d) * scale;
#pragma unroll
                for (int e = 0; e < kBwdMaxE; ++e) acc[e] = fmaf(ds, kv[e], acc[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < kBwdMaxE; ++e) {
            const int c = lane + 32 * e;
            if (c < hd) st(dq + row * hd + c, acc[e]);
        }
        if (lane == 0) dsum[row] = d;
    }
}

template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_dkdv_kernel(AttnProblem p, const T* __restrict__ dout,
                                                             const float* __restrict__ dsum,
                                                             T* __restrict__ dk, T* __restrict__ dv) {
    const int lane = threadIdx.x & 31;
    const int H = p.heads, Hkv = p.kv_heads, hd = p.head_dim, G = H / Hkv;
    const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
    const int64_t n_rows = slots * Hkv;
    const int64_t warp0 = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const T* q = static_cast<const T*>(p.q);
    const T* k = static_cast<const T*>(p.k);
    const T* v = static_cast<const T*>(p.v);
    const float scale = p.scale, log2e = 1.4426950408889634f;
    for (int64_t row = warp0; row < n_rows; row += n_warps) {
        const int64_t j = row / Hkv;
        const int g = static_cast<int>(row - j * Hkv);
        int64_t lo, hi;
        float kj[kBwdMaxE], vj[kBwdMaxE], ak[kBwdMaxE], av[kBwdMaxE];
        const bool in_doc = doc_of_slot(p, j, lo, hi);
#pragma unroll
        for (int e = 0; e < kBwdMaxE; ++e) {
            const int c = lane + 32 * e;
            kj[e] = (in_doc && c < hd) ? ld(k + row * hd + c) : 0.f;
            vj[e] = (in_doc && c < hd) ? ld(v + row * hd + c) : 0.f;
            ak[e] = av[e] = 0.f;
        }
        if (in_doc) {
            int64_t i0 = lo, i1 = hi;  // queries that see key j: [i0, i1)
            if (p.causal) {
                i0 = j;
                if (p.window > 0 && j + p.window < i1) i1 = j + p.window;
            }
            for (int h = g * G; h < (g + 1) * G; ++h) {
                for (int64_t i = i0; i < i1; ++i) {
                    const int64_t qrow = i * H + h;
                    const T* qi = q + qrow * hd;
                    const T* gi = dout + qrow * hd;
                    float qv[kBwdMaxE], gv[kBwdMaxE];
                    float s = 0.f, dp = 0.f;
#pragma unroll
                    for (int e = 0; e < kBwdMaxE; ++e) {
                        const int c = lane + 32 * e;
                        qv[e] = c < hd ? ld(qi + c) : 0.f;
                        gv[e] = c < hd ? ld(gi + c) : 0.f;
                        s = fmaf(qv[e], kj[e], s);
                        dp = fmaf(gv[e], vj[e], dp);
                    }
                    warp_sum2(s, dp);
                    const float pij = exp2f((s * scale - __ldg(p.lse + qrow)) * log2e);
                    const float ds = pij * (dp - __ldg(dsum + qrow)) * scale;
#pragma unroll
                    for (int e = 0; e < kBwdMaxE; ++e) {
                        ak[e] = fmaf(ds, qv[e], ak[e]);
                        av[e] = fmaf(pij, gv[e], av[e]);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < kBwdMaxE; ++e) {
            const int c = lane + 32 * e;
            if (c < hd) {
                st(dk + row * hd + c, ak[e]);
                st(dv + row * hd + c, av[e]);
            }
        }
    }
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnProblem& p, const void* dout, float* dsum, void* dq, void* dk,
                            void* dv, int is_bf16, cudaStream_t stream) {
    const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
    if (slots == 0) return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int threads = 256;
    auto grid_for = [&](int64_t rows) {
        const int64_t blocks = (rows * 32 + threads - 1) / threads;
        const int64_t cap = static_cast<int64_t>(sms) * 16;
        return static_cast<int>(blocks < cap ? blocks : cap);
    };
    if (is_bf16) {
        attn_bwd_dq_kernel<__nv_bfloat16><<<grid_for(slots * p.heads), threads, 0, stream>>>(
            p, static_cast<const __nv_bfloat16*>(dout), dsum, static_cast<__nv_bfloat16*>(dq));
        attn_bwd_dkdv_kernel<__nv_bfloat16><<<grid_for(slots * p.kv_heads), threads, 0, stream>>>(
            p, static_cast<const __nv_bfloat16*>(dout), dsum, static_cast<__nv_bfloat16*>(dk),
            static_cast<__nv_bfloat16*>(dv));
    } else {
        attn_bwd_dq_kernel<float><<<grid_for(slots * p.heads), threads, 0, stream>>>(
            p, static_cast<const float*>(dout), dsum, static_cast<float*>(dq));
        attn_bwd_dkdv_kernel<float><<<grid_for(slots * p.kv_heads), threads, 0, stream>>>(
            p, static_cast<const float*>(dout), dsum, static_cast<float*>(dk), static_cast<float*>(dv));
    }
    return cudaGetLastError();
}

}  // namespace pha
