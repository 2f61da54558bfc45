// attn_f32.cu -- exact float32 attention forward on CUDA cores (the fp32 path; small problems).
//
// One thread per (query slot, head) row: a single pass over the visible keys with the running
// max / running sum of the online softmax, all in IEEE float32 (no approximate exponentials, no
// tensor cores, whose reduced-precision inputs could not meet a 1e-5 relative bound).
// Semantics as the bf16 tensor-core kernel: causal, optional window counted in key slots,
// varlen documents, GQA, and the paired head view (slot 2t + h/(H/2)).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.cuh"

namespace pha {

constexpr int kMaxHeadDimF32 = 128;

__global__ void __launch_bounds__(128) attn_f32_kernel(AttnProblem p, int64_t n_rows) {
    const int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (r >= n_rows) return;
    const int H = p.heads, Hkv = p.kv_heads, D = p.head_dim;
    const int64_t i = r / H;  // query slot
    const int h = static_cast<int>(r % H);
    const int g = h / (H / Hkv);
    // document of slot i: last b with cu[b] * mult <= i
    int a = 0, z = p.batch;
    while (z - a > 1) {
        const int mid = (a + z) >> 1;
        if (static_cast<int64_t>(p.cu_seqlens[mid]) * p.slot_mult <= i) a = mid; else z = mid;
    }
    const int64_t doc_lo = static_cast<int64_t>(p.cu_seqlens[a]) * p.slot_mult;
    const int64_t doc_hi = static_cast<int64_t>(p.cu_seqlens[a + 1]) * p.slot_mult;
    if (i < doc_lo || i >= doc_hi) return;  // slot outside every document: not an output row
    int64_t lo = doc_lo, hi = doc_hi;
    if (p.causal) {
        hi = i + 1;
        if (p.window > 0 && i - p.window + 1 > lo) lo = i - p.window + 1;
    }
    const float* q = static_cast<const float*>(p.q) + (i * H + h) * D;
    const float* kb = static_cast<const float*>(p.k);
    const float* vb = static_cast<const float*>(p.v);
    float qr[kMaxHeadDimF32], acc[kMaxHeadDimF32];
    for (int d = 0; d < D; ++d) {
        qr[d] = q[d];
        acc[d] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int64_t j = lo; j < hi; ++j) {
        const float* kj = kb + (j * Hkv + g) * D;
        float s = 0.f;
        for (int d = 0; d < D; ++d) s = fmaf(qr[d], kj[d], s);
        s *= p.scale;
        if (s > m) {
            const float corr = expf(m - s);  // 0 on the first visible key
            l *= corr;
            for (int d = 0; d < D; ++d) acc[d] *= corr;
            m = s;
        }
        const float e = expf(s - m);
        l += e;
        const float* vj = vb + (j * Hkv + g) * D;
        for (int d = 0; d < D; ++d) acc[d] = fmaf(e, vj[d], acc[d]);
    }
    float* o = static_cast<float*>(p.o) + (i * H + h) * D;
    const float inv = 1.f / l;
    for (int d = 0; d < D; ++d) o[d] = acc[d] * inv;
    if (p.lse) p.lse[i * H + h] = m + logf(l);
}

cudaError_t launch_attn_f32(const AttnProblem& p, cudaStream_t stream) {
    const int64_t n_rows = static_cast<int64_t>(p.total_tokens) * p.slot_mult * p.heads;
    if (n_rows == 0) return cudaSuccess;
    const int threads = 128;
    const int64_t blocks = (n_rows + threads - 1) / threads;
    attn_f32_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(p, n_rows);
    return cudaGetLastError();
}

}  // namespace pha
