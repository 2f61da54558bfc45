// attn_tc.cu -- bf16 attention forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every scheduled (query tile, head) work item, O = softmax(scale * Q K^T) V over
// the visible keys and the row log-sum-exp, with the online (running max / running sum) softmax
// of FlashAttention ("Training an LLM from scratch (part 2)", section "4. GQA & FlashAttention":
// tiled, exact, no score matrix in HBM). The paired-head variant needs nothing here: the caller's
// buffers are read as the [2T][H/2][hd] slot view and the scheduler doubles the documents
// ("modded-nanogpt Paired Head Attention record" page, sections "3. the paired branch of the
// forward pass" and "sequence length and window handling").
//
// CTA = 6 warps, persistent (one CTA per SM, static round-robin over the longest-first work list):
//   warp 4      TMA producer: Q tile (2 buffers) and K / V tiles (kStages-deep rings), 64x128
//               boxes with 128-byte swizzle.
//   warp 5      MMA issuer (one thread): S = Q K^T into one of two TMEM S buffers
//               (M=128, N=128, K=hd), then O += P V into TMEM (M=128, N=hd, K=128).
//               Also owns the TMEM allocation (512 columns).
//   warps 0-3   softmax: thread r owns query row r (= TMEM lane r). Reads its S row from TMEM,
//               masks boundary tiles only, updates the running max / sum, rescales its O row in
//               TMEM only when the max grew by more than 2^8, writes P (bf16) to a swizzled
//               shared tile, and at the end normalises O and writes O and the LSE.
// Every wait is bounded (1 s); on expiry the CTA records a status, drains its own in-flight
// copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.cuh"

namespace pha {

template <int HD>
struct TcLayout {
    static constexpr int kChunk = 128 * 128;  // one [128 rows][64 bf16] swizzled chunk (bytes)
    static constexpr int kQBytes = kBlockM * HD * 2;
    static constexpr int kKVBytes = kBlockN * HD * 2;
    static constexpr int kPBytes = kBlockM * kBlockN * 2;
    static constexpr int kStages = HD == 128 ? 2 : 3;
    static constexpr int kQBufs = 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBufs * kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffP = kOffV + kStages * kKVBytes;
    static constexpr int kOffBar = kOffP + kPBytes;
    static constexpr int kBarBytes = 512;
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + slack to align to 1024
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kTmS = 0;  // S buffer b at columns kTmS + 128 * b
    static constexpr uint32_t kTmO = 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct TcBars {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full, pv_done, drain;
    uint32_t tmem_base;
    int abort;
};

constexpr int kTcThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Drain wait used on the exit path: bounded, ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_test(bar, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs) return;
}

// K-major 128-row tile (Q, K or P): k-step kk covers 16 bf16 of the contraction dimension.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
}
// MN-major V tile ([keys][hd] in 64-column chunks): k-step kk covers 16 keys.
__device__ __forceinline__ uint64_t desc_v(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + kk * 2048, 16384, 1024);
}

template <int HD>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnProblem p,
                   const int4* __restrict__ items, WorkspaceHeader* hdr) {
    using L = TcLayout<HD>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const uint32_t sbase = smem_u32(smem);
    TcBars* bars = reinterpret_cast<TcBars*>(smem + L::kOffBar);
    volatile int* abort_flag = &bars->abort;
    int* dev_status = &hdr->status;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 4 && lane == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->s_free[b], 128);
        }
        for (int s = 0; s < 3; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 5) {
        tmem_alloc(&bars->tmem_base, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    const int n_items = *reinterpret_cast<volatile int*>(&hdr->n_items);
    const int H = p.heads;
    const int G = p.heads / p.kv_heads;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t q_cnt = 0, kv_cnt = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const int4 w = __ldg(items + it);
                const int head = w.y >> 16;
                const int g = head / G;
                const int n_kv = (w.w - w.z + kBlockN - 1) / kBlockN;
                const uint32_t qb = q_cnt & 1;
                if (!mbar_wait(&bars->q_empty[qb], ((q_cnt >> 1) & 1) ^ 1, abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars->q_full[qb], L::kQBytes);
                for (int c = 0; c < HD / 64; ++c)
                    tma_load_2d(smem + L::kOffQ + qb * L::kQBytes + c * L::kChunk, &tm_q,
                                head * HD + 64 * c, w.x, &bars->q_full[qb]);
                ++q_cnt;
                for (int t = 0; t < n_kv; ++t) {
                    const uint32_t s = kv_cnt % L::kStages;
                    const uint32_t ph = (kv_cnt / L::kStages) & 1;
                    const int row = w.z + t * kBlockN;
                    if (!mbar_wait(&bars->k_empty[s], ph ^ 1, abort_flag, dev_status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bars->k_full[s], L::kKVBytes);
                    for (int c = 0; c < HD / 64; ++c)
                        tma_load_2d(smem + L::kOffK + s * L::kKVBytes + c * L::kChunk, &tm_k,
                                    g * HD + 64 * c, row, &bars->k_full[s]);
                    if (!mbar_wait(&bars->v_empty[s], ph ^ 1, abort_flag, dev_status)) {
                        ++kv_cnt;  // K of this tile is in flight
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->v_full[s], L::kKVBytes);
                    for (int c = 0; c < HD / 64; ++c)
                        tma_load_2d(smem + L::kOffV + s * L::kKVBytes + c * L::kChunk, &tm_v,
                                    g * HD + 64 * c, row, &bars->v_full[s]);
                    ++kv_cnt;
                }
            }
            if (!ok) {
                // Wait (bounded) for the copies this thread issued last on every buffer.
                for (uint32_t n = (q_cnt > 2 ? q_cnt - 2 : 0); n < q_cnt; ++n)
                    drain_wait(&bars->q_full[n & 1], (n >> 1) & 1);
                for (uint32_t n = (kv_cnt > L::kStages ? kv_cnt - L::kStages : 0); n < kv_cnt; ++n) {
                    drain_wait(&bars->k_full[n % L::kStages], (n / L::kStages) & 1);
                    drain_wait(&bars->v_full[n % L::kStages], (n / L::kStages) & 1);
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, HD, 0, 1);
            const uint32_t q_tile0 = sbase + L::kOffQ, k_tile0 = sbase + L::kOffK;
            const uint32_t v_tile0 = sbase + L::kOffV, p_tile = sbase + L::kOffP;
            uint32_t q_cnt = 0, kv_cnt = 0, s_cnt = 0, pv_cnt = 0;
            bool ok = true;
            auto issue_pv = [&](uint32_t kv_index, bool first) -> bool {
                if (!mbar_wait(&bars->p_full, pv_cnt & 1, abort_flag, dev_status)) return false;
                const uint32_t s = kv_index % L::kStages;
                if (!mbar_wait(&bars->v_full[s], (kv_index / L::kStages) & 1, abort_flag, dev_status))
                    return false;
                tc_fence_after();
                const uint32_t v_tile = v_tile0 + s * L::kKVBytes;
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk)
                    umma_f16_ss(tmem + L::kTmO, desc_kmajor(p_tile, kk), desc_v(v_tile, kk), idesc_pv,
                                (first && kk == 0) ? 0u : 1u);
                umma_commit(&bars->pv_done);
                umma_commit(&bars->v_empty[s]);
                ++pv_cnt;
                return true;
            };
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const int4 w = __ldg(items + it);
                const int n_kv = (w.w - w.z + kBlockN - 1) / kBlockN;
                const uint32_t qb = q_cnt & 1;
                if (!mbar_wait(&bars->q_full[qb], (q_cnt >> 1) & 1, abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t q_tile = q_tile0 + qb * L::kQBytes;
                const uint32_t kv_base = kv_cnt;
                for (int t = 0; t < n_kv; ++t) {
                    const uint32_t kv_index = kv_base + t;
                    const uint32_t s = kv_index % L::kStages;
                    const uint32_t sb = s_cnt & 1;
                    if (!mbar_wait(&bars->s_free[sb], ((s_cnt >> 1) & 1) ^ 1, abort_flag, dev_status) ||
                        !mbar_wait(&bars->k_full[s], (kv_index / L::kStages) & 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_tile = k_tile0 + s * L::kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_f16_ss(tmem + L::kTmS + 128 * sb, desc_kmajor(q_tile, kk), desc_kmajor(k_tile, kk),
                                    idesc_qk, kk == 0 ? 0u : 1u);
                    umma_commit(&bars->s_full[sb]);
                    umma_commit(&bars->k_empty[s]);
                    if (t == n_kv - 1) umma_commit(&bars->q_empty[qb]);
                    ++s_cnt;
                    if (t > 0 && !issue_pv(kv_index - 1, t == 1)) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                if (!issue_pv(kv_base + n_kv - 1, n_kv == 1)) {
                    ok = false;
                    break;
                }
                kv_cnt += n_kv;
                ++q_cnt;
            }
            // Wait (bounded) until every MMA this thread issued has finished.
            umma_commit(&bars->drain);
            drain_wait(&bars->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps 0-3
        const int row = threadIdx.x;  // query row in the tile == TMEM lane
        const uint32_t tm_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float scale_log2 = p.scale * kLog2e;
        const int window = p.window;
        uint8_t* p_tile = smem + L::kOffP;
        uint32_t s_cnt = 0, p_cnt = 0;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const int4 w = __ldg(items + it);
            const int q0 = w.x, head = w.y >> 16, n_q = w.y & 0xFFFF;
            const int kv_lo = w.z, kv_hi = w.w;
            const int n_kv = (kv_hi - kv_lo + kBlockN - 1) / kBlockN;
            const int i = q0 + row;
            // visible key slots of this row: [j_min, j_max]
            const int j_max = p.causal ? min(i, kv_hi - 1) : kv_hi - 1;
            const int j_min = window > 0 ? i - window + 1 : INT32_MIN / 2;
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int t = 0; t < n_kv && ok; ++t) {
                const int kv0 = kv_lo + t * kBlockN;
                const uint32_t sb = s_cnt & 1;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars->s_full[sb], (s_cnt >> 1) & 1, abort_flag, dev_status));
                if (!ok) break;
                tc_fence_after();
                float s[kBlockN];
                {
                    uint32_t r[kBlockN];
#pragma unroll
                    for (int c = 0; c < kBlockN / 32; ++c)
                        tmem_ld32(tm_lane + L::kTmS + 128 * sb + 32 * c, r + 32 * c);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < kBlockN; ++e) s[e] = __uint_as_float(r[e]);
                }
                tc_fence_before();
                mbar_arrive(&bars->s_free[sb]);
                ++s_cnt;

                const bool full_tile = (kv0 + kBlockN - 1 < kv_hi) &&
                                       (!p.causal || kv0 + kBlockN - 1 <= q0) &&
                                       (window <= 0 || (q0 + n_q - 1) - kv0 < window);
                if (!full_tile) {
                    const int c_lo = j_min - kv0, c_hi = j_max - kv0;
#pragma unroll
                    for (int c = 0; c < kBlockN; ++c)
                        if (c < c_lo || c > c_hi) s[c] = -INFINITY;
                }
                float mx = s[0];
#pragma unroll
                for (int c = 1; c < kBlockN; ++c) mx = fmaxf(mx, s[c]);
                const float m_new = fmaxf(m, mx * scale_log2);
                // Keep the reference max until the row max grows by more than 8 (a factor 256):
                // the final O / l and lse are exact for any reference value.
                const bool rescale = m_new > m + 8.0f;
                const float alpha = rescale ? ex2(m - m_new) : 1.0f;
                if (rescale) m = m_new;
                const float m_safe = (m == -INFINITY) ? 0.f : m;
                float sum = 0.f;
#pragma unroll
                for (int c = 0; c < kBlockN; ++c) {
                    s[c] = ex2(fmaf(s[c], scale_log2, -m_safe));
                    sum += s[c];
                }
                l = l * alpha + sum;

                // P buffer and O are ours once the previous P.V has finished.
                if (p_cnt > 0) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&bars->pv_done, (p_cnt - 1) & 1, abort_flag, dev_status));
                    if (!ok) break;
                    tc_fence_after();
                }
                if (t > 0 && __any_sync(0xffffffffu, rescale)) {
                    uint32_t r[32];
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        tmem_ld32(tm_lane + L::kTmO + 32 * c, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(tm_lane + L::kTmO + 32 * c, r);
                    }
                    tmem_wait_st();
                }
                // P row -> shared memory, K-major with the 128-byte swizzle of the MMA operand.
#pragma unroll
                for (int c16 = 0; c16 < kBlockN / 8; ++c16) {
                    const uint4 v4 = make_uint4(pack_bf16x2(s[8 * c16 + 0], s[8 * c16 + 1]),
                                                pack_bf16x2(s[8 * c16 + 2], s[8 * c16 + 3]),
                                                pack_bf16x2(s[8 * c16 + 4], s[8 * c16 + 5]),
                                                pack_bf16x2(s[8 * c16 + 6], s[8 * c16 + 7]));
                    const int off = (c16 >> 3) * 16384 + row * 128 + (((c16 & 7) ^ (row & 7)) << 4);
                    *reinterpret_cast<uint4*>(p_tile + off) = v4;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bars->p_full);
                ++p_cnt;
            }
            if (!ok) break;
            // epilogue: O / l and lse for the valid rows
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars->pv_done, (p_cnt - 1) & 1, abort_flag, dev_status));
            if (!ok) break;
            tc_fence_after();
            const bool valid = row < n_q;
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) +
                                  (static_cast<int64_t>(i) * H + head) * HD;
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                tmem_ld32(tm_lane + L::kTmO + 32 * c, r);
                tmem_wait_ld();
                if (valid) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                            __uint_as_float(r[2 * e + 1]) * inv_l);
                    uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
                    dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
                }
            }
            if (valid && p.lse) p.lse[static_cast<int64_t>(i) * H + head] = (m + log2f(l)) * kLn2;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, L::kTmemCols);
}

template <int HD>
static cudaError_t launch_tc_hd(const AttnProblem& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const int4* items, WorkspaceHeader* hdr,
                                cudaStream_t stream) {
    using L = TcLayout<HD>;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    attn_tc_kernel<HD><<<sms, kTcThreads, L::kSmemBytes, stream>>>(tq, tk, tv, p, items, hdr);
    return cudaGetLastError();
}

cudaError_t launch_attn_tc(const AttnProblem& p, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, const int4* items, WorkspaceHeader* hdr,
                           cudaStream_t stream) {
    if (p.head_dim == 128) return launch_tc_hd<128>(p, tm_q, tm_k, tm_v, items, hdr, stream);
    if (p.head_dim == 64) return launch_tc_hd<64>(p, tm_q, tm_k, tm_v, items, hdr, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pha
