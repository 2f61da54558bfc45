// attn_tc.cu -- bf16 attention forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every scheduled (query block, head) work item, O = softmax(scale * Q K^T) V over
// the visible keys and the row log-sum-exp, with the online (running max / running sum) softmax
// of FlashAttention ("Training an LLM from scratch (part 2)", section "4. GQA & FlashAttention":
// tiled, exact, no score matrix in HBM). The paired-head variant needs nothing here: the caller's
// buffers are read as the [2T][H/2][hd] slot view and the scheduler doubles the documents
// ("modded-nanogpt Paired Head Attention record" page, sections "3. the paired branch of the
// forward pass" and "sequence length and window handling").
//
// A work item is a block of up to 256 query slots split into two 128-row sub-tiles r = 0, 1 that
// share one stream of 128-key K / V tiles. CTA = 12 warps, persistent (one CTA per SM; the
// longest-first work list is dealt out in snake order); the softmax warpgroups run with 200
// registers per thread, the third warpgroup with 88:
//   warps 0-3   softmax of sub-tile 0      warps 4-7   softmax of sub-tile 1
//               thread = query row = TMEM lane. The whole 128-column S row is loaded from TMEM
//               with one wait, its max and its exponentials are taken from registers with
//               independent accumulator chains, and P (bf16) is written back to TMEM. Masks are
//               applied only on tiles that straddle a causal / window / document edge, per
//               32-column chunk and only where some row of the warp needs them. O is rescaled in
//               TMEM only when the running max grew by more than 2^8. At the end the row is
//               normalised and O and the LSE are stored.
//   warp 8      TMA producer: Q sub-tiles into a ring of 3 slots (so the next item's Q arrives
//               while the current item computes), K and V tiles into their rings (64-column x
//               128-row boxes, 128-byte swizzle; FP8: one hd-byte x 128-row box per tile, V into
//               an unswizzled staging ring).
//   warp 9      MMA issuer (one thread) and TMEM owner (512 columns)
//   warps 10-11 FP8: widen each landed e4m3 V tile to f16; value embedding: add aux_v's rows to
//               each landed V tile (rounded to bf16 as a bf16 tensor addition); otherwise idle
//   S and P.V, per sub-tile:
//               S_r = Q_r K^T   tcgen05.mma kind::f16 (FP8: kind::f8f6f4 on e4m3 tiles), A and B
//                               from shared memory, M=128 N=128
//               O_r += P_r V    tcgen05.mma kind::f16 (bf16; FP8: f16 P and V), A (P) from TMEM,
//                               B (V) from shared memory
//               The issue order is software-pipelined per sub-tile: once P_r of key tile g-1 is
//               ready, O_r += P_r V_{g-1} is issued and then at once S_r of key tile g, so sub-tile
//               r's next softmax starts while the other sub-tile's softmax is still running and
//               the tensor core alternates between the two. A sub-tile skips the key tiles that
//               lie wholly outside its own causal / window range.
// TMEM columns: S_r at 128 r, O_r at 256 + hd r. P_r: hd 64 -- columns 384 + 64 r, apart from S_r,
// so S_r of the next tile never waits for the P.V that reads P_r; hd 128 -- the first 64 columns
// of S_r (all 512 columns are taken), so before S_r of the next tile is issued the MMA thread
// waits until that P.V has completed.
// Ordering: the commit that signals S_r of a tile (s_full[r]) follows the previous tile's
// O_r += P_r V, so when the softmax sees S_r, that P.V is complete: P_r may be overwritten and O_r
// rescaled. At a work item's first key tile the P.V products that end the previous item's
// sub-tiles are issued before anything of the new item is awaited (their epilogues free the Q
// slots the producer waits for).
// Every wait is bounded (1 s); on expiry the CTA records a status, drains its own in-flight
// copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_common.cuh"
#include "kernels.cuh"

namespace pha {

// A decoded work item and the per-sub-tile key ranges (identical in every role).
struct Item {
    int q0, n_q, head, kv_lo, kv_hi, n_kv, n_sub;
    int nr[2];                  // valid rows of sub-tile r (0 = sub-tile absent)
    int t_first[2], t_last[2];  // key tiles sub-tile r needs
};

__device__ __forceinline__ Item decode_item(int4 w, const AttnProblem& p) {
    Item it;
    it.q0 = w.x;
    it.head = w.y >> 16;
    it.n_q = w.y & 0xFFFF;
    it.kv_lo = w.z;
    it.kv_hi = w.w;
    it.n_kv = (w.w - w.z + kBlockN - 1) / kBlockN;
    it.n_sub = it.n_q > kBlockM ? 2 : 1;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int qr0 = it.q0 + kBlockM * r;
        int nr = it.n_q - kBlockM * r;
        nr = nr < 0 ? 0 : (nr > kBlockM ? kBlockM : nr);
        it.nr[r] = nr;
        int lo = it.kv_lo, hi = it.kv_hi;
        if (p.causal) {
            hi = qr0 + nr;
            if (p.window > 0 && qr0 - p.window + 1 > lo) lo = qr0 - p.window + 1;
        }
        it.t_first[r] = (lo - it.kv_lo) / kBlockN;
        it.t_last[r] = nr > 0 ? (hi - 1 - it.kv_lo) / kBlockN : -1;
    }
    return it;
}

// Shared memory of the block kernel. bf16: Q slots, K and V rings of [hd / 64][128 rows][128 B]
// chunks. FP8: Q and K tiles hold e4m3 ([128 rows][hd B], one swizzled box), V arrives as e4m3
// in a staging ring ([128 rows][hd B], unswizzled) and is widened to f16 into the V ring, which
// has the bf16 layout.
template <int HD, bool F8>
struct BlockLayout {
    static constexpr int kChunk = 128 * 128;  // one [128 rows][64 x 16-bit] swizzled chunk
    static constexpr int kQSub = kBlockM * HD * (F8 ? 1 : 2);
    static constexpr int kK = kBlockN * HD * (F8 ? 1 : 2);
    static constexpr int kV = kBlockN * HD * 2;
    static constexpr int kV8 = F8 ? kBlockN * HD : 0;
    static constexpr int kQSlots = 3;
    static constexpr int kKStages = (F8 || HD == 64) ? 4 : 2;
    static constexpr int kVStages = (!F8 && HD == 64) ? 4 : 2;
    static constexpr int kV8Stages = F8 ? 2 : 1;  // (kV8 = 0 without FP8: no space)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQSlots * kQSub;
    static constexpr int kOffV = kOffK + kKStages * kK;
    static constexpr int kOffV8 = kOffV + kVStages * kV;
    static constexpr int kOffBar = kOffV8 + kV8Stages * kV8;
    static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // barriers + slack to align to 1024
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kTmO = 256;
    // rows of a warp staged at a time in the epilogue (O as bf16 through the Q slot)
    static constexpr int kStageRows = kQSub / (4 * HD * 2) < 32 ? kQSub / (4 * HD * 2) : 32;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(sizeof(TcBars) <= 512, "barrier block");
    static_assert(kStageRows == 16 || kStageRows == 32, "epilogue staging");
};

// Converter warps (FP8): e4m3 V tile [128 rows][HD B] -> f16 in the V ring's layout; thread t of
// 64 takes 16-byte units t, t + 64, ... (16 values of one row each).
template <int HD>
__device__ __forceinline__ void widen_v_tile(const uint8_t* v8, uint8_t* vh, int t) {
    constexpr int kUnitsPerRow = HD / 16;
    constexpr int kUnits = kBlockN * kUnitsPerRow;
#pragma unroll 4
    for (int u = t; u < kUnits; u += 64) {
        const int r = u / kUnitsPerRow, j = u % kUnitsPerRow;
        const uint4 w = *reinterpret_cast<const uint4*>(v8 + r * HD + 16 * j);
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t h[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            h[2 * e] = e4m3x2_to_f16x2(static_cast<uint16_t>(in[e] & 0xFFFFu));
            h[2 * e + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(in[e] >> 16));
        }
        // values 16j .. 16j + 15 = 16-byte units 2(j % 4), 2(j % 4) + 1 of chunk j / 4 of row r
        uint8_t* row = vh + (j >> 2) * (kBlockN * 128) + r * 128;
        const int u0 = 2 * (j & 3);
        *reinterpret_cast<uint4*>(row + ((u0 ^ (r & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(row + (((u0 + 1) ^ (r & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
    }
}

// K-major descriptor of an e4m3 Q / K tile, k-step kk of 32 values (32 bytes).
template <int HD>
__device__ __forceinline__ uint64_t desc_kmajor_e4m3(uint32_t tile, int kk) {
    return HD == 128 ? smem_desc_sw128(tile + kk * 32, 16, 1024)
                     : smem_desc_sw64(tile + kk * 32, 16, 512);
}

template <int HD, bool F8, bool AUXV>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnProblem p,
                   const int4* __restrict__ items, WorkspaceHeader* hdr) {
    using L = BlockLayout<HD, F8>;
    static_assert(!(F8 && AUXV), "the value embedding is a bf16 path");
    // P_r apart from S_r where TMEM has room for it (hd 64), else in the first 64 columns of S_r.
    constexpr bool kSepP = HD == 64;
    constexpr uint32_t kTmP = kSepP ? L::kTmO + 2 * HD : 0;
    static_assert(!kSepP || kTmP + 128 <= L::kTmemCols, "TMEM columns");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const uint32_t sbase = smem_u32(smem);
    TcBars* bars = reinterpret_cast<TcBars*>(smem + L::kOffBar);
    volatile int* abort_flag = &bars->abort;
    int* dev_status = &hdr->status;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 8 && lane == 0) {
        for (int s = 0; s < 3; ++s) {
            mbar_init(&bars->q_full[s], 1);
            // freed by the MMA thread's commit after the sub-tile's last S and by the 4 warps of
            // its softmax warpgroup after the epilogue has staged O through the slot
            mbar_init(&bars->q_empty[s], 5);
        }
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            // FP8: filled by the 64 converter threads; bf16: by the producer's TMA
            mbar_init(&bars->v_full[s], F8 ? 64 : 1);
            mbar_init(&bars->v_empty[s], 1);
            mbar_init(&bars->v_add[s], 64);
        }
        for (int r = 0; r < 2; ++r) {
            mbar_init(&bars->s_full[r], 1);
            mbar_init(&bars->p_full[r], 128);
            mbar_init(&bars->pv_done[r], 1);
            mbar_init(&bars->o_ready[r], 1);
            mbar_init(&bars->v8_full[r], 1);
            mbar_init(&bars->v8_empty[r], 64);
            mbar_init(&bars->s_free[r], 128);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 9) {
        tmem_alloc(&bars->tmem_base, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    grid_dep_wait();  // the work list (written by the scheduler kernel) is complete from here on
    const int n_items = *reinterpret_cast<volatile int*>(&hdr->n_items);
    const int H = p.heads;
    const int G = p.heads / p.kv_heads;
    static_assert(8 * kTcRegsSoftmax + 4 * kTcRegsOther <= 12 * 168, "register split");

    if (warp >= 8) regs_decrease<kTcRegsOther>();  // the whole third warpgroup, then its roles
    if (warp >= 10) {
        // ------------------------------------------------- FP8: V converter; aux_v: adder; else idle
        if (AUXV) {
            // V tiles in the producer's order: once one has landed, aux_v's matching rows are
            // added in place and the tile is published to the MMA issuer (v_add)
            const int at = threadIdx.x - 320;  // 0 .. 63
            const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
            const __nv_bfloat16* aux = static_cast<const __nv_bfloat16*>(p.v_aux);
            uint32_t vc = 0;
            bool ok = true;
            ItemWalk wk;
            for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
                if (!wk.has()) continue;
                const Item it = decode_item(wk.cur, p);
                for (int t = 0; ok && t < it.n_kv; ++t, ++vc) {
                    const uint32_t sv = vc % L::kVStages;
                    ok = mbar_wait(&bars->v_full[sv], (vc / L::kVStages) & 1, abort_flag, dev_status);
                    if (!ok) break;
                    add_aux_tile<HD, 64, 8>(smem + L::kOffV + sv * L::kV, aux, it.kv_lo + t * kBlockN,
                                            it.head / G, p.kv_heads, slots, at);
                    fence_proxy_async_smem();  // the tensor cores read the tile next
                    mbar_arrive(&bars->v_add[sv]);
                }
            }
        }
        if (F8) {
            const int ct = threadIdx.x - 320;  // 0 .. 63
            uint32_t vc = 0;
            bool ok = true;
            ItemWalk wk;
            for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
                if (!wk.has()) continue;
                const Item it = decode_item(wk.cur, p);
                for (int t = 0; ok && t < it.n_kv; ++t, ++vc) {
                    const uint32_t s8 = vc % L::kV8Stages, sv = vc % L::kVStages;
                    ok = mbar_wait(&bars->v8_full[s8], (vc / L::kV8Stages) & 1, abort_flag, dev_status) &&
                         mbar_wait(&bars->v_empty[sv], ((vc / L::kVStages) & 1) ^ 1, abort_flag, dev_status);
                    if (!ok) break;
                    widen_v_tile<HD>(smem + L::kOffV8 + s8 * L::kV8, smem + L::kOffV + sv * L::kV, ct);
                    fence_proxy_async_smem();  // the tensor cores read the f16 tile next
                    mbar_arrive(&bars->v_full[sv]);
                    mbar_arrive(&bars->v8_empty[s8]);
                }
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t qc = 0, kc = 0, vc = 0;
            bool ok = true;
            ItemWalk wk;
            for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
                if (!wk.has()) continue;
                const Item it = decode_item(wk.cur, p);
                const int g = it.head / G;
                for (int r = 0; r < it.n_sub; ++r) {
                    const uint32_t sq = qc % L::kQSlots;
                    if (!mbar_wait(&bars->q_empty[sq], ((qc / L::kQSlots) & 1) ^ 1, abort_flag,
                                   dev_status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->q_full[sq], L::kQSub);
                    if (F8)
                        tma_load_2d(smem + L::kOffQ + sq * L::kQSub, &tm_q, it.head * HD,
                                    it.q0 + kBlockM * r, &bars->q_full[sq]);
                    else
                        for (int c = 0; c < HD / 64; ++c)
                            tma_load_2d(smem + L::kOffQ + sq * L::kQSub + c * L::kChunk, &tm_q,
                                        it.head * HD + 64 * c, it.q0 + kBlockM * r, &bars->q_full[sq]);
                    ++qc;
                }
                for (int t = 0; ok && t < it.n_kv; ++t) {
                    const int row = it.kv_lo + t * kBlockN;
                    const uint32_t sk = kc % L::kKStages;
                    if (!mbar_wait(&bars->k_empty[sk], ((kc / L::kKStages) & 1) ^ 1, abort_flag,
                                   dev_status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->k_full[sk], L::kK);
                    if (F8)
                        tma_load_2d(smem + L::kOffK + sk * L::kK, &tm_k, g * HD, row, &bars->k_full[sk]);
                    else
                        for (int c = 0; c < HD / 64; ++c)
                            tma_load_2d(smem + L::kOffK + sk * L::kK + c * L::kChunk, &tm_k,
                                        g * HD + 64 * c, row, &bars->k_full[sk]);
                    ++kc;
                    if (F8) {
                        // e4m3 V into the staging ring; the converter widens it into the V ring
                        const uint32_t s8 = vc % L::kV8Stages;
                        if (!mbar_wait(&bars->v8_empty[s8], ((vc / L::kV8Stages) & 1) ^ 1, abort_flag,
                                       dev_status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars->v8_full[s8], L::kV8);
                        tma_load_2d(smem + L::kOffV8 + s8 * L::kV8, &tm_v, g * HD, row, &bars->v8_full[s8]);
                    } else {
                        const uint32_t sv = vc % L::kVStages;
                        if (!mbar_wait(&bars->v_empty[sv], ((vc / L::kVStages) & 1) ^ 1, abort_flag,
                                       dev_status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars->v_full[sv], L::kV);
                        for (int c = 0; c < HD / 64; ++c)
                            tma_load_2d(smem + L::kOffV + sv * L::kV + c * L::kChunk, &tm_v,
                                        g * HD + 64 * c, row, &bars->v_full[sv]);
                    }
                    ++vc;
                }
            }
            if (!ok) {
                // Wait (bounded) for the copies this thread issued last into every buffer.
                for (uint32_t n = qc > L::kQSlots ? qc - L::kQSlots : 0; n < qc; ++n)
                    drain_wait(&bars->q_full[n % L::kQSlots], (n / L::kQSlots) & 1);
                for (uint32_t n = kc > L::kKStages ? kc - L::kKStages : 0; n < kc; ++n)
                    drain_wait(&bars->k_full[n % L::kKStages], (n / L::kKStages) & 1);
                if (F8) {
                    for (uint32_t n = vc > L::kV8Stages ? vc - L::kV8Stages : 0; n < vc; ++n)
                        drain_wait(&bars->v8_full[n % L::kV8Stages], (n / L::kV8Stages) & 1);
                } else {
                    for (uint32_t n = vc > L::kVStages ? vc - L::kVStages : 0; n < vc; ++n)
                        drain_wait(&bars->v_full[n % L::kVStages], (n / L::kVStages) & 1);
                }
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_f32(kBlockM, kBlockN)
                                             : idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
            constexpr uint32_t idesc_pv = F8 ? idesc_f16_f32(kBlockM, HD, 0, 1)
                                             : idesc_bf16_f32(kBlockM, HD, 0, 1);
            uint32_t qc = 0;    // Q sub-tiles of the items before the current one
            uint32_t g = 0;     // global index of the current key tile (the K / V ring position)
            uint32_t p_cnt[2] = {0, 0};         // P.V products issued per sub-tile
            uint32_t s_cnt[2] = {0, 0};         // S products issued per sub-tile
            bool pv_open[2] = {false, false};   // hd 128: the last P.V of r not yet seen complete
            // the key tile g - 1 as sub-tile r used it: its S was issued, its P.V not yet
            bool pend[2] = {false, false}, pend_first[2] = {false, false}, pend_last[2] = {false, false};
            bool ok = true;

            // O_r += P_r V_{g-1} (V_{g-1} has landed); first: the sub-tile's first key tile of its
            // item (O starts from zero), last: its last one (O is complete afterwards)
            auto issue_pv = [&](int r, bool first, bool last) -> bool {
                if (!mbar_wait(&bars->p_full[r], p_cnt[r] & 1, abort_flag, dev_status)) return false;
                tc_fence_after();
                const uint32_t v_tile = sbase + L::kOffV + ((g - 1) % L::kVStages) * L::kV;
                const uint32_t a_p = tmem + (kSepP ? kTmP + 64 * r : 128 * r);
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk)
                    umma_f16_ts(tmem + L::kTmO + HD * r, a_p + 8 * kk, desc_v(v_tile, kk), idesc_pv,
                                (!first || kk > 0) ? 1u : 0u);
                umma_commit(&bars->pv_done[r]);
                if (last) umma_commit(&bars->o_ready[r]);
                ++p_cnt[r];
                pv_open[r] = !kSepP;
                return true;
            };
            auto wait_v_prev = [&]() -> bool {
                const uint32_t n = g - 1;
                uint64_t* bar = AUXV ? &bars->v_add[n % L::kVStages] : &bars->v_full[n % L::kVStages];
                if (!mbar_wait(bar, (n / L::kVStages) & 1, abort_flag, dev_status))
                    return false;
                return true;
            };

            ItemWalk wk;
            for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
                if (!wk.has()) continue;
                const Item it = decode_item(wk.cur, p);
                uint32_t q_slot[2], q_par[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    q_slot[r] = (qc + r) % L::kQSlots;
                    q_par[r] = ((qc + r) / L::kQSlots) & 1;
                }
                for (int t = 0; t < it.n_kv && ok; ++t, ++g) {
                    // every key tile has a user (the two sub-tiles' ranges are contiguous and
                    // cover the item's), so V_{g-1} is awaited and released once, in order
                    if (g > 0 && !wait_v_prev()) {
                        ok = false;
                        break;
                    }
                    // the previous item's last P.V products first: their epilogues free the Q slots
                    // the producer may be waiting for before it loads this tile
                    if (t == 0) {
                        for (int r = 0; r < 2 && ok; ++r)
                            if (pend[r]) {
                                ok = issue_pv(r, pend_first[r], pend_last[r]);
                                pend[r] = false;
                            }
                        if (!ok) break;
                    }
                    const uint32_t sk = g % L::kKStages;
                    if (!mbar_wait(&bars->k_full[sk], (g / L::kKStages) & 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t k_tile = sbase + L::kOffK + sk * L::kK;
                    // the P.V products of tile g - 1 still to issue (hd 64: after both S of tile g)
                    bool pv_now[2] = {false, false}, pv_first[2], pv_last[2];
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        pv_now[r] = pend[r];
                        pv_first[r] = pend_first[r];
                        pv_last[r] = pend_last[r];
                        pend[r] = false;
                        if (!kSepP && pv_now[r]) {
                            if (!issue_pv(r, pv_first[r], pv_last[r])) {
                                ok = false;
                                break;
                            }
                            pv_now[r] = false;
                        }
                        if (t < it.t_first[r] || t > it.t_last[r]) continue;
                        if (kSepP) {
                            // hd 64: S_r is free once the softmax has read its last tile
                            if (s_cnt[r] > 0 && !mbar_wait(&bars->s_free[r], (s_cnt[r] - 1) & 1,
                                                           abort_flag, dev_status)) {
                                ok = false;
                                break;
                            }
                        } else if (pv_open[r]) {
                            // hd 128: S_r overwrites the columns that P_r shares with it
                            if (!mbar_wait(&bars->pv_done[r], (p_cnt[r] - 1) & 1, abort_flag,
                                           dev_status)) {
                                ok = false;
                                break;
                            }
                            pv_open[r] = false;
                        }
                        if (t == it.t_first[r] &&
                            !mbar_wait(&bars->q_full[q_slot[r]], q_par[r], abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t q_tile = sbase + L::kOffQ + q_slot[r] * L::kQSub;
                        if (F8) {
#pragma unroll
                            for (int kk = 0; kk < HD / 32; ++kk)
                                umma_f8_ss(tmem + 128 * r, desc_kmajor_e4m3<HD>(q_tile, kk),
                                           desc_kmajor_e4m3<HD>(k_tile, kk), idesc_qk, kk == 0 ? 0u : 1u);
                        } else {
#pragma unroll
                            for (int kk = 0; kk < HD / 16; ++kk)
                                umma_f16_ss(tmem + 128 * r, desc_kmajor(q_tile, kk),
                                            desc_kmajor(k_tile, kk), idesc_qk, kk == 0 ? 0u : 1u);
                        }
                        umma_commit(&bars->s_full[r]);
                        if (t == it.t_last[r]) umma_commit(&bars->q_empty[q_slot[r]]);
                        ++s_cnt[r];
                        pend[r] = true;
                        pend_first[r] = t == it.t_first[r];
                        pend_last[r] = t == it.t_last[r];
                    }
                    if (!ok) break;
                    if (kSepP) {
                        for (int r = 0; r < 2 && ok; ++r)
                            if (pv_now[r]) ok = issue_pv(r, pv_first[r], pv_last[r]);
                        if (!ok) break;
                    }
                    if (g > 0) umma_commit(&bars->v_empty[(g - 1) % L::kVStages]);
                    umma_commit(&bars->k_empty[sk]);
                }
                qc += it.n_sub;
            }
            // the last key tile's P.V products
            if (ok && g > 0) {
                ok = wait_v_prev();
                for (int r = 0; r < 2 && ok; ++r)
                    if (pend[r]) ok = issue_pv(r, pend_first[r], pend_last[r]);
                if (ok) umma_commit(&bars->v_empty[(g - 1) % L::kVStages]);
            }
            // Wait (bounded) until every MMA this thread issued has finished.
            umma_commit(&bars->drain);
            drain_wait(&bars->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax, sub-tile r
        regs_increase<kTcRegsSoftmax>();
        const int r = warp >> 2;
        const int row = threadIdx.x & 127;  // query row in the sub-tile == TMEM lane
        const int r0 = (warp & 3) * 32;     // first row of this warp
        const uint32_t tm_lane = tmem + (static_cast<uint32_t>(r0) << 16);
        const uint32_t tm_s = tm_lane + 128 * r;
        const uint32_t tm_p = kSepP ? tm_lane + kTmP + 64 * r : tm_s;
        const uint32_t tm_o = tm_lane + L::kTmO + HD * r;
        const float scale_log2 = p.scale * (F8 ? p.qk_scale : 1.0f) * kLog2e;
        const uint64_t scale2 = f32x2(scale_log2, scale_log2);
        const int window = p.window;
        uint32_t s_cnt = 0, o_cnt = 0;
        uint32_t pv_seen = 0;  // hd 64: P.V completions of this sub-tile awaited so far
        uint32_t q_seq = 0;  // index of the current item's first Q sub-tile in this CTA's stream
        bool ok = true;
        ItemWalk wk;
        for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
            if (!wk.has()) continue;
            const Item it = decode_item(wk.cur, p);
            // per-sub-tile fields by select (r is not a compile-time index here)
            const int nr = r ? it.nr[1] : it.nr[0];
            const int t_first = r ? it.t_first[1] : it.t_first[0];
            const int t_last = r ? it.t_last[1] : it.t_last[0];
            const uint32_t my_q = q_seq + r;
            q_seq += it.n_sub;
            if (nr == 0) continue;
            const int qr0 = it.q0 + kBlockM * r;
            const int i = qr0 + row;
            // visible key slots of this row: [j_min, j_max]
            const int j_max = p.causal ? min(i, it.kv_hi - 1) : it.kv_hi - 1;
            const int j_min = window > 0 ? i - window + 1 : INT32_MIN / 2;
            // a tile needs the lower / upper bound iff some valid row of the sub-tile does:
            // the largest j_min belongs to the last valid row, the smallest j_max to the first
            const int tile_jmin = window > 0 ? qr0 + nr - window : INT32_MIN / 2;
            const int tile_jmax = p.causal ? min(qr0, it.kv_hi - 1) : it.kv_hi - 1;
            float m = -INFINITY, l = 0.f;
            for (int t = t_first; t <= t_last; ++t) {
                const int kv0 = it.kv_lo + t * kBlockN;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars->s_full[r], s_cnt & 1, abort_flag, dev_status));
                if (!ok) break;
                ++s_cnt;
                tc_fence_after();
                // the whole S row, one wait
                uint32_t v[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tm_s + 32 * c, v + 32 * c);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) regs_after_wait(v + 32 * c);
                if (kSepP) {
                    // S_r may be overwritten by the next tile's product from here on
                    tc_fence_before();
                    mbar_arrive(&bars->s_free[r]);
                }
                const int c_lo = j_min - kv0, c_hi = j_max - kv0;
                // Masked tiles: the hidden scores are set to -inf in place, per 32-column chunk
                // classed uniformly over this warp's 32 rows [r0, r0 + 31]. The row bounds c_lo(row),
                // c_hi(row) grow with the row, so a chunk is wholly hidden when it lies below the
                // first row's c_lo or above the last row's c_hi, needs no mask when it lies wholly
                // inside [last row's c_lo, first row's c_hi], and is masked element by element
                // otherwise. The max and the exponentials then run unmasked (2^-inf = 0).
                const bool full_tile = (tile_jmin <= kv0) && (kv0 + kBlockN - 1 <= tile_jmax);
                if (!full_tile) {
                    // bit e of vis[c]: column 32 c + e visible for this row; chunks wholly visible or
                    // wholly hidden for every row of the warp need no per-row test
                    const int lo_first = window > 0 ? qr0 + r0 - window + 1 - kv0 : INT32_MIN / 2;
                    const int lo_last = window > 0 ? lo_first + 31 : INT32_MIN / 2;
                    const int hi_first = (p.causal ? min(qr0 + r0, it.kv_hi - 1) : it.kv_hi - 1) - kv0;
                    const int hi_last = (p.causal ? min(qr0 + r0 + 31, it.kv_hi - 1) : it.kv_hi - 1) - kv0;
                    uint32_t vis[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int lo = 32 * c, hi = lo + 31;
                        const int a = c_lo - lo, b = c_hi - lo;  // visible e in [a, b]
                        const uint32_t below = a <= 0 ? 0u : (a >= 32 ? ~0u : (1u << a) - 1u);
                        const uint32_t above = b >= 31 ? 0u : (b < 0 ? ~0u : ~((2u << b) - 1u));
                        vis[c] = (hi < lo_first || lo > hi_last) ? 0u
                                 : (lo >= lo_last && hi <= hi_first) ? ~0u : ~(below | above);
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            v[32 * c + e] = ((vis[c] >> e) & 1u) ? v[32 * c + e] : __float_as_uint(-INFINITY);
                }
                // row max over the visible columns
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    mx = fmaxf(mx, chunk_max<kMaskNone>(v + 32 * c, 32 * c, c_lo, c_hi));
                const float m_new = fmaxf(m, mx * scale_log2);
                // Keep the reference max until the row max grows by more than 8 (a factor 256):
                // O / l and the lse are exact for any reference value.
                const bool rescale = m_new > m + 8.0f;
                const float alpha = rescale ? ex2(m - m_new) : 1.0f;
                if (rescale) m = m_new;
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                const uint64_t negm2 = f32x2(neg_m, neg_m);
                // P = 2^(s * scale * log2e - m) (written after the whole row was read, so it may
                // share the columns of S)
                uint64_t sum_a = f32x2(0.f, 0.f), sum_b = f32x2(0.f, 0.f);
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    chunk_exp<kMaskNone, F8>(v + 32 * c, 32 * c, c_lo, c_hi, scale2, negm2, sum_a, sum_b,
                                             pk + 16 * (c & 1));
                    if (c == 1 && kSepP && pv_seen < s_cnt - 1) {
                        // hd 64: the last P.V of this sub-tile reads P_r and adds into O_r; it must be
                        // complete before P_r is overwritten and O_r rescaled
                        ok = __all_sync(0xffffffffu, mbar_wait(&bars->pv_done[r], pv_seen & 1,
                                                               abort_flag, dev_status));
                        ++pv_seen;
                        tc_fence_after();
                    }
                    if (c & 1) {
                        tmem_st16(tm_p + 16 * (c - 1), pk);
                        tmem_st16(tm_p + 16 * c, pk + 16);
                    }
                }
                if (!ok) break;
                const uint64_t sum2 = add_f32x2(sum_a, sum_b);
                float s_lo, s_hi;
                f32x2_split(sum2, s_lo, s_hi);
                l = l * alpha + (s_lo + s_hi);
                if (t > t_first && __any_sync(0xffffffffu, rescale)) {
                    uint32_t ov[HD];
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) tmem_ld32(tm_o + 32 * c, ov + 32 * c);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        regs_after_wait(ov + 32 * c);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            ov[32 * c + e] = __float_as_uint(__uint_as_float(ov[32 * c + e]) * alpha);
                        tmem_st32(tm_o + 32 * c, ov + 32 * c);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[r]);
            }
            if (!ok) break;
            // epilogue: O / l and lse for the valid rows
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars->o_ready[r], o_cnt & 1, abort_flag, dev_status));
            if (!ok) break;
            ++o_cnt;
            tc_fence_after();
            const bool valid = row < nr;
            const float inv_l = l > 0.f ? (F8 ? p.v_scale : 1.f) / l : 0.f;
            // O / l -> bf16, staged through this sub-tile's Q slot (its last S has completed):
            // each warp writes kStageRows of its rows at a time (all 32 when the slot holds them,
            // 16 for the narrower e4m3 slot) with an XOR swizzle of the 16-byte chunks, then copies
            // them out two rows per instruction at hd 128, so every global store of the warp covers
            // 512 contiguous bytes. Rows past the end of the document are not written.
            constexpr int kChunks = HD / 8;  // 16-byte chunks per row
            constexpr int kSR = L::kStageRows;
            uint8_t* stage = smem + L::kOffQ + (my_q % L::kQSlots) * L::kQSub + (warp & 3) * kSR * (HD * 2);
            uint32_t ov[HD];
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) tmem_ld32(tm_o + 32 * c, ov + 32 * c);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) regs_after_wait(ov + 32 * c);
#pragma unroll 1
            for (int ps = 0; ps < 32 / kSR; ++ps) {
                if ((lane / kSR) == ps) {
                    const int wrow = lane % kSR;
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint32_t* w8 = ov + 32 * c + 8 * q4;
                            const uint4 w4 = make_uint4(
                                pack_bf16x2(__uint_as_float(w8[0]) * inv_l, __uint_as_float(w8[1]) * inv_l),
                                pack_bf16x2(__uint_as_float(w8[2]) * inv_l, __uint_as_float(w8[3]) * inv_l),
                                pack_bf16x2(__uint_as_float(w8[4]) * inv_l, __uint_as_float(w8[5]) * inv_l),
                                pack_bf16x2(__uint_as_float(w8[6]) * inv_l, __uint_as_float(w8[7]) * inv_l));
                            const int chunk = 4 * c + q4;
                            *reinterpret_cast<uint4*>(stage + wrow * (HD * 2) +
                                                      ((chunk ^ (wrow & (kChunks - 1))) << 4)) = w4;
                        }
                    }
                }
                __syncwarp();
                const int row0 = qr0 + r0 + ps * kSR;  // first slot of the staged rows
                constexpr int kRowsPerIter = 32 / kChunks;
#pragma unroll 4
                for (int j = 0; j < kSR / kRowsPerIter; ++j) {
                    const int rl = j * kRowsPerIter + lane / kChunks;
                    const int chunk = lane % kChunks;
                    if (r0 + ps * kSR + rl < nr) {
                        const uint4 w4 = *reinterpret_cast<const uint4*>(
                            stage + rl * (HD * 2) + ((chunk ^ (rl & (kChunks - 1))) << 4));
                        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.o) +
                                             (static_cast<int64_t>(row0 + rl) * H + it.head) * HD + chunk * 8;
                        *reinterpret_cast<uint4*>(dst) = w4;
                    }
                }
                __syncwarp();
            }
            __syncwarp();
            fence_proxy_async_smem();  // the slot's next fill is written by the async proxy (TMA)
            if (lane == 0) mbar_arrive(&bars->q_empty[my_q % L::kQSlots]);
            tc_fence_before();
            if (valid && p.lse) p.lse[static_cast<int64_t>(i) * H + it.head] = (m + log2f(l)) * kLn2;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, L::kTmemCols);
}

template <int HD, bool F8, bool AUXV>
static cudaError_t launch_tc_hd(const AttnProblem& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const int4* items, WorkspaceHeader* hdr,
                                cudaStream_t stream) {
    using L = BlockLayout<HD, F8>;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD, F8, AUXV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    // programmatic stream serialization: the prologue overlaps the scheduler kernel before it
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = L::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_tc_kernel<HD, F8, AUXV>, tq, tk, tv, p, items, hdr);
}

cudaError_t launch_attn_tc(const AttnProblem& p, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, const int4* items, WorkspaceHeader* hdr,
                           cudaStream_t stream, bool fp8) {
    const bool aux = p.v_aux != nullptr;
    if (fp8 && aux) return cudaErrorInvalidValue;
    if (p.head_dim == 128)
        return fp8 ? launch_tc_hd<128, true, false>(p, tm_q, tm_k, tm_v, items, hdr, stream)
               : aux ? launch_tc_hd<128, false, true>(p, tm_q, tm_k, tm_v, items, hdr, stream)
                     : launch_tc_hd<128, false, false>(p, tm_q, tm_k, tm_v, items, hdr, stream);
    if (p.head_dim == 64)
        return fp8 ? launch_tc_hd<64, true, false>(p, tm_q, tm_k, tm_v, items, hdr, stream)
               : aux ? launch_tc_hd<64, false, true>(p, tm_q, tm_k, tm_v, items, hdr, stream)
                     : launch_tc_hd<64, false, false>(p, tm_q, tm_k, tm_v, items, hdr, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pha
