// attn_band.cu -- bf16 attention forward on the sm_100a tensor cores for causal sliding windows
// of at most 128 key slots (the paired-head workload's window: "modded-nanogpt Paired Head
// Attention record" page, section "sequence length and window handling").
//
// Same arithmetic as attn_tc.cu (S = Q K^T and O += P V as tcgen05 MMAs into TMEM, online
// softmax in the log2 domain with lazy rescaling, O / l and the LSE in the epilogue), with a
// different work decomposition. With window <= 128 and query / key tiles of 128 slots counted
// from the document start, query tile j sees only key tile j - 1 (window part, an upper
// triangle) and key tile j (causal part, a lower triangle). So a run of consecutive query tiles
// of one (document, head) streams the key tiles once, in order, and at step s the key tile s is
// used by two query tiles at once: the one whose causal tile it is and the next one, whose
// window tile it is. Consecutive query tiles alternate between the two softmax warpgroups, so
// both warpgroups have one tile at every step and every K / V tile is read from HBM once per run.
//
// CTA = 12 warps (16 with the value embedding), persistent, one per SM, items in snake order over
// the longest-first list; the softmax warpgroups run with 200 registers per thread (184 with the
// value embedding):
//   warps 0-3, 4-7   softmax warpgroups w = 0, 1: query tiles n (CTA-wide count) with n % 2 == w.
//                    The whole 128-column S row is loaded from TMEM with one wait; hidden scores
//                    are set to -inf in registers (per-row bit masks, skipped for 32-column chunks
//                    that are wholly visible or hidden for every row of the warp); max and
//                    exponentials run on independent accumulator chains
//   warp 8           TMA producer: Q tiles into a ring of 3 slots, K and V tiles into their rings
//   warps 9, 10      MMA issuers, one per warpgroup (warp 9 also owns the 512 TMEM columns), so a
//                    warpgroup's next S never waits behind the other warpgroup's softmax
//   warp 11          idle (completes the third warpgroup for the register split)
//   warps 12-15      value embedding only: add aux_v to each landed V tile
// TMEM columns: S_w at 128 w (P_w aliases its first 64 columns), O_w at 256 + hd w.
// A K / V stage is released when both issuers have arrived for its step: by a commit after
// their MMAs on it, or by a plain arrive on a step their warpgroup does not use.
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

// 8 softmax warps; producer, 2 MMA issuers and an idle warp (a whole third warpgroup for the
// register split); with the value embedding a fourth warpgroup of adders.
constexpr int kBandThreads = 384;
constexpr int kBandAuxThreads = 512;
// Register split, per thread: the softmax warpgroups hold a whole 128-column score row. Without
// the embedding 8 x 200 + 4 x 88 = 1952 <= 12 x 168 (the launch allocation of 384 threads); with
// it 8 x 184 + 8 x 72 = 2048 <= 16 x 128 (512 threads), so that the adders keep eight 16-byte
// aux_v loads in flight (measured: 184 / 72 with eight in flight 140 us on the paired workload,
// 200 / 56 with four 171 us).
constexpr int kBandRegsSoftmax = 200;
constexpr int kBandRegsOther = 88;
constexpr int kBandRegsSoftmaxAux = 184;
constexpr int kBandRegsOtherAux = 72;
constexpr int kBandAuxBatch = 8;  // aux_v loads in flight per adder thread

struct BandBars {
    uint64_t q_full[3], q_empty[3];
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    uint64_t v_add[4];  // value embedding: the landed V tile has had aux_v added
    uint64_t s_full[2], p_full[2], pv_done[2], o_ready[2];
    uint64_t drain[2];
    uint64_t stall;  // never signalled: the failure-detection test hook waits on it
    uint32_t tmem_base;
    int abort;
};

template <int HD, bool AUXV>
__global__ void __launch_bounds__(AUXV ? kBandAuxThreads : kBandThreads, 1)
    attn_band_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_out, const AttnProblem p,
                     const int4* __restrict__ items, WorkspaceHeader* hdr) {
    using L = TcLayout<HD>;
    constexpr int S = L::kKStages;
    static_assert(L::kKStages == L::kVStages, "K and V rings step together");
    static_assert(sizeof(BandBars) <= L::kBarBytes, "barrier block");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const uint32_t sbase = smem_u32(smem);
    BandBars* bars = reinterpret_cast<BandBars*>(smem + L::kOffBar);
    volatile int* abort_flag = &bars->abort;
    int* dev_status = &hdr->status;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 8 && lane == 0) {
        for (int s = 0; s < 3; ++s) {
            mbar_init(&bars->q_full[s], 1);
            // freed by the issuer's commit after the tile's last S and by the 4 warps of its
            // softmax warpgroup after the epilogue has staged O through the slot
            mbar_init(&bars->q_empty[s], 5);
        }
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bars->v_add[s], 128);
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 2);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 2);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(&bars->s_full[w], 1);
            mbar_init(&bars->p_full[w], 128);
            mbar_init(&bars->pv_done[w], 1);
            mbar_init(&bars->o_ready[w], 1);
            mbar_init(&bars->drain[w], 1);
        }
        mbar_init(&bars->stall, 1);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_out);
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
    static_assert(8 * kBandRegsSoftmax + 4 * kBandRegsOther <= 12 * 168, "register split");
    static_assert(8 * kBandRegsSoftmaxAux + 8 * kBandRegsOtherAux <= 16 * 128, "register split");

    if (warp >= 8) {  // every warp of the third (and fourth) warpgroup, then their roles
        if (AUXV)
            regs_decrease<kBandRegsOtherAux>();
        else
            regs_decrease<kBandRegsOther>();
    }
    if (warp == 11) {
        // ------------------------------------------------------------ idle (register split only)
    } else if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t qc = 0, kc = 0, vc = 0;  // Q / K / V tiles issued so far
            bool ok = true;
            ItemWalk wk;
            for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
                if (!wk.has()) continue;
                const BandItem it = decode_band(wk.cur);
                const int gk = it.head / G;
                const int kv_first = it.q0 - (it.hp ? kBlockN : 0);
                const uint32_t qn = qc;  // CTA-wide index of the item's first query tile
                for (int s = 0; ok && s < it.n_qt + it.hp; ++s) {
                    // query tiles first needed at this step: the window user s - hp + 1, and
                    // at step 0 of a run from the document start also tile 0 (causal user)
                    const int u_hi = s - it.hp + 1;
                    const int u_lo = (s == 0 && !it.hp) ? 0 : u_hi;
                    for (int u = u_lo; u <= u_hi && u < it.n_qt; ++u) {
                        const uint32_t n = qn + u, sq = n % L::kQSlots;
                        if (!mbar_wait(&bars->q_empty[sq], ((n / L::kQSlots) & 1) ^ 1, abort_flag,
                                       dev_status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars->q_full[sq], L::kQSub);
                        for (int c = 0; c < HD / 64; ++c)
                            tma_load_2d(smem + L::kOffQ + sq * L::kQSub + c * L::kChunk, &tm_q,
                                        it.head * HD + 64 * c, it.q0 + kBlockM * u,
                                        &bars->q_full[sq]);
                        ++qc;
                    }
                    if (!ok) break;
                    const int row = kv_first + s * kBlockN;
                    const uint32_t sk = kc % S;
                    if (!mbar_wait(&bars->k_empty[sk], ((kc / S) & 1) ^ 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->k_full[sk], L::kKV);
                    for (int c = 0; c < HD / 64; ++c)
                        tma_load_2d(smem + L::kOffK + sk * L::kKV + c * L::kChunk, &tm_k,
                                    gk * HD + 64 * c, row, &bars->k_full[sk]);
                    ++kc;
                    const uint32_t sv = vc % S;
                    if (!mbar_wait(&bars->v_empty[sv], ((vc / S) & 1) ^ 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->v_full[sv], L::kKV);
                    for (int c = 0; c < HD / 64; ++c)
                        tma_load_2d(smem + L::kOffV + sv * L::kKV + c * L::kChunk, &tm_v,
                                    gk * HD + 64 * c, row, &bars->v_full[sv]);
                    ++vc;
                }
            }
            if (!ok) {
                // Wait (bounded) for the copies this thread issued last into every buffer.
                for (uint32_t n = qc > L::kQSlots ? qc - L::kQSlots : 0; n < qc; ++n)
                    drain_wait(&bars->q_full[n % L::kQSlots], (n / L::kQSlots) & 1);
                for (uint32_t n = kc > S ? kc - S : 0; n < kc; ++n)
                    drain_wait(&bars->k_full[n % S], (n / S) & 1);
                for (uint32_t n = vc > S ? vc - S : 0; n < vc; ++n)
                    drain_wait(&bars->v_full[n % S], (n / S) & 1);
            }
        }
        __syncwarp();
    } else if (AUXV && warp >= 12) {
        // ------------------------------------------------------------ adder warpgroup
        // V tiles in the producer's order; each gets aux_v added once it has landed, then is
        // published to the MMA issuers.
        const int at = threadIdx.x - kBandThreads;
        const int64_t slots = static_cast<int64_t>(p.total_tokens) * p.slot_mult;
        const __nv_bfloat16* aux = static_cast<const __nv_bfloat16*>(p.v_aux);
        uint32_t vc = 0;
        bool ok = true;
        ItemWalk wk;
        for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
            if (!wk.has()) continue;
            const BandItem it = decode_band(wk.cur);
            const int gk = it.head / G;
            const int kv_first = it.q0 - (it.hp ? kBlockN : 0);
            for (int s = 0; ok && s < it.n_qt + it.hp; ++s) {
                const uint32_t sv = vc % S;
                ok = __all_sync(0xffffffffu, mbar_wait(&bars->v_full[sv], (vc / S) & 1, abort_flag,
                                                       dev_status));
                if (!ok) break;
                add_aux_tile<HD, 128, kBandAuxBatch>(smem + L::kOffV + sv * L::kKV, aux, kv_first + s * kBlockN,
                                         gk, p.kv_heads, slots, at);
                fence_proxy_async_smem();  // the tensor cores read the tile next
                mbar_arrive(&bars->v_add[sv]);
                ++vc;
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------ MMA issuer of warpgroup w
        const int w = warp - 9;
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, HD, 0, 1);
            const uint32_t tm_s = tmem + 128 * w;
            const uint32_t tm_o = tmem + L::kTmO + HD * w;
            uint32_t qn = 0, g = 0, p_cnt = 0;
            bool ok = true;
            ItemWalk wk;
            for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
                if (!wk.has()) continue;
                const BandItem it = decode_band(wk.cur);
                const int n_steps = it.n_qt + it.hp;
                for (int s = 0; s < n_steps; ++s) {
                    const uint32_t gs = g + s, st = gs % S, ph = (gs / S) & 1;
                    // this warpgroup's user of key tile s: the query tile whose causal tile it
                    // is (ud), or the next one, whose window tile it is (ud + 1)
                    const int ud = s - it.hp;
                    int u = -1;
                    bool diag = false;
                    if (ud >= 0 && ((qn + ud) & 1) == static_cast<uint32_t>(w)) {
                        u = ud;
                        diag = true;
                    } else if (ud + 1 < it.n_qt && ((qn + ud + 1) & 1) == static_cast<uint32_t>(w)) {
                        u = ud + 1;
                    }
                    // first tile of its query tile: a window tile, or the causal tile of a
                    // document's first query tile
                    const bool first = !diag || (ud + it.hp == 0);
                    const uint32_t n = qn + (u < 0 ? 0 : u), sq = n % L::kQSlots;
                    if (!mbar_wait(&bars->k_full[st], ph, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    if (u >= 0) {
                        if ((first && !mbar_wait(&bars->q_full[sq], (n / L::kQSlots) & 1,
                                                 abort_flag, dev_status)) ||
                            (p_cnt > 0 && !mbar_wait(&bars->pv_done[w], (p_cnt - 1) & 1,
                                                     abort_flag, dev_status))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t q_tile = sbase + L::kOffQ + sq * L::kQSub;
                        const uint32_t k_tile = sbase + L::kOffK + st * L::kKV;
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk)
                            umma_f16_ss(tm_s, desc_kmajor(q_tile, kk), desc_kmajor(k_tile, kk),
                                        idesc_qk, kk == 0 ? 0u : 1u);
                        umma_commit(&bars->s_full[w]);
                        if (diag) umma_commit(&bars->q_empty[sq]);
                        umma_commit(&bars->k_empty[st]);
                    } else {
                        mbar_arrive(&bars->k_empty[st]);
                    }
                    // every fill is observed in order, used or not (the adder's barrier when the
                    // value embedding is on), so no wait can alias a fill one lap later
                    if (!mbar_wait(AUXV ? &bars->v_add[st] : &bars->v_full[st], ph, abort_flag,
                                   dev_status)) {
                        ok = false;
                        break;
                    }
                    if (u >= 0) {
                        if (!mbar_wait(&bars->p_full[w], p_cnt & 1, abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t v_tile = sbase + L::kOffV + st * L::kKV;
#pragma unroll
                        for (int kk = 0; kk < kBlockN / 16; ++kk)
                            umma_f16_ts(tm_o, tm_s + 8 * kk, desc_v(v_tile, kk), idesc_pv,
                                        (!first || kk > 0) ? 1u : 0u);
                        umma_commit(&bars->pv_done[w]);
                        if (diag) umma_commit(&bars->o_ready[w]);
                        umma_commit(&bars->v_empty[st]);
                        ++p_cnt;
                    } else {
                        mbar_arrive(&bars->v_empty[st]);
                    }
                }
                qn += it.n_qt;
                g += n_steps;
            }
            // Wait (bounded) until every MMA this thread issued has finished.
            umma_commit(&bars->drain[w]);
            drain_wait(&bars->drain[w], 0);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax of warpgroup w
        if (AUXV)
            regs_increase<kBandRegsSoftmaxAux>();
        else
            regs_increase<kBandRegsSoftmax>();
        const int w = warp >> 2;
        const int row = threadIdx.x & 127;  // query row in the tile == TMEM lane
        const int r0 = (warp & 3) * 32;     // first row of this warp
        const uint32_t tm_lane = tmem + (static_cast<uint32_t>(r0) << 16);
        const uint32_t tm_s = tm_lane + 128 * w;
        const uint32_t tm_o = tm_lane + L::kTmO + HD * w;
        const float scale_log2 = p.scale * kLog2e;
        const uint64_t scale2 = f32x2(scale_log2, scale_log2);
        const int window = p.window;
        uint32_t s_cnt = 0, o_cnt = 0, qn = 0;
        bool ok = true;
        // Q slot whose rows this warp's TMA stores are still reading (-1: none); released once
        // the stores have read it, at the warpgroup's next tile or at the end
        int pending_slot = -1;
        auto release_pending = [&]() {
            if (pending_slot < 0) return;
            if (lane == 0) {
                tma_store_wait_read();
                mbar_arrive(&bars->q_empty[pending_slot]);
            }
            __syncwarp();
            pending_slot = -1;
        };
        if (p.test_stall_us > 0)  // the wait runs out: status 3, and every role winds down
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->stall, 0, abort_flag, dev_status,
                                                   1000ull * static_cast<uint64_t>(p.test_stall_us)));
        ItemWalk wk;
        for (wk.start(items, n_items); ok && !wk.done(); wk.advance()) {
            if (!wk.has()) continue;
            const BandItem it = decode_band(wk.cur);
            const uint32_t qn_item = qn;
            qn += it.n_qt;
            for (int u = static_cast<int>((qn_item ^ w) & 1); u < it.n_qt; u += 2) {
                release_pending();
                const uint32_t n = qn_item + u;
                const int q_start = it.q0 + kBlockM * u;
                const int nr = min(kBlockM, it.doc_end - q_start);
                const int n_t = (u + it.hp >= 1) ? 2 : 1;  // window tile (if any), causal tile
                const int i = q_start + row;
                float m = -INFINITY, l = 0.f;
                for (int t = 0; t < n_t; ++t) {
                    const int kv0 = q_start - (t + 1 < n_t ? kBlockN : 0);
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&bars->s_full[w], s_cnt & 1, abort_flag, dev_status));
                    if (!ok) break;
                    ++s_cnt;
                    tc_fence_after();
                    // visible columns of this row: [c_lo, c_hi] (keys i - window + 1 .. i)
                    const int c_lo = i - window + 1 - kv0, c_hi = i - kv0;
                    // the whole S row, one wait
                    uint32_t v[128];
#pragma unroll
                    for (int c = 0; c < 4; ++c) tmem_ld32(tm_s + 32 * c, v + 32 * c);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c) regs_after_wait(v + 32 * c);
                    // Chunks of 32 columns are classed over this warp's rows (the bounds grow with
                    // the row): wholly hidden below the first row's lower bound or above the last
                    // row's upper bound (left out of the max; P = 0 without exponentials), wholly
                    // visible inside [last row's lower bound, first row's upper bound] (no test),
                    // else partial: there hidden scores are set to -inf in place (bit e of vis[c]:
                    // column 32 c + e visible for this row). The max and the exponentials then run
                    // unmasked (2^-inf = 0).
                    uint32_t hidden = 0;   // bit c: chunk c is hidden for every row of this warp
                    uint32_t partial = 0;  // bit c: chunk c is neither wholly visible nor hidden
                    {
                        const int lo_first = q_start + r0 - window + 1 - kv0, lo_last = lo_first + 31;
                        const int hi_first = q_start + r0 - kv0, hi_last = hi_first + 31;
                        uint32_t vis[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int lo = 32 * c, hi = lo + 31;
                            const int a = c_lo - lo, b = c_hi - lo;  // visible e in [a, b]
                            const uint32_t below = a <= 0 ? 0u : (a >= 32 ? ~0u : (1u << a) - 1u);
                            const uint32_t above = b >= 31 ? 0u : (b < 0 ? ~0u : ~((2u << b) - 1u));
                            const bool none = hi < lo_first || lo > hi_last;
                            const bool all = lo >= lo_last && hi <= hi_first;
                            hidden |= none ? (1u << c) : 0u;
                            partial |= (none || all) ? 0u : (1u << c);
                            vis[c] = ~(below | above);
                        }
                        // both classes are the same for every lane of the warp: the branches are
                        // uniform, and only the partial chunks (the diagonal one for window 128)
                        // pay the per-element test
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            if ((partial >> c) & 1u) {
#pragma unroll
                                for (int e = 0; e < 32; ++e)
                                    v[32 * c + e] = ((vis[c] >> e) & 1u) ? v[32 * c + e]
                                                                         : __float_as_uint(-INFINITY);
                            }
                    }
                    // row max over the visible columns (hidden chunks hold stale scores: skipped)
                    float mx = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (!((hidden >> c) & 1u))
                            mx = fmaxf(mx, chunk_max<kMaskNone>(v + 32 * c, 32 * c, c_lo, c_hi));
                    const float m_new = fmaxf(m, mx * scale_log2);
                    // Keep the reference max until the row max grows by more than 8 (a factor
                    // 256): O / l and the lse are exact for any reference value.
                    const bool rescale = m_new > m + 8.0f;
                    const bool o_nonzero = m != -INFINITY;  // some key seen: O may be nonzero
                    const float alpha = rescale ? ex2(m - m_new) : 1.0f;
                    if (rescale) m = m_new;
                    const float neg_m = (m == -INFINITY) ? 0.f : -m;
                    const uint64_t negm2 = f32x2(neg_m, neg_m);
                    // P = 2^(s * scale * log2e - m) as bf16 into the first half of S (the whole
                    // row is in registers already)
                    uint64_t sum_a = f32x2(0.f, 0.f), sum_b = f32x2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (!((hidden >> c) & 1u)) {
                            uint32_t pk[16];
                            chunk_exp<kMaskNone>(v + 32 * c, 32 * c, c_lo, c_hi, scale2, negm2, sum_a, sum_b, pk);
                            tmem_st16(tm_s + 16 * c, pk);
                        }
                    }
                    // chunks no row of the warp sees: P = 0, no exponentials
                    if (hidden) {
                        uint32_t zero[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) zero[e] = 0u;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            if ((hidden >> c) & 1u) tmem_st16(tm_s + 16 * c, zero);
                    }
                    const uint64_t sum2 = add_f32x2(sum_a, sum_b);
                    float s_lo, s_hi;
                    f32x2_split(sum2, s_lo, s_hi);
                    l = l * alpha + (s_lo + s_hi);
                    if (t > 0 && __any_sync(0xffffffffu, rescale && o_nonzero)) {
#pragma unroll 1
                        for (int c = 0; c < HD / 32; ++c) {
                            uint32_t v[32];
                            tmem_ld32(tm_o + 32 * c, v);
                            tmem_wait_ld();
                            regs_after_wait(v);
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                            tmem_st32(tm_o + 32 * c, v);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&bars->p_full[w]);
                }
                if (!ok) break;
                // epilogue: O / l and lse for the valid rows
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars->o_ready[w], o_cnt & 1, abort_flag, dev_status));
                if (!ok) break;
                ++o_cnt;
                tc_fence_after();
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                // O / l -> bf16, staged through this tile's Q slot (its last S has completed) in
                // the slot's own layout (the TMA box layout: [hd / 64][128 rows][128 B], 16-byte
                // units XOR-swizzled by row % 8). A warp whose 32 rows all lie inside the document
                // stores them with TMA stores (one 64 x 32 box per 64 columns), asynchronously;
                // otherwise it copies its valid rows out with plain stores, two rows per
                // instruction (hd 128), so each warp store covers 512 contiguous bytes.
                uint8_t* slot_base = smem + L::kOffQ + (n % L::kQSlots) * L::kQSub;
                auto unit_addr = [&](int r, int u) -> uint8_t* {
                    return slot_base + (u >> 3) * L::kChunk + r * 128 + (((u & 7) ^ (r & 7)) << 4);
                };
                {
                    uint32_t ov[HD];
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) tmem_ld32(tm_o + 32 * c, ov + 32 * c);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        regs_after_wait(ov + 32 * c);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint32_t* w8 = ov + 32 * c + 8 * q4;
                            const uint4 w4 = make_uint4(
                                pack_bf16x2(__uint_as_float(w8[0]) * inv_l, __uint_as_float(w8[1]) * inv_l),
                                pack_bf16x2(__uint_as_float(w8[2]) * inv_l, __uint_as_float(w8[3]) * inv_l),
                                pack_bf16x2(__uint_as_float(w8[4]) * inv_l, __uint_as_float(w8[5]) * inv_l),
                                pack_bf16x2(__uint_as_float(w8[6]) * inv_l, __uint_as_float(w8[7]) * inv_l));
                            *reinterpret_cast<uint4*>(unit_addr(row, 4 * c + q4)) = w4;
                        }
                    }
                }
                if (r0 + 31 < nr) {
                    fence_proxy_async_smem();  // the rows are read by the async proxy (TMA)
                    __syncwarp();
                    if (lane == 0) {
                        for (int c = 0; c < HD / 64; ++c)
                            tma_store_2d(&tm_out, it.head * HD + 64 * c, q_start + r0,
                                         slot_base + c * L::kChunk + r0 * 128);
                        tma_store_commit();
                    }
                    // the slot may be refilled once the stores have read the rows: released at
                    // this warpgroup's next tile, off this tile's critical path
                    pending_slot = static_cast<int>(n % L::kQSlots);
                } else {
                    __syncwarp();
                    constexpr int kChunks = HD / 8;  // 16-byte units per row
                    constexpr int kRowsPerIter = 32 / kChunks;
#pragma unroll 4
                    for (int j = 0; j < 32 / kRowsPerIter; ++j) {
                        const int rl = j * kRowsPerIter + lane / kChunks;
                        const int unit = lane % kChunks;
                        if (r0 + rl < nr) {
                            const uint4 w4 = *reinterpret_cast<const uint4*>(unit_addr(r0 + rl, unit));
                            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.o) +
                                                 (static_cast<int64_t>(q_start + r0 + rl) * H + it.head) * HD +
                                                 unit * 8;
                            *reinterpret_cast<uint4*>(dst) = w4;
                        }
                    }
                    __syncwarp();
                    fence_proxy_async_smem();  // the slot's next fill is written by the async proxy
                    if (lane == 0) mbar_arrive(&bars->q_empty[n % L::kQSlots]);
                }
                tc_fence_before();
                if (row < nr && p.lse)
                    p.lse[static_cast<int64_t>(i) * H + it.head] = (m + log2f(l)) * kLn2;
            }
        }
        if (ok) release_pending();
    }

    // ---------------------------------------------------------------- teardown
    if (warp < 8 && lane == 0) tma_store_wait_all();  // the epilogue's O stores have completed
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, L::kTmemCols);
}

template <int HD, bool AUXV>
static cudaError_t launch_band_hd(const AttnProblem& p, const CUtensorMap& tq,
                                  const CUtensorMap& tk, const CUtensorMap& tv,
                                  const CUtensorMap& to, const int4* items, WorkspaceHeader* hdr,
                                  cudaStream_t stream) {
    using L = TcLayout<HD>;
    cudaError_t e = cudaFuncSetAttribute(attn_band_kernel<HD, AUXV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    // programmatic stream serialization: the prologue overlaps the scheduler kernel before it
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(AUXV ? kBandAuxThreads : kBandThreads);
    cfg.dynamicSmemBytes = L::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_band_kernel<HD, AUXV>, tq, tk, tv, to, p, items, hdr);
}

cudaError_t launch_attn_band(const AttnProblem& p, const CUtensorMap& tm_q,
                             const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_o, const int4* items, WorkspaceHeader* hdr,
                             cudaStream_t stream) {
    if (!band_applies(p)) return cudaErrorInvalidValue;
    const bool aux = p.v_aux != nullptr;
    if (p.head_dim == 128)
        return aux ? launch_band_hd<128, true>(p, tm_q, tm_k, tm_v, tm_o, items, hdr, stream)
                   : launch_band_hd<128, false>(p, tm_q, tm_k, tm_v, tm_o, items, hdr, stream);
    if (p.head_dim == 64)
        return aux ? launch_band_hd<64, true>(p, tm_q, tm_k, tm_v, tm_o, items, hdr, stream)
                   : launch_band_hd<64, false>(p, tm_q, tm_k, tm_v, tm_o, items, hdr, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pha
