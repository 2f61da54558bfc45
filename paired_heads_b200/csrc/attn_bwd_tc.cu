// attn_bwd_tc.cu -- backward of the band attention (causal, window <= 128 key slots, bf16,
// head_dim 64 or 128) on the sm_100a tensor cores.
//
// The gradients through the row softmax, with P recomputed from q, k and the forward's lse and
// D_i = dO_i . O_i precomputed (FlashAttention's backward: "Training an LLM from scratch (part 2)",
// section "4. GQA & FlashAttention"):
//   dP = dO V^T,  dS = P o (dP - D),  dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
// Tiles of 128 slots are counted from the document start, as in the forward's band decomposition
// ("modded-nanogpt Paired Head Attention record" page, section "sequence length and window
// handling"): query tile j sees key tiles j - 1 and j, so key tile j is seen by query tiles j and
// j + 1. One kernel template, two instances:
//   key-major (dK, dV): outer tile = key tile (X = K, V), inner steps = the query tiles that see
//     it, for every query head of its group (Y = Q, dO):  S^T = K Q^T, dP^T = V dO^T, then
//     dV += P^T dO and dK += dS^T Q with P^T, dS^T in TMEM as the A operand.
//   query-major (dQ): outer tile = query tile (X = Q, dO), inner steps = the key tiles it sees
//     (Y = K, V): S = Q K^T, dP = dO V^T, then dQ += dS K.
// In both, the 128 x 128 scores go to TMEM columns [0, 128), dP to [128, 256). An inner step's
// columns are split in two halves of 64 (Y rows 64 h .. 64 h + 63), one per elementwise
// warpgroup: the bf16 P and dS of half h overwrite the first 32 of the half's own columns
// (64 h + [0, 32) and 128 + 64 h + [0, 32)), and are the A operand of the half's second products
// (K = 64), issued as soon as that warpgroup is done. The accumulators sit at 256 (dV or dQ) and
// 256 + hd (dK).
// A tile loaded for the K-major S / dP product (rows = slots, [64-column chunks] 128-byte
// swizzled) is the MN-major B operand of the second product as it stands.
// Epilogue (hd 128): a warp whose 32 rows lie inside the document stages them in shared memory in
// the TMA box layout and writes them with TMA stores (dQ: a 32 KB tile, one 64 x 32 box per warp;
// dK, dV: a private 2 KB box per warp, 16 rows per store); other warps store row by row.
//
// CTA = 10 warps, persistent, one per SM, band items in snake order:
//   warps 0-7  elementwise, two warpgroups: warpgroup h takes half h of every inner step (row =
//              TMEM lane; P, dS from S, dP) and half h of the accumulator columns in the epilogue
//              (accumulators -> bf16 -> global); two warps per scheduler hide each other's latency
//   warp 8     producer: X tiles (one buffer), Y tiles (two-slot ring) by TMA; in the key-major
//              instance also lse * log2(e) and D of the fill's 128 queries into shared memory
//   warp 9     MMA issuer, owner of the 512 TMEM columns
// Every wait is bounded (1 s); on expiry the CTA records a status, drains its own copies and
// MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_common.cuh"
#include "kernels.cuh"

namespace pha {

namespace {

// 8 elementwise warps; producer, MMA issuer and two idle warps (a whole third warpgroup for the
// register split: the elementwise warpgroups hold 64 columns of S and of dP per thread)
constexpr int kBwdTcThreads = 384;

template <int HD, bool KEYMAJOR>
struct BwdLayout {
    static constexpr int kChunk = 128 * 128;   // one [128 rows][64 bf16] swizzled chunk (bytes)
    static constexpr int kTile = 128 * HD * 2;
    static constexpr int kYStages = 2;
    static constexpr int kOffX = 0;                                  // X0, X1
    static constexpr int kOffY = kOffX + 2 * kTile;                  // [stage] Y0, Y1
    // key-major: [stage] lse2[128], D[128], then per warp a 16-row x 64-column staging box (2 KB)
    // for the dK / dV TMA stores; query-major: the dQ tile staged for its TMA stores
    static constexpr int kOffVec = kOffY + kYStages * 2 * kTile;
    static constexpr int kVecBytes = KEYMAJOR ? kYStages * 2 * 128 * 4 : 0;
    static constexpr int kOffStg = kOffVec + kVecBytes;
    static constexpr int kStgBytes = KEYMAJOR ? 8 * 2048 : kTile;
    static constexpr int kOffBar = kOffStg + kStgBytes;
    static constexpr int kBarBytes = 256;
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;   // + slack to align to 1024
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kTmS = 0, kTmDP = 128, kTmAcc = 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct BwdBars {
    uint64_t x_full, x_empty;
    uint64_t y_full[2], y_empty[2];
    uint64_t s_full[2], p_full[2], m2_done[2];  // per half
    uint64_t acc_full, acc_empty, drain;
    uint32_t tmem_base;
    int abort;
};

// The steps of one outer tile (u-th tile of a band item, or the tile of a tile item).
struct OuterTile {
    int row0;     // first slot of the outer tile
    int n_sub;    // inner steps
    int nq;       // key-major: query tiles per head (band: 1 or 2)
    int first;    // GEN: document tile index of the first inner step's Y tile
};

// GEN (tile items, any causal / window setting): query-major, the key tiles the query tile sees;
// key-major, the query tiles that see the key tile, for every query head of its group. Tiles are
// the document's 128-slot tiles counted from its start.
template <bool KEYMAJOR, bool GEN>
__device__ __forceinline__ OuterTile outer_tile(const BandItem& it, int u, int G,
                                                const AttnProblem& p) {
    OuterTile o;
    o.row0 = it.q0 + kBlockM * u;
    o.first = 0;
    if (GEN) {
        const int a = it.doc_start, b = it.doc_end;
        const int j = (o.row0 - a) / kBlockN, last = (b - a - 1) / kBlockN;
        int lo = 0, hi = last;
        if (!KEYMAJOR) {
            if (p.causal) {
                hi = j;
                if (p.window > 0 && o.row0 - p.window + 1 > a) lo = (o.row0 - p.window + 1 - a) / kBlockN;
            }
            o.nq = 0;
            o.n_sub = hi - lo + 1;
        } else {
            if (p.causal) {
                lo = j;
                if (p.window > 0) {
                    const int n_rows = min(kBlockM, b - o.row0);
                    const int q_last = o.row0 + n_rows - 1 + p.window - 1;
                    hi = ((q_last < b ? q_last : b - 1) - a) / kBlockN;
                }
            }
            o.nq = hi - lo + 1;
            o.n_sub = G * o.nq;
        }
        o.first = lo;
        return o;
    }
    if (KEYMAJOR) {
        o.nq = o.row0 + kBlockM < it.doc_end ? 2 : 1;  // the diagonal query tile, then the next
        o.n_sub = G * o.nq;
    } else {
        o.nq = 0;
        o.n_sub = (u + it.hp >= 1) ? 2 : 1;  // the previous key tile (if any), then the diagonal
    }
    return o;
}

// Inner step s of an outer tile: the head and first slot of its Y tiles.
template <bool KEYMAJOR, bool GEN>
__device__ __forceinline__ void inner_step(const BandItem& it, const OuterTile& o, int s, int G,
                                           int& y_head, int& y_row) {
    if (GEN) {
        if (KEYMAJOR) {
            y_head = (it.head / G) * G + s / o.nq;
            y_row = it.doc_start + kBlockN * (o.first + s % o.nq);
        } else {
            y_head = it.head / G;
            y_row = it.doc_start + kBlockN * (o.first + s);
        }
        return;
    }
    if (KEYMAJOR) {
        const int g = it.head / G;
        y_head = g * G + s / o.nq;
        y_row = o.row0 + kBlockM * (s % o.nq);
    } else {
        y_head = it.head / G;
        y_row = o.row0 - (s + 1 < o.n_sub ? kBlockN : 0);
    }
}

// Items of the key-major instance: one per kv head (the item of the group's first query head);
// its item walk visits only those (ItemWalk with the head group), so this always holds there.
template <bool KEYMAJOR>
__device__ __forceinline__ bool item_used(const BandItem& it, int G) {
    return !KEYMAJOR || it.head % G == 0;
}

// Y fills (two-slot ring) and the inner steps that read them. With reuse, a Y tile shared by
// consecutive outer tiles of a run is filled once: query-major, the key tile of q-tile u's
// diagonal step is the previous-tile step of q-tile u + 1; key-major with one query head per kv
// head, the query tile of key tile u's next-tile step is the diagonal step of key tile u + 1.
// Without reuse (key-major, several query heads per kv head) every step has its own fill.
struct StepFill {
    uint32_t idx;  // position in this CTA's fill sequence: slot idx & 1, lap idx >> 1
    bool first;    // the step is the fill's first reader (the producer loads it for this step)
    bool last;     // ... and its last reader (the slot is released after the step)
};

template <bool KEYMAJOR>
struct FillTrack {
    uint32_t n = 0;      // fills so far
    uint32_t carry = 0;  // the fill the next outer tile's shared step reads
    __device__ __forceinline__ StepFill step(bool reuse, int u, int n_tiles, int s, int n_sub) {
        StepFill f;
        if (!reuse) {
            f.idx = n++;
            f.first = f.last = true;
            return f;
        }
        // the step shared with the previous outer tile: query-major the previous key tile (the
        // first of two steps), key-major the diagonal query tile (step 0)
        const bool shared = KEYMAJOR ? s == 0 : s + 1 < n_sub;
        if (shared) {
            f.first = u == 0;  // a run's first tile has no predecessor that filled it
            f.idx = f.first ? n++ : carry;
            f.last = true;
        } else {
            f.idx = n++;
            f.first = true;
            f.last = u + 1 == n_tiles;  // else carried to the next outer tile
            carry = f.idx;
        }
        return f;
    }
};

template <int HD, bool KEYMAJOR, bool GEN>
__global__ void __launch_bounds__(kBwdTcThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_st,
                       const __grid_constant__ CUtensorMap tm_st2, const AttnProblem p,
                       const float* __restrict__ dsum, __nv_bfloat16* __restrict__ out_a,
                       __nv_bfloat16* __restrict__ out_b, const int4* __restrict__ items,
                       WorkspaceHeader* hdr) {
    // out_a: dQ (query-major) or dK (key-major); out_b: dV (key-major); tm_st: a map over dQ with
    // a 64 x 32 box (query-major) or over dK with a 64 x 16 box (key-major); tm_st2: over dV with a
    // 64 x 16 box (key-major)
    using L = BwdLayout<HD, KEYMAJOR>;
    static_assert(sizeof(BwdBars) <= L::kBarBytes, "barrier block");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const uint32_t sbase = smem_u32(smem);
    BwdBars* bars = reinterpret_cast<BwdBars*>(smem + L::kOffBar);
    float* vec = reinterpret_cast<float*>(smem + L::kOffVec);
    volatile int* abort_flag = &bars->abort;
    int* dev_status = &hdr->status;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 8 && lane == 0) {
        mbar_init(&bars->x_full, 1);
        mbar_init(&bars->x_empty, 1);
        for (int s = 0; s < 2; ++s) {
            // the TMA arrival, plus (key-major) the 32 producer lanes after writing lse2 / D
            mbar_init(&bars->y_full[s], KEYMAJOR ? 33 : 1);
            mbar_init(&bars->y_empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bars->s_full[h], 1);
            mbar_init(&bars->p_full[h], 128);
            mbar_init(&bars->m2_done[h], 1);
        }
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->acc_empty, 256);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
    }
    if (warp == 9) {
        tmem_alloc(&bars->tmem_base, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    const int n_items = *reinterpret_cast<volatile int*>(&hdr->n_items);
    const int H = p.heads, Hkv = p.kv_heads, G = H / Hkv;
    static_assert(8 * kTcRegsSoftmax + 4 * kTcRegsOther <= 12 * 168, "register split");
    if (warp >= 8) regs_decrease<kTcRegsOther>();  // the whole third warpgroup, then its roles
    const bool reuse = !GEN && (!KEYMAJOR || G == 1);
    // X = (K, V) and Y = (Q, dO) (key-major), or the other way round
    const CUtensorMap* mx0 = KEYMAJOR ? &tm_k : &tm_q;
    const CUtensorMap* mx1 = KEYMAJOR ? &tm_v : &tm_do;
    const CUtensorMap* my0 = KEYMAJOR ? &tm_q : &tm_k;
    const CUtensorMap* my1 = KEYMAJOR ? &tm_do : &tm_v;

    if (warp >= 10) {
        // ------------------------------------------------------------ idle (register split only)
    } else if (warp == 8) {
        // ------------------------------------------------------------ producer
        // Per outer tile: with reuse its new Y fills, then X (the order in which their slots are
        // released); without, X and then one fill per step.
        uint32_t oc = 0;  // outer tiles issued so far
        FillTrack<KEYMAJOR> ft;
        bool ok = true;
        auto load_y = [&](const BandItem& it, const OuterTile& o, int s, uint32_t idx) -> bool {
            const uint32_t st = idx & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->y_empty[st], ((idx >> 1) & 1) ^ 1,
                                                   abort_flag, dev_status)))
                return false;
            int y_head, y_row;
            inner_step<KEYMAJOR, GEN>(it, o, s, G, y_head, y_row);
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars->y_full[st], 2 * L::kTile);
                uint8_t* y = smem + L::kOffY + st * 2 * L::kTile;
                for (int c = 0; c < HD / 64; ++c) {
                    tma_load_2d(y + c * L::kChunk, my0, y_head * HD + 64 * c, y_row, &bars->y_full[st]);
                    tma_load_2d(y + L::kTile + c * L::kChunk, my1, y_head * HD + 64 * c, y_row,
                                &bars->y_full[st]);
                }
            }
            if (KEYMAJOR) {
                // lse * log2(e) and D of the fill's queries (0 past the document end)
                float* l2 = vec + st * 256;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * lane + e, qs = y_row + c;
                    const bool in = qs < it.doc_end;
                    const int64_t r = static_cast<int64_t>(qs) * H + y_head;
                    l2[c] = in ? p.lse[r] * kLog2e : 0.f;
                    l2[128 + c] = in ? dsum[r] : 0.f;
                }
                mbar_arrive(&bars->y_full[st]);
            }
            return true;
        };
        ItemWalk wk;
        for (wk.start(items, n_items, KEYMAJOR ? G : 1, H); ok && !wk.done(); wk.advance()) {
            if (!wk.has()) continue;
            const BandItem it = decode_band(wk.cur);
            if (!item_used<KEYMAJOR>(it, G)) continue;
            const int x_head = KEYMAJOR ? it.head / G : it.head;
            for (int u = 0; ok && u < it.n_qt; ++u) {
                const OuterTile o = outer_tile<KEYMAJOR, GEN>(it, u, G, p);
                for (int s = 0; ok && reuse && s < o.n_sub; ++s) {
                    const StepFill f = ft.step(true, u, it.n_qt, s, o.n_sub);
                    if (f.first) ok = load_y(it, o, s, f.idx);
                }
                if (!ok) break;
                ok = __all_sync(0xffffffffu, mbar_wait(&bars->x_empty, (oc & 1) ^ 1, abort_flag,
                                                       dev_status));
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars->x_full, 2 * L::kTile);
                    for (int c = 0; c < HD / 64; ++c) {
                        tma_load_2d(smem + L::kOffX + c * L::kChunk, mx0, x_head * HD + 64 * c,
                                    o.row0, &bars->x_full);
                        tma_load_2d(smem + L::kOffX + L::kTile + c * L::kChunk, mx1,
                                    x_head * HD + 64 * c, o.row0, &bars->x_full);
                    }
                }
                ++oc;
                for (int s = 0; ok && !reuse && s < o.n_sub; ++s)
                    ok = load_y(it, o, s, ft.step(false, u, it.n_qt, s, o.n_sub).idx);
            }
        }
        if (!ok && lane == 0) {
            // Wait (bounded) for the copies this warp issued last into every buffer.
            if (oc > 0) drain_wait(&bars->x_full, (oc - 1) & 1);
            for (uint32_t n = ft.n > 2 ? ft.n - 2 : 0; n < ft.n; ++n)
                drain_wait(&bars->y_full[n & 1], (n >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc1 = idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
            constexpr uint32_t idesc2 = idesc_bf16_f32(kBlockM, HD, 0, 1);
            const uint32_t tm_s = tmem + L::kTmS, tm_dp = tmem + L::kTmDP;
            const uint32_t tm_acc_p = tmem + L::kTmAcc;                         // dV
            const uint32_t tm_acc_ds = tmem + L::kTmAcc + (KEYMAJOR ? HD : 0);  // dK or dQ
            const uint32_t x0 = sbase + L::kOffX, x1 = x0 + L::kTile;
            uint32_t oc = 0, sc = 0;
            FillTrack<KEYMAJOR> ft;
            bool ok = true;
            ItemWalk wk;
            for (wk.start(items, n_items, KEYMAJOR ? G : 1, H); ok && !wk.done(); wk.advance()) {
                if (!wk.has()) continue;
                const BandItem it = decode_band(wk.cur);
                if (!item_used<KEYMAJOR>(it, G)) continue;
                for (int u = 0; ok && u < it.n_qt; ++u) {
                    const OuterTile o = outer_tile<KEYMAJOR, GEN>(it, u, G, p);
                    if (!mbar_wait(&bars->x_full, oc & 1, abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    for (int s = 0; s < o.n_sub; ++s) {
                        const StepFill f = ft.step(reuse, u, it.n_qt, s, o.n_sub);
                        const uint32_t st = f.idx & 1;
                        const uint32_t y0 = sbase + L::kOffY + st * 2 * L::kTile, y1 = y0 + L::kTile;
                        // each fill is waited for once, by its first reader, in fill order
                        if (f.first &&
                            !mbar_wait(&bars->y_full[st], (f.idx >> 1) & 1, abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        // S = X0 Y0^T and dP = X1 Y1^T at full width (N = 128); their columns are free
                        // once the previous step's second products of both halves are done
                        for (int h = 0; ok && h < 2; ++h)
                            if (sc > 0 && !mbar_wait(&bars->m2_done[h], (sc - 1) & 1, abort_flag,
                                                     dev_status))
                                ok = false;
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk) {
                            umma_f16_ss(tm_s, desc_kmajor(x0, kk), desc_kmajor(y0, kk), idesc1,
                                        kk == 0 ? 0u : 1u);
                            umma_f16_ss(tm_dp, desc_kmajor(x1, kk), desc_kmajor(y1, kk), idesc1,
                                        kk == 0 ? 0u : 1u);
                        }
                        umma_commit(&bars->s_full[0]);  // one per elementwise warpgroup
                        umma_commit(&bars->s_full[1]);
                        if (!ok) break;
                        if (s + 1 == o.n_sub) umma_commit(&bars->x_empty);
                        // second products of half h: K = the half's 64 Y rows
                        for (int h = 0; ok && h < 2; ++h) {
                            if (!mbar_wait(&bars->p_full[h], sc & 1, abort_flag, dev_status) ||
                                (s == 0 && h == 0 && oc > 0 &&
                                 !mbar_wait(&bars->acc_empty, (oc - 1) & 1, abort_flag, dev_status))) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t acc = (s > 0 || h > 0 || kk > 0) ? 1u : 0u;
                                umma_f16_ts(tm_acc_ds, tm_dp + 64 * h + 8 * kk, desc_v(y0, 4 * h + kk),
                                            idesc2, acc);
                                if (KEYMAJOR)
                                    umma_f16_ts(tm_acc_p, tm_s + 64 * h + 8 * kk, desc_v(y1, 4 * h + kk),
                                                idesc2, acc);
                            }
                            umma_commit(&bars->m2_done[h]);
                        }
                        if (!ok) break;
                        if (f.last) umma_commit(&bars->y_empty[st]);
                        if (s + 1 == o.n_sub) umma_commit(&bars->acc_full);
                        ++sc;
                    }
                    ++oc;
                }
            }
            // Wait (bounded) until every MMA this thread issued has finished.
            umma_commit(&bars->drain);
            drain_wait(&bars->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ elementwise warpgroups
        regs_increase<kTcRegsSoftmax>();
        const int h = warp >> 2;              // the half of every step this warpgroup takes
        const int row = threadIdx.x & 127;    // TMEM lane == row of the outer tile
        const int r0 = (warp & 3) * 32;       // first row of this warp
        const uint32_t tm_lane = tmem + (static_cast<uint32_t>(r0) << 16);
        const float scale_log2 = p.scale * kLog2e;
        const int window = p.window;
        uint32_t oc = 0, sc = 0;
        FillTrack<KEYMAJOR> ft;
        bool ok = true;
        ItemWalk wk;
        for (wk.start(items, n_items, KEYMAJOR ? G : 1, H); ok && !wk.done(); wk.advance()) {
            if (!wk.has()) continue;
            const BandItem it = decode_band(wk.cur);
            if (!item_used<KEYMAJOR>(it, G)) continue;
            for (int u = 0; ok && u < it.n_qt; ++u) {
                const OuterTile o = outer_tile<KEYMAJOR, GEN>(it, u, G, p);
                const int slot = o.row0 + row;  // key slot (key-major) or query slot
                const bool valid = slot < it.doc_end;
                float lse2 = 0.f, dd = 0.f;  // query-major: this row's lse * log2(e) and D
                if (!KEYMAJOR && valid) {
                    const int64_t r = static_cast<int64_t>(slot) * H + it.head;
                    lse2 = p.lse[r] * kLog2e;
                    dd = dsum[r];
                }
                for (int s = 0; s < o.n_sub; ++s) {
                    const StepFill f = ft.step(reuse, u, it.n_qt, s, o.n_sub);
                    const uint32_t st = f.idx & 1;
                    int y_head, y_row;
                    inner_step<KEYMAJOR, GEN>(it, o, s, G, y_head, y_row);
                    // visible columns [c_lo, c_hi] of this row
                    int c_lo, c_hi;
                    if (GEN) {
                        const int a = it.doc_start, b = it.doc_end;
                        if (KEYMAJOR) {  // the queries that see key `slot`
                            c_lo = (p.causal ? slot : a) - y_row;
                            c_hi = ((p.causal && window > 0) ? min(slot + window - 1, b - 1) : b - 1) - y_row;
                        } else {         // the keys query `slot` sees
                            c_lo = ((window > 0) ? max(a, slot - window + 1) : a) - y_row;
                            c_hi = (p.causal ? slot : b - 1) - y_row;
                        }
                        if (!valid) c_hi = c_lo - 1;
                    } else if (KEYMAJOR) {  // queries slot .. slot + window - 1, inside the document
                        c_lo = slot - y_row;
                        c_hi = min(slot + window - 1, it.doc_end - 1) - y_row;
                    } else {         // keys slot - window + 1 .. slot
                        c_lo = slot - window + 1 - y_row;
                        c_hi = valid ? slot - y_row : c_lo - 1;
                    }
                    // key-major: the fill's lse2 / D (every reader waits; a fill's slot is not
                    // refilled before its last reader has finished, so no wait can see a later lap)
                    if (KEYMAJOR)
                        ok = __all_sync(0xffffffffu, mbar_wait(&bars->y_full[st], (f.idx >> 1) & 1,
                                                               abort_flag, dev_status));
                    if (!ok) break;
                    const int w_lo = __reduce_min_sync(0xffffffffu, c_lo);
                    const int w_hi = __reduce_max_sync(0xffffffffu, c_hi);
                    const float* l2v = vec + st * 256;
                    {
                        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[h], sc & 1, abort_flag,
                                                               dev_status));
                        if (!ok) break;
                        tc_fence_after();
                        // the half's 64 columns of S and dP, one wait
                        uint32_t sv[64], dv[64];
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            tmem_ld32(tm_lane + L::kTmS + 32 * (2 * h + cc), sv + 32 * cc);
                            tmem_ld32(tm_lane + L::kTmDP + 32 * (2 * h + cc), dv + 32 * cc);
                        }
                        tmem_wait_ld();
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            regs_after_wait(sv + 32 * cc);
                            regs_after_wait(dv + 32 * cc);
                        }
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const int c = 2 * h + cc;
                            uint32_t pk[16], dk[16];
#pragma unroll
                            for (int e = 0; e < 32; e += 4) {
                                // key-major: the four columns' lse * log2(e) and D, one broadcast
                                // 16-byte shared load each
                                float l2q[4] = {lse2, lse2, lse2, lse2}, dq4[4] = {dd, dd, dd, dd};
                                if (KEYMAJOR) {
                                    const float4 a4 = *reinterpret_cast<const float4*>(l2v + 32 * c + e);
                                    const float4 b4 = *reinterpret_cast<const float4*>(l2v + 128 + 32 * c + e);
                                    l2q[0] = a4.x; l2q[1] = a4.y; l2q[2] = a4.z; l2q[3] = a4.w;
                                    dq4[0] = b4.x; dq4[1] = b4.y; dq4[2] = b4.z; dq4[3] = b4.w;
                                }
                                float pr[4], dr[4];
#pragma unroll
                                for (int x = 0; x < 4; ++x) {
                                    const int col = 32 * c + e + x;
                                    const bool vis = col >= c_lo && col <= c_hi;
                                    const float pe = ex2(fmaf(__uint_as_float(sv[32 * cc + e + x]), scale_log2, -l2q[x]));
                                    pr[x] = vis ? pe : 0.f;
                                    dr[x] = pr[x] * (__uint_as_float(dv[32 * cc + e + x]) - dq4[x]);
                                }
                                pk[e >> 1] = pack_bf16x2(pr[0], pr[1]);
                                pk[(e >> 1) + 1] = pack_bf16x2(pr[2], pr[3]);
                                dk[e >> 1] = pack_bf16x2(dr[0], dr[1]);
                                dk[(e >> 1) + 1] = pack_bf16x2(dr[2], dr[3]);
                            }
                            // packed pairs of the half's 64 columns: 32 TMEM columns from 64 h, over
                            // columns of this half already read
                            if (KEYMAJOR) tmem_st16(tm_lane + L::kTmS + 16 * c + 32 * h, pk);
                            tmem_st16(tm_lane + L::kTmDP + 16 * c + 32 * h, dk);
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&bars->p_full[h]);
                    }
                    if (!ok) break;
                    ++sc;
                }
                if (!ok) break;
                // epilogue: accumulators -> bf16 rows of dQ, or of dK (scaled) and dV
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars->acc_full, oc & 1, abort_flag, dev_status));
                if (!ok) break;
                ++oc;
                tc_fence_after();
                const int out_heads = KEYMAJOR ? Hkv : H;
                const int out_head = KEYMAJOR ? it.head / G : it.head;
                const int64_t base = (static_cast<int64_t>(slot) * out_heads + out_head) * HD;
                // key-major with hd 128, a warp whose 32 rows all lie inside the document: its
                // rows of dK (times scale), then of dV (this warpgroup's 64 columns) go out
                // through its 2 KB staging box, 16 rows (one TMA store) at a time
                const bool tma_km = KEYMAJOR && HD == 128 && o.row0 + r0 + 31 < it.doc_end;
                if (tma_km) {
                    uint8_t* stg = smem + L::kOffStg + warp * 2048;
#pragma unroll 1
                    for (int a = 0; a < 2; ++a) {
                        const uint32_t col0 = L::kTmAcc + (a == 0 ? HD : 0);
                        const float mul = a == 0 ? p.scale : 1.f;
                        uint4 w8[8];
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            uint32_t v[32];
                            tmem_ld32(tm_lane + col0 + 32 * (2 * h + cc), v);
                            tmem_wait_ld();
                            regs_after_wait(v);
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                w8[4 * cc + q4] = make_uint4(
                                    pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * mul, __uint_as_float(v[8 * q4 + 1]) * mul),
                                    pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * mul, __uint_as_float(v[8 * q4 + 3]) * mul),
                                    pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * mul, __uint_as_float(v[8 * q4 + 5]) * mul),
                                    pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * mul, __uint_as_float(v[8 * q4 + 7]) * mul));
                        }
#pragma unroll 1
                        for (int half = 0; half < 2; ++half) {
                            if ((lane >> 4) == half) {
                                const int r = lane & 15;  // row of the 16-row box
#pragma unroll
                                for (int u = 0; u < 8; ++u)
                                    *reinterpret_cast<uint4*>(stg + r * 128 + ((u ^ (r & 7)) << 4)) = w8[u];
                            }
                            fence_proxy_async_smem();  // the rows are read by the async proxy (TMA)
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_2d(a == 0 ? &tm_st : &tm_st2, (it.head / G) * HD + 64 * h,
                                             o.row0 + r0 + 16 * half, stg);
                                tma_store_commit();
                                tma_store_wait_read();  // the box is rewritten next
                            }
                            __syncwarp();
                        }
                    }
                }
                // query-major with hd 128 (warpgroup h owns the 64-column chunk h), a warp whose 32
                // rows all lie inside the document: its dQ rows are staged in the TMA box layout
                // and written by one TMA store; otherwise every thread stores its own row
                const bool tma_rows = !KEYMAJOR && HD == 128 && o.row0 + r0 + 31 < it.doc_end;
#pragma unroll 1
                for (int a = 0; !tma_km && a < (KEYMAJOR ? 2 : 1); ++a) {
                    // a = 0: the dS product (dQ or dK, times scale); a = 1: dV
                    const uint32_t col0 = L::kTmAcc + (KEYMAJOR && a == 0 ? HD : 0);
                    const float mul = a == 0 ? p.scale : 1.f;
                    __nv_bfloat16* dst = (a == 0 ? out_a : out_b) + base;
#pragma unroll 1
                    for (int c = h * (HD / 64); c < (h + 1) * (HD / 64); ++c) {  // this half's columns
                        uint32_t v[32];
                        tmem_ld32(tm_lane + col0 + 32 * c, v);
                        tmem_wait_ld();
                        regs_after_wait(v);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint4 w4 = make_uint4(
                                pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * mul, __uint_as_float(v[8 * q4 + 1]) * mul),
                                pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * mul, __uint_as_float(v[8 * q4 + 3]) * mul),
                                pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * mul, __uint_as_float(v[8 * q4 + 5]) * mul),
                                pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * mul, __uint_as_float(v[8 * q4 + 7]) * mul));
                            if (tma_rows) {
                                const int u = 4 * c + q4;  // 16-byte unit of the row
                                *reinterpret_cast<uint4*>(smem + L::kOffStg + (u >> 3) * L::kChunk +
                                                          row * 128 + (((u & 7) ^ (row & 7)) << 4)) = w4;
                            } else if (valid) {
                                *reinterpret_cast<uint4*>(dst + 32 * c + 8 * q4) = w4;
                            }
                        }
                    }
                }
                if (!KEYMAJOR && tma_rows) {
                    fence_proxy_async_smem();  // the rows are read by the async proxy (TMA)
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tm_st, it.head * HD + 64 * h, o.row0 + r0,
                                     smem + L::kOffStg + h * L::kChunk + r0 * 128);
                        tma_store_commit();
                        tma_store_wait_read();  // the staging area is rewritten by the next tile
                    }
                    __syncwarp();
                }
                tc_fence_before();
                mbar_arrive(&bars->acc_empty);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    if (warp < 8 && lane == 0) tma_store_wait_all();  // the epilogue's TMA stores have completed
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, L::kTmemCols);
}

template <int HD, bool KEYMAJOR, bool GEN>
cudaError_t launch_bwd_tc_one(const AttnProblem& p, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const CUtensorMap& tdo,
                              const CUtensorMap& tst, const CUtensorMap& tst2, const float* dsum,
                              __nv_bfloat16* out_a, __nv_bfloat16* out_b, const int4* items,
                              WorkspaceHeader* hdr, int sms, cudaStream_t stream) {
    using L = BwdLayout<HD, KEYMAJOR>;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel<HD, KEYMAJOR, GEN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    attn_bwd_tc_kernel<HD, KEYMAJOR, GEN><<<sms, kBwdTcThreads, L::kSmemBytes, stream>>>(
        tq, tk, tv, tdo, tst, tst2, p, dsum, out_a, out_b, items, hdr);
    return cudaGetLastError();
}

template <int HD, bool GEN>
cudaError_t launch_bwd_tc_hd(const AttnProblem& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& tdo,
                             const CUtensorMap& tdq, const CUtensorMap& tdk,
                             const CUtensorMap& tdv, const float* dsum,
                             void* dq, void* dk, void* dv, const int4* items, WorkspaceHeader* hdr,
                             int which, cudaStream_t stream) {
    int dev = 0, sms = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((which & 1) &&
        (e = launch_bwd_tc_one<HD, false, GEN>(p, tq, tk, tv, tdo, tdq, tdq, dsum,
                                               static_cast<__nv_bfloat16*>(dq), nullptr, items, hdr,
                                               sms, stream)) != cudaSuccess)
        return e;
    if (which & 2)
        return launch_bwd_tc_one<HD, true, GEN>(p, tq, tk, tv, tdo, tdk, tdv, dsum,
                                                static_cast<__nv_bfloat16*>(dk),
                                                static_cast<__nv_bfloat16*>(dv), items, hdr, sms,
                                                stream);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const AttnProblem& p, const CUtensorMap& tm_q,
                               const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                               const CUtensorMap& tm_do, const CUtensorMap& tm_dq,
                               const CUtensorMap& tm_dk, const CUtensorMap& tm_dv,
                               const float* dsum, void* dq, void* dk, void* dv, const int4* items,
                               WorkspaceHeader* hdr, int which, cudaStream_t stream) {
    const bool band = band_applies(p);
    if (p.head_dim == 128)
        return band ? launch_bwd_tc_hd<128, false>(p, tm_q, tm_k, tm_v, tm_do, tm_dq, tm_dk, tm_dv, dsum, dq,
                                                   dk, dv, items, hdr, which, stream)
                    : launch_bwd_tc_hd<128, true>(p, tm_q, tm_k, tm_v, tm_do, tm_dq, tm_dk, tm_dv, dsum, dq,
                                                  dk, dv, items, hdr, which, stream);
    if (p.head_dim == 64)
        return band ? launch_bwd_tc_hd<64, false>(p, tm_q, tm_k, tm_v, tm_do, tm_dq, tm_dk, tm_dv, dsum, dq,
                                                  dk, dv, items, hdr, which, stream)
                    : launch_bwd_tc_hd<64, true>(p, tm_q, tm_k, tm_v, tm_do, tm_dq, tm_dk, tm_dv, dsum, dq,
                                                 dk, dv, items, hdr, which, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pha
