// attn_common.cuh -- pieces shared by the two tcgen05 attention kernels (attn_tc.cu: blocks of
// 256 query slots with shared key tiles; attn_band.cu: sliding runs for windows <= 128): shared
// memory layout, barriers, matrix descriptors and the softmax row routines.
#pragma once

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
    static constexpr int kQSub = kBlockM * HD * 2;
    static constexpr int kKV = kBlockN * HD * 2;
    static constexpr int kQSlots = 3;
    static constexpr int kKStages = HD == 128 ? 2 : 4;
    static constexpr int kVStages = HD == 128 ? 2 : 4;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQSlots * kQSub;
    static constexpr int kOffV = kOffK + kKStages * kKV;
    static constexpr int kOffBar = kOffV + kVStages * kKV;
    static constexpr int kBarBytes = 512;
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + slack to align to 1024
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kTmO = 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct TcBars {
    uint64_t q_full[3], q_empty[3];
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    uint64_t s_full[2], p_full[2], pv_done[2], o_ready[2];
    uint64_t s_free[2];                // hd 64: the softmax has read S_r into registers
    uint64_t v8_full[2], v8_empty[2];  // FP8: the e4m3 V staging ring
    uint64_t v_add[4];                 // value embedding: aux_v added to the landed V tile
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// Block kernel (attn_tc.cu): two softmax warpgroups, then a third warpgroup whose warps 8 and 9 are
// the TMA producer and the MMA issuer (10 and 11 only give the register split a whole warpgroup).
constexpr int kTcThreads = 384;
// Register split of the block kernel, per thread: the softmax warpgroups hold a whole 128-column
// score row in registers. 8 warps x 200 + 4 warps x 88 = 1952 <= 12 warps x 168 (the launch
// allocation), so the increase never waits for registers that cannot be freed.
constexpr int kTcRegsSoftmax = 200;
constexpr int kTcRegsOther = 88;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Drain wait used on the exit path: bounded, ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_test(bar, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs) return;
}

// K-major 128-row tile (Q or K): k-step kk covers 16 bf16 of the contraction dimension.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
}
// MN-major V tile ([keys][hd] in 64-column chunks): k-step kk covers 16 keys.
__device__ __forceinline__ uint64_t desc_v(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + kk * 2048, 16384, 1024);
}

// Mask modes of one (sub-tile, key tile): which column bounds some row of the tile needs.
enum : int { kMaskNone = 0, kMaskLo = 1, kMaskHi = 2, kMaskBoth = 3 };

template <int MODE>
__device__ __forceinline__ float mask_col(float s, int c, int c_lo, int c_hi) {
    if (MODE & kMaskLo) s = c < c_lo ? -INFINITY : s;
    if (MODE & kMaskHi) s = c > c_hi ? -INFINITY : s;
    return s;
}

// Pass 1 over 32 columns starting at `base`: running max of the visible scores.
template <int MODE>
__device__ __forceinline__ float row_max32(const uint32_t* v, int base, int c_lo, int c_hi, float mx) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const float a = mask_col<MODE>(__uint_as_float(v[e]), base + e, c_lo, c_hi);
        const float b = mask_col<MODE>(__uint_as_float(v[e + 1]), base + e + 1, c_lo, c_hi);
        mx = fmax3(mx, a, b);
    }
    return mx;
}

// Pass 2 over 32 columns: 16 packed bf16 pairs of p = 2^(s * scale_log2 - m), 0 where masked.
template <int MODE>
__device__ __forceinline__ uint64_t row_exp32(const uint32_t* v, int base, int c_lo, int c_hi,
                                              uint64_t scale2, uint64_t negm2, uint64_t sum2,
                                              uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const float a = mask_col<MODE>(__uint_as_float(v[e]), base + e, c_lo, c_hi);
        const float b = mask_col<MODE>(__uint_as_float(v[e + 1]), base + e + 1, c_lo, c_hi);
        float xa, xb;
        f32x2_split(fma_f32x2(f32x2(a, b), scale2, negm2), xa, xb);
        const float pa = ex2(xa), pb = ex2(xb);
        sum2 = add_f32x2(sum2, f32x2(pa, pb));
        pk[e >> 1] = pack_bf16x2(pa, pb);
    }
    return sum2;
}

// Pass 1 over 64 columns starting at `base`: running max of the visible scores.
template <int MODE>
__device__ __forceinline__ float row_max64(const uint32_t* v, int base, int c_lo, int c_hi,
                                           float mx) {
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const float a = mask_col<MODE>(__uint_as_float(v[e]), base + e, c_lo, c_hi);
        const float b = mask_col<MODE>(__uint_as_float(v[e + 1]), base + e + 1, c_lo, c_hi);
        mx = fmax3(mx, a, b);
    }
    return mx;
}

// Pass 2 over 64 columns: p = 2^(s * scale_log2 - m) for the visible scores (0 elsewhere),
// packed into 32 bf16 pairs; returns the (two-lane) partial row sum.
template <int MODE>
__device__ __forceinline__ uint64_t row_exp64(const uint32_t* v, int base, int c_lo, int c_hi,
                                              uint64_t scale2, uint64_t negm2, uint64_t sum2,
                                              uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const float a = mask_col<MODE>(__uint_as_float(v[e]), base + e, c_lo, c_hi);
        const float b = mask_col<MODE>(__uint_as_float(v[e + 1]), base + e + 1, c_lo, c_hi);
        float xa, xb;
        f32x2_split(fma_f32x2(f32x2(a, b), scale2, negm2), xa, xb);
        const float pa = ex2(xa), pb = ex2(xb);
        sum2 = add_f32x2(sum2, f32x2(pa, pb));
        pk[e >> 1] = pack_bf16x2(pa, pb);
    }
    return sum2;
}

// Row routines over a whole 32-column chunk held in registers, with independent accumulator
// chains (the max and the sum are associative up to rounding of the sum, which the softmax's
// float32 accumulation already allows).

// Max of the visible scores among 32 columns starting at `base` (-inf if none is visible).
template <int MODE>
__device__ __forceinline__ float chunk_max(const uint32_t* v, int base, int c_lo, int c_hi) {
    float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            m[j] = fmax3(m[j], mask_col<MODE>(__uint_as_float(v[e + 2 * j]), base + e + 2 * j, c_lo, c_hi),
                         mask_col<MODE>(__uint_as_float(v[e + 2 * j + 1]), base + e + 2 * j + 1, c_lo, c_hi));
    }
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// p = 2^(s * scale_log2 - m) for 32 columns (0 where masked), packed into 16 bf16 pairs (f16
// pairs when F16P); the values are added into two packed partial sums.
template <int MODE, bool F16P = false>
__device__ __forceinline__ void chunk_exp(const uint32_t* v, int base, int c_lo, int c_hi,
                                          uint64_t scale2, uint64_t negm2, uint64_t& sum_a,
                                          uint64_t& sum_b, uint32_t* pk) {
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        const float a0 = mask_col<MODE>(__uint_as_float(v[e]), base + e, c_lo, c_hi);
        const float a1 = mask_col<MODE>(__uint_as_float(v[e + 1]), base + e + 1, c_lo, c_hi);
        const float a2 = mask_col<MODE>(__uint_as_float(v[e + 2]), base + e + 2, c_lo, c_hi);
        const float a3 = mask_col<MODE>(__uint_as_float(v[e + 3]), base + e + 3, c_lo, c_hi);
        float x0, x1, x2, x3;
        f32x2_split(fma_f32x2(f32x2(a0, a1), scale2, negm2), x0, x1);
        f32x2_split(fma_f32x2(f32x2(a2, a3), scale2, negm2), x2, x3);
        const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
        sum_a = add_f32x2(sum_a, f32x2(p0, p1));
        sum_b = add_f32x2(sum_b, f32x2(p2, p3));
        pk[e >> 1] = F16P ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
        pk[(e >> 1) + 1] = F16P ? pack_f16x2(p2, p3) : pack_bf16x2(p2, p3);
    }
}

// Adder threads (value embedding): add rows [row0, row0 + 128) of aux_v (head hs of the slot
// view, heads_slot heads per slot row, the same layout as v) to the landed bf16 V tile in shared
// memory, rounding each sum to bf16 as a bf16 tensor addition does. Rows past the tensor are left
// as they are. Thread t of the NT takes 16-byte unit t % (hd / 8) of every (8 NT / hd)-th row;
// its global loads are issued BATCH rows at a time, all before the adds of those rows.
template <int HD, int NT, int BATCH>
__device__ __forceinline__ void add_aux_tile(uint8_t* tile, const __nv_bfloat16* aux, int row0, int hs,
                                             int heads_slot, int64_t slots, int at) {
    constexpr int kUnits = HD / 8;
    constexpr int kRowsPerPass = NT / kUnits;
    constexpr int kPasses = kBlockN / kRowsPerPass;
    static_assert(kPasses % BATCH == 0, "batches of passes");
    const int unit = at % kUnits;
#pragma unroll 1
    for (int k0 = 0; k0 < kPasses; k0 += BATCH) {
        uint4 a[BATCH];
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
            const int r = at / kUnits + (k0 + k) * kRowsPerPass;
            const int64_t slot = static_cast<int64_t>(row0) + r;
            a[k] = slot < slots ? __ldg(reinterpret_cast<const uint4*>(
                                      aux + (slot * heads_slot + hs) * HD + unit * 8))
                                : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
            const int r = at / kUnits + (k0 + k) * kRowsPerPass;
            if (static_cast<int64_t>(row0) + r >= slots) break;
            // unit u of row r in the 128-byte-swizzled [128 rows][64 bf16] chunks of the tile
            uint4* addr = reinterpret_cast<uint4*>(tile + (unit >> 3) * (kBlockN * 128) + r * 128 +
                                                   (((unit & 7) ^ (r & 7)) << 4));
            const uint4 v = *addr;
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w}, aw[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)  // bf16 + bf16 is exact in float32; one rounding to bf16
                o[e] = pack_bf16x2(__uint_as_float(vw[e] << 16) + __uint_as_float(aw[e] << 16),
                                   __uint_as_float(vw[e] & 0xFFFF0000u) + __uint_as_float(aw[e] & 0xFFFF0000u));
            *addr = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// Band work item (see kernels.cuh), decoded.
struct BandItem {
    int q0, n_qt, hp, head, doc_end, doc_start;
};

__device__ __forceinline__ BandItem decode_band(int4 w) {
    BandItem it;
    it.q0 = w.x;
    it.head = w.y >> 16;
    it.hp = (w.y >> 15) & 1;
    it.n_qt = w.y & 0x7FFF;
    it.doc_end = w.z;
    it.doc_start = w.w;
    return it;
}

// Index of this CTA's k-th item: the longest-first list is dealt out in rows of gridDim.x items,
// left to right on even rows and right to left on odd rows. -1 past the end of the list, -2 when
// the last (partial) row has no item for this CTA.
__device__ __forceinline__ int band_item_index(int k, int n_items) {
    const int64_t base = static_cast<int64_t>(k) * gridDim.x;
    if (base >= n_items) return -1;
    const int64_t idx = base + ((k & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x);
    return idx < n_items ? static_cast<int>(idx) : -2;
}

// Walks this CTA's items in order, keeping the next one's descriptor in flight. With a head group
// G > 1 (H heads per block of the list, the scheduler's layout) it walks only the items of each
// group's first head, slot * H + g * G, as one list of n / G items, so that those items, not all
// of them, are dealt evenly to the CTAs.
struct ItemWalk {
    const int4* items;
    int n_items, k, idx, nidx;
    int grp = 1, heads = 1;
    int4 cur, nxt;
    __device__ __forceinline__ int real(int i) const {
        if (grp == 1) return i;
        const int hkv = heads / grp;
        return (i / hkv) * heads + (i % hkv) * grp;
    }
    __device__ __forceinline__ void start(const int4* it, int n, int g = 1, int h = 1) {
        items = it;
        grp = g;
        heads = h;
        n_items = n / g;
        k = 0;
        idx = band_item_index(0, n_items);
        cur = idx >= 0 ? __ldg(items + real(idx)) : make_int4(0, 0, 0, 0);
        prefetch();
    }
    __device__ __forceinline__ void prefetch() {
        nidx = idx == -1 ? -1 : band_item_index(k + 1, n_items);
        nxt = nidx >= 0 ? __ldg(items + real(nidx)) : make_int4(0, 0, 0, 0);
    }
    __device__ __forceinline__ bool done() const { return idx == -1; }
    __device__ __forceinline__ bool has() const { return idx >= 0; }
    __device__ __forceinline__ void advance() {
        idx = nidx;
        cur = nxt;
        ++k;
        prefetch();
    }
};

}  // namespace pha
