// rope.cu -- rotary tables and the in-place rotary kernel (standard and paired / staggered).
//
// Method: "modded-nanogpt Paired Head Attention record" page, sections "zero-copy RoPE and delayed
// reshape" (one elementwise pass y = cos * x + sin * x_flip, x_flip swapping the two members of
// each adjacent pair), "staggered rotary" and "4. interleave index in the Triton kernel" (odd
// heads read the second half of the 2*head_dim-wide paired row), "2. building the paired rotary
// table" (row p packs the angles of positions 2p and 2p+1). Frequencies: "Training an LLM from
// scratch (part 2)", section "2. RoPE".
//
// The rotation is HBM-bound: one warp per token moves the token's q and k rows in 16-byte chunks
// (coalesced 512-byte warp accesses, several chunks in flight per lane); the table row of a token
// is shared by all of its heads and is served from L1/L2. Every output is the correctly rounded (nearest even) value of the rotation
// with the tables' float32 cosines and sines:
//   bf16: y = fma(c, a, s*b) in float32 differs from the exact value by at most
//         ulp(y)/2 + ulp(s*b)/2; when y lies farther than that from the nearest bf16 rounding
//         midpoint, rounding y gives the same bf16 as rounding the exact value. The rare rest is
//         recomputed in float64, where bf16 x float32 products are exact, and rounded from there.
//   f32:  always float64 (exact products, one rounding), then rounded to float32.
//
// Factored tables (pha_rope_factored and its norm / backward forms): instead of a float32 row per
// position, two small float64 tables of (cos, sin) pairs, which stay in L1 / L2, so that the
// rotation reads only q and k from HBM. Table row p = kRopeLoRows * r + l splits each angle into
// a coarse part (row kRopeLoRows * r; for a paired row, its even position) and a fine part (row
// l, either half), and cos(a + b) = cos a cos b - sin a sin b, sin(a + b) = sin a cos b +
// cos a sin b in float64, rounded once to float32, give the value that the stored table holds,
// or its neighbour next to a float32 rounding midpoint, or (values very close to zero) a value
// off by the two forms' float64 angle difference (~5e-11 at 1.4e5 rad). This path rotates with
// compensated float32 arithmetic and a cheaper exactness test (rot_chunk_bf16_comp); its bf16
// results are correctly rounded too.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.cuh"

namespace pha {

__global__ void rope_tables_kernel(float* __restrict__ cos_tab, float* __restrict__ sin_tab,
                                   int rows, int head_dim, int paired, double base) {
    const int width = paired ? 2 * head_dim : head_dim;
    const int64_t n = static_cast<int64_t>(rows) * width;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t p = idx / width;
        const int col = static_cast<int>(idx % width);
        const int half = col / head_dim;  // paired: 0 -> position 2p, 1 -> position 2p+1
        const int j = col % head_dim;
        const double pos = paired ? 2.0 * static_cast<double>(p) + half : static_cast<double>(p);
        const double freq = pow(base, -2.0 * static_cast<double>(j / 2) / head_dim);
        double s, c;
        sincos(pos * freq, &s, &c);
        cos_tab[idx] = static_cast<float>(c);
        sin_tab[idx] = static_cast<float>(s);
    }
}

// Factored tables, (cos, sin) pairs of float64: first kRopeLoRows fine rows of A entries
// (A = head_dim / 2, or head_dim when paired: entry a = half * head_dim / 2 + i holds the angle
// of position l (standard) or 2l + half (paired) at frequency i), then ceil(rows / kRopeLoRows)
// coarse rows of head_dim / 2 entries (row r, entry i: position kRopeLoRows * r, or twice that
// when paired, at frequency i). Frequencies and float64 angles as in rope_tables_kernel.
__global__ void rope_factor_tables_kernel(double2* __restrict__ fac, int rows, int head_dim,
                                          int paired, double base) {
    const int half_hd = head_dim / 2;
    const int a_width = paired ? head_dim : half_hd;
    const int64_t n_lo = static_cast<int64_t>(kRopeLoRows) * a_width;
    const int64_t n = n_lo + static_cast<int64_t>(rope_hi_rows(rows)) * half_hd;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        double pos;
        int i;
        if (idx < n_lo) {
            const int l = static_cast<int>(idx / a_width);
            const int a = static_cast<int>(idx % a_width);
            const int half = a / half_hd;
            i = a % half_hd;
            pos = paired ? 2.0 * l + half : static_cast<double>(l);
        } else {
            const int64_t r = (idx - n_lo) / half_hd;
            i = static_cast<int>((idx - n_lo) % half_hd);
            pos = static_cast<double>(r) * kRopeLoRows * (paired ? 2.0 : 1.0);
        }
        const double freq = pow(base, -2.0 * static_cast<double>(i) / head_dim);
        double sv, cv;
        sincos(pos * freq, &sv, &cv);
        fac[idx] = make_double2(cv, sv);
    }
}

// Nearest bfloat16 (ties to even) of a double, as its 16-bit pattern; one rounding step.
__device__ __noinline__ uint32_t bf16_bits_rne(double y) {
    const uint64_t b = static_cast<uint64_t>(__double_as_longlong(y));
    const uint32_t sign = static_cast<uint32_t>(b >> 48) & 0x8000u;
    const int e = static_cast<int>((b >> 52) & 0x7FF);
    const uint64_t man = b & 0xFFFFFFFFFFFFFull;
    if (e == 0x7FF) return sign | 0x7F80u | (man ? 0x40u : 0u);  // inf, nan
    const int eb = e - 1023 + 127;                                // bf16 biased exponent
    if (eb >= 255) return sign | 0x7F80u;                        // overflow
    if (eb <= 0)  // bf16 subnormal range: count units of 2^-133 (rint rounds half to even;
                  // 128 units carry into the smallest normal's bit pattern)
        return sign | static_cast<uint32_t>(rint(fabs(y) * 0x1p133));
    const uint32_t keep = static_cast<uint32_t>(man >> 45);      // 7 mantissa bits kept
    const uint64_t rem = man & ((1ull << 45) - 1), half = 1ull << 44;
    uint32_t bits = (static_cast<uint32_t>(eb) << 7) | keep;
    if (rem > half || (rem == half && (keep & 1u))) ++bits;      // may carry into the exponent
    return sign | bits;
}

// float32 ulps from y to the bf16 rounding midpoint of y's binade (bit pattern ...8000), as a
// float: the low 16 bits OR-ed into 2^23 give 2^23 + low16 exactly.
__device__ __forceinline__ float ulps_to_midpoint(float y) {
    return __uint_as_float((__float_as_uint(y) & 0xFFFFu) | 0x4B000000u) - 8421376.0f;  // 2^23 + 2^15
}

// y = fma(c, a, t) with t = rounded s*b is within ulp(y)/2 + |t| 2^-24 < (1/2 + |t|/|y|) ulp(y)
// of the exact c*a + s*b; when y lies more than that (plus 1.5 ulp of margin) from the bf16
// rounding midpoint, rounding y gives the bf16 of the exact value.
__device__ __forceinline__ bool rounds_like_exact(float y, float t) {
    return fabsf(t) <= fabsf(y) * (fabsf(ulps_to_midpoint(y)) - 2.0f);
}

// One rotated pair (x0, x1) with the pair's table values c, s:
//   y0 = c x0 - s x1,  y1 = c x1 + s x0   (packed f32x2 arithmetic)
// as two bf16 of the exact values (16-bit patterns, y0 in the low half).
__device__ __forceinline__ uint32_t rot_pair_bf16(float x0, float x1, float c, float s) {
    const uint64_t t2 = mul_f32x2(f32x2(-s, s), f32x2(x1, x0));
    const uint64_t y2 = fma_f32x2(f32x2(c, c), f32x2(x0, x1), t2);
    float y0, y1, t0, t1;
    f32x2_split(y2, y0, y1);
    f32x2_split(t2, t0, t1);
    if (rounds_like_exact(y0, t0) && rounds_like_exact(y1, t1)) return pack_bf16x2(y0, y1);
    // rare: recompute in float64, where bf16 x float32 products are exact
    const double e0 = fma(static_cast<double>(c), static_cast<double>(x0),
                          -static_cast<double>(s) * static_cast<double>(x1));
    const double e1 = fma(static_cast<double>(c), static_cast<double>(x1),
                          static_cast<double>(s) * static_cast<double>(x0));
    return bf16_bits_rne(e0) | (bf16_bits_rne(e1) << 16);
}

// Correctly rounded rotation from compensated float32 arithmetic (the factored-table path): the
// products s*x are split exactly into t = fl(s*x) and e = s*x - t (one fma each), and
// y = fl(fl(c*x' + t) + e) is within one float32 ulp of the exact value even under cancellation
// (where fl(c*x' + t) is exact). When y lies more than eight float32 ulps from a bf16 rounding
// midpoint, rounding y gives the bf16 of the exact value; otherwise the pair is recomputed in
// float64 as in rot_pair_bf16 (measured on the paired workload: the test and its branch cost
// about 7 us of the 78 us factored RoPE; testing a whole chunk at once, or rounding y +- 8 ulps
// twice and comparing, measured slower).

// The rare pair near a bf16 midpoint: float64 (exact products), one rounding. Out of line, so
// that the fast path of the rotation loop stays small.
__device__ __noinline__ uint32_t rot_pair_bf16_f64(float x0, float x1, float c, float s) {
    const double e0 = fma(static_cast<double>(c), static_cast<double>(x0),
                          -static_cast<double>(s) * static_cast<double>(x1));
    const double e1 = fma(static_cast<double>(c), static_cast<double>(x1),
                          static_cast<double>(s) * static_cast<double>(x0));
    return bf16_bits_rne(e0) | (bf16_bits_rne(e1) << 16);
}

// More than eight float32 ulps from the bf16 rounding midpoint of y's binade (the low 16 bits
// outside 0x8000 +- 8): y and anything within one ulp of it round to the same bf16. Adding 0x8008
// maps that window of the low 16 bits onto 0x0000..0x000F.
__device__ __forceinline__ bool far_from_bf16_midpoint(float y) {
    return ((__float_as_uint(y) + 0x8008u) & 0xFFF0u) != 0u;
}

__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Four pairs (one 16-byte bf16 chunk) in two groups of two pairs a, b, each packed by member:
// X0 = (x0 of a, x0 of b), X1 = (x1 of a, x1 of b), C and S their table values. Then
//   y0 = c x0 - s x1:  T = fl(-S X1),  E = S X1 + T exactly (the rounding error of S X1),
//                      Y0 = fl(fl(C X0 + T) - E)
//   y1 = c x1 + s x0:  T' = fl(S X0), E' = -S X0 + T' exactly,  Y1 = fl(fl(C X1 + T') - E')
// (four packed operations a pair). Each pair is tested on its own; a pair near a bf16 rounding
// midpoint takes the float64 path.
__device__ __forceinline__ uint4 rot_chunk_bf16_comp(const float (&x)[8], const float (&c)[8],
                                                     const float (&s)[8]) {
    uint32_t o[4];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const int a = 2 * g, b = 2 * g + 1;  // pairs; pair p holds x[2p], x[2p + 1], angle c[2p]
        const uint64_t x0 = f32x2(x[2 * a], x[2 * b]), x1 = f32x2(x[2 * a + 1], x[2 * b + 1]);
        const uint64_t cc = f32x2(c[2 * a], c[2 * b]), ss = f32x2(s[2 * a], s[2 * b]);
        const uint64_t sn = f32x2(-s[2 * a], -s[2 * b]);
        const uint64_t t0 = mul_f32x2(sn, x1);
        const uint64_t y0 = sub_f32x2(fma_f32x2(cc, x0, t0), fma_f32x2(ss, x1, t0));
        const uint64_t t1 = mul_f32x2(ss, x0);
        const uint64_t y1 = sub_f32x2(fma_f32x2(cc, x1, t1), fma_f32x2(sn, x0, t1));
        float y0a, y0b, y1a, y1b;
        f32x2_split(y0, y0a, y0b);
        f32x2_split(y1, y1a, y1b);
        o[a] = (far_from_bf16_midpoint(y0a) && far_from_bf16_midpoint(y1a))
                   ? pack_bf16x2(y0a, y1a)
                   : rot_pair_bf16_f64(x[2 * a], x[2 * a + 1], c[2 * a], s[2 * a]);
        o[b] = (far_from_bf16_midpoint(y0b) && far_from_bf16_midpoint(y1b))
                   ? pack_bf16x2(y0b, y1b)
                   : rot_pair_bf16_f64(x[2 * b], x[2 * b + 1], c[2 * b], s[2 * b]);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}


// 16-byte chunks of a row: 8 bf16 (4 pairs) or 4 f32 (2 pairs). to_floats gives the exact values;
// rotate_f rotates E float values with the chunk's table values c[j], s[j] (j = element within
// the chunk) and rounds once to the buffer type; pack_f only rounds.
template <typename T>
struct Chunk16;

template <>
struct Chunk16<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ static void to_floats(uint4 a, float (&x)[E]) {
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[2 * e] = __uint_as_float(w[e] << 16);
            x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
    template <bool COMP = false>
    __device__ static uint4 rotate_f(const float (&x)[E], const float (&c)[E], const float (&s)[E]) {
        if (COMP) return rot_chunk_bf16_comp(x, c, s);
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)  // both members of a pair share one angle: c[2e] == c[2e+1]
            o[e] = rot_pair_bf16(x[2 * e], x[2 * e + 1], c[2 * e], s[2 * e]);
        return make_uint4(o[0], o[1], o[2], o[3]);
    }
    __device__ static uint4 pack_f(const float (&x)[E]) {
        return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                          pack_bf16x2(x[6], x[7]));
    }
    template <bool COMP = false>
    __device__ static uint4 rotate(uint4 a, const float (&c)[E], const float (&s)[E]) {
        if (COMP) {
            float x[E];
            to_floats(a, x);
            return rot_chunk_bf16_comp(x, c, s);
        }
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xFFFF0000u);
            o[e] = rot_pair_bf16(x0, x1, c[2 * e], s[2 * e]);
        }
        return make_uint4(o[0], o[1], o[2], o[3]);
    }
};

template <>
struct Chunk16<float> {
    static constexpr int E = 4;
    __device__ static void to_floats(uint4 a, float (&x)[E]) {
        x[0] = __uint_as_float(a.x);
        x[1] = __uint_as_float(a.y);
        x[2] = __uint_as_float(a.z);
        x[3] = __uint_as_float(a.w);
    }
    template <bool COMP = false>  // float32 results: always float64, correctly rounded
    __device__ static uint4 rotate_f(const float (&x)[E], const float (&c)[E], const float (&s)[E]) {
        float y[E];
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            // products of float32 values are exact in double: one rounding in the fma, one to f32
            y[e] = __double2float_rn(fma(static_cast<double>(c[e]), static_cast<double>(x[e]),
                                         -static_cast<double>(s[e]) * static_cast<double>(x[e + 1])));
            y[e + 1] = __double2float_rn(fma(static_cast<double>(c[e + 1]), static_cast<double>(x[e + 1]),
                                             static_cast<double>(s[e + 1]) * static_cast<double>(x[e])));
        }
        return make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                          __float_as_uint(y[3]));
    }
    __device__ static uint4 pack_f(const float (&x)[E]) {
        return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                          __float_as_uint(x[3]));
    }
    template <bool COMP = false>
    __device__ static uint4 rotate(uint4 a, const float (&c)[E], const float (&s)[E]) {
        float x[E];
        to_floats(a, x);
        return rotate_f(x, c, s);
    }
};

// One warp per token. The token's q row (n_heads * head_dim contiguous elements) followed by its
// k row is cut into 16-byte chunks; lane l takes chunks l, l + 32, ... in batches of kRopeBatch,
// so every load instruction of the warp reads 512 contiguous bytes and each lane keeps
// kRopeBatch x 16 bytes of HBM reads in flight (six for the rotation: a whole token of 12 q + k
// heads of 64, or 6 of 128, in one batch; four with the norm, whose extra pass needs the
// registers); the first batch is issued before the table loads. All heads of the token share its
// table row, which is read from HBM once and then served from L1.
template <bool NORM>
constexpr int kRopeBatch = NORM ? 4 : 6;

// NORM: each head row is first RMS-normalised over head_dim in float32 ("Training an LLM from
// scratch (part 2)", section "1. RMSNorm": x / sqrt(mean(x^2) + eps) * weight; weight NULL = 1),
// then rotated; one rounding at the end. The chunks of one head row sit on cph consecutive lanes
// (cph divides 32), so the row's sum of squares is a shuffle reduction over those lanes. Tokens
// whose position lies outside the table are normalised but not rotated.
// Resident 256-thread blocks per SM: four (64 registers) for the plain bf16 rotation with stored
// tables; three (80 registers) for the others, whose factor loads, float64 arithmetic or norm
// need the registers (measured: the factored bf16 rotation at four blocks spills and runs ~12 %
// slower).
template <typename T, bool NORM, bool FACT>
constexpr int rope_min_blocks() { return (sizeof(T) == 2 && !NORM && !FACT) ? 4 : 3; }

// The cosines and sines of table columns [col, col + E) of one row (E even, inside one half of a
// paired row; both members of a pair get the pair's value). Stored tables: crow / srow point at
// the row. Factored (FACT): lo_row / hi_row point at the row's fine and coarse factor rows.
template <int E, bool FACT, bool NEG>
__device__ __forceinline__ void table_cs(const float* crow, const float* srow,
                                         const double2* lo_row, const double2* hi_row, int col,
                                         int head_dim, float (&c)[E], float (&s)[E]) {
    if (!FACT) {
#pragma unroll
        for (int e = 0; e < E; e += 4) {
            const float4 cv = __ldg(reinterpret_cast<const float4*>(crow + col + e));
            const float4 sv = __ldg(reinterpret_cast<const float4*>(srow + col + e));
            c[e] = cv.x; c[e + 1] = cv.y; c[e + 2] = cv.z; c[e + 3] = cv.w;
            s[e] = NEG ? -sv.x : sv.x; s[e + 1] = NEG ? -sv.y : sv.y;
            s[e + 2] = NEG ? -sv.z : sv.z; s[e + 3] = NEG ? -sv.w : sv.w;
        }
    } else {
        const int upper = col >= head_dim;            // paired rows: second half (position 2p+1)
        const int i0 = ((col - (upper ? head_dim : 0)) >> 1);  // frequency of the first pair
        const int a0 = (upper ? head_dim >> 1 : 0) + i0;
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const double2 f = __ldg(lo_row + a0 + e / 2);  // fine angle b
            const double2 g = __ldg(hi_row + i0 + e / 2);  // coarse angle a
            const float cv = __double2float_rn(fma(g.x, f.x, -(g.y * f.y)));
            const float sv = __double2float_rn(fma(g.y, f.x, g.x * f.y));
            c[e] = cv;
            c[e + 1] = cv;
            s[e] = NEG ? -sv : sv;
            s[e + 1] = NEG ? -sv : sv;
        }
    }
}

// NEG: the backward of RoPE (the gradient with respect to the input is the transposed rotation,
// i.e. the rotation by -angle): the sines enter negated, which is exact.
// FACT: factored tables (fac; cos_tab / sin_tab unused, tab_rows = the rows they stand for), and
// the bf16 rotation of rot_chunk_bf16_comp.
template <typename T, bool NORM, bool NEG = false, bool FACT = false>
__global__ void __launch_bounds__(256, (rope_min_blocks<T, NORM, FACT>())) rope_kernel(T* __restrict__ q, T* __restrict__ k,
                                                   const float* __restrict__ cos_tab,
                                                   const float* __restrict__ sin_tab,
                                                   int tab_rows, int tab_width,
                                                   const int32_t* __restrict__ positions,
                                                   int64_t total_tokens, int n_heads,
                                                   int n_kv_heads, int head_dim, int paired,
                                                   int stagger_offset,
                                                   const float* __restrict__ q_weight,
                                                   const float* __restrict__ k_weight, float eps,
                                                   const double2* __restrict__ fac) {
    constexpr int E = Chunk16<T>::E;
    const int cph = head_dim / E;                  // chunks per head row
    // NORM: 1 / head_dim is exact (head_dim is a power of two here), so ss * inv_hd + eps rounds
    // once, as ss / head_dim + eps does
    const float inv_hd = 1.0f / static_cast<float>(head_dim);
    const int q_chunks = n_heads * cph;
    const int n_chunks = q_chunks + n_kv_heads * cph;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    // the position of the warp's next token is loaded one token ahead, so that the table loads
    // of a token go out with its q / k loads instead of after a dependent position load
    int pos_next = warp0 < total_tokens ? __ldg(positions + warp0) : 0;
    for (int64_t t = warp0; t < total_tokens; t += n_warps) {
        const int pos = pos_next;
        if (t + n_warps < total_tokens) pos_next = __ldg(positions + t + n_warps);
        uint4* qrow = reinterpret_cast<uint4*>(q + t * n_heads * static_cast<int64_t>(head_dim));
        uint4* krow = reinterpret_cast<uint4*>(k + t * n_kv_heads * static_cast<int64_t>(head_dim));
        // the first batch of the token's q / k chunks goes out before the table loads
        uint4 raw[kRopeBatch<NORM>];
#pragma unroll
        for (int j = 0; j < kRopeBatch<NORM>; ++j) {
            const int i = 32 * j + lane;
            if (i < n_chunks) raw[j] = i < q_chunks ? qrow[i] : krow[i - q_chunks];
        }
        const bool in_range = pos >= 0 && pos < tab_rows;
        const int prow = in_range ? pos : 0;
        const float* crow = FACT ? nullptr : cos_tab + static_cast<int64_t>(prow) * tab_width;
        const float* srow = FACT ? nullptr : sin_tab + static_cast<int64_t>(prow) * tab_width;
        const double2* lo_row =
            FACT ? fac + (prow % kRopeLoRows) * (paired ? head_dim : head_dim >> 1) : nullptr;
        const double2* hi_row =
            FACT ? fac + kRopeLoRows * (paired ? head_dim : head_dim >> 1) +
                       static_cast<int64_t>(prow / kRopeLoRows) * (head_dim >> 1)
                 : nullptr;
        // When cph divides 32 (and, paired, 32/cph is even so the head parity is fixed too), every
        // chunk of this lane sits at the same table columns: load them once per token.
        const bool uniform_cols = (32 % cph == 0) && (!paired || ((32 / cph) % 2 == 0));
        float cu[E], su[E];
        if (uniform_cols && in_range) {
            const int h0 = (lane % n_chunks) / cph;  // any chunk of this lane gives the columns
            const int col0 = ((paired && (h0 & 1)) ? stagger_offset : 0) + (lane % cph) * E;
            table_cs<E, FACT, NEG>(crow, srow, lo_row, hi_row, col0, head_dim, cu, su);
        }
        // NORM: a lane's chunks always sit at element offset (lane % cph) * E of their head row
        // (cph divides 32), so its q and k weights are the same for every chunk and token.
        float wq[E], wk[E];
        if (NORM) {
            const int off = (lane % cph) * E;
#pragma unroll
            for (int e = 0; e < E; e += 4) {
                const float4 a = q_weight ? __ldg(reinterpret_cast<const float4*>(q_weight + off + e))
                                          : make_float4(1.f, 1.f, 1.f, 1.f);
                const float4 b = k_weight ? __ldg(reinterpret_cast<const float4*>(k_weight + off + e))
                                          : make_float4(1.f, 1.f, 1.f, 1.f);
                wq[e] = a.x; wq[e + 1] = a.y; wq[e + 2] = a.z; wq[e + 3] = a.w;
                wk[e] = b.x; wk[e + 1] = b.y; wk[e + 2] = b.z; wk[e + 3] = b.w;
            }
        }
        for (int base = 0; base < n_chunks; base += 32 * kRopeBatch<NORM>) {
            if (base > 0) {
#pragma unroll
                for (int j = 0; j < kRopeBatch<NORM>; ++j) {
                    const int i = base + 32 * j + lane;
                    if (i < n_chunks) raw[j] = i < q_chunks ? qrow[i] : krow[i - q_chunks];
                }
            }
            float inv[kRopeBatch<NORM>];
            if (NORM) {
                // 1 / rms of the head row of each chunk (all lanes take part in the shuffles)
#pragma unroll
                for (int j = 0; j < kRopeBatch<NORM>; ++j) {
                    float ss = 0.f;
                    if (base + 32 * j + lane < n_chunks) {
                        float x[E];
                        Chunk16<T>::to_floats(raw[j], x);
#pragma unroll
                        for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)  // offsets cph / 2 .. 1 (cph divides 32)
                        if (o < cph) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                    inv[j] = rsqrtf(fmaf(ss, inv_hd, eps));
                }
            } else if (!in_range) {
                continue;  // positions outside the table: leave the token unchanged
            }
#pragma unroll
            for (int j = 0; j < kRopeBatch<NORM>; ++j) {
                const int i = base + 32 * j + lane;
                if (i >= n_chunks) break;
                float x[E];
                if (NORM) {
                    Chunk16<T>::to_floats(raw[j], x);
                    const bool is_q = i < q_chunks;
#pragma unroll
                    for (int e = 0; e < E; ++e) x[e] = x[e] * inv[j] * (is_q ? wq[e] : wk[e]);
                    if (!in_range) {
                        const uint4 y = Chunk16<T>::pack_f(x);
                        if (i < q_chunks) qrow[i] = y; else krow[i - q_chunks] = y;
                        continue;
                    }
                }
                float c[E], s[E];
                if (uniform_cols) {
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        c[e] = cu[e];
                        s[e] = su[e];
                    }
                } else {
                    const int ih = i < q_chunks ? i : i - q_chunks;  // chunk index within q or k row
                    const int h = ih / cph;
                    const int col = ((paired && (h & 1)) ? stagger_offset : 0) + (ih - h * cph) * E;
                    table_cs<E, FACT, NEG>(crow, srow, lo_row, hi_row, col, head_dim, c, s);
                }
                // y = cos * x + sign * sin * x_flip, x_flip swapping each adjacent pair; the sign
                // is -1 on the even member and +1 on the odd member (a rotation by +angle).
                const uint4 y = NORM ? Chunk16<T>::template rotate_f<FACT>(x, c, s)
                                     : Chunk16<T>::template rotate<FACT>(raw[j], c, s);
                if (i < q_chunks) qrow[i] = y; else krow[i - q_chunks] = y;
            }
        }
    }
}

// Factored-table rotation with the tokens' q and k rows staged in shared memory: each warp keeps a
// private ring of R slots, and each lane copies its own 16-byte chunks of the unit R - 1 steps
// ahead into it with cp.async, so R - 1 units of HBM reads per warp are in flight without holding
// registers; before a unit is rotated the lane waits for its own copy group (a hardware wait) and
// reads back only the chunks it copied (no barrier). A unit is a token's q and k chunks, or, when
// a token is too wide for the ring, one of its n_seg segments of seg chunks (seg a multiple of 32,
// so that a lane's chunks keep their table columns and a head row stays inside one 32-chunk
// round). Used when every chunk of a lane sits at the same table columns (as in rope_kernel's
// uniform case).
// NORM: the QK RMS-norm of each head row first, as in rope_kernel (the row's chunks sit on cph
// consecutive lanes of one 32-chunk round, whose lanes all take part in the shuffles).
template <typename T, bool NEG, bool NORM, bool SEG, int R, int MINB>
__global__ void __launch_bounds__(256, MINB)
    rope_ring_kernel(T* __restrict__ q, T* __restrict__ k, const int32_t* __restrict__ positions,
                     int64_t total_tokens, int n_heads, int n_kv_heads, int head_dim, int paired,
                     int stagger_offset, int tab_rows, const double2* __restrict__ fac,
                     const float* __restrict__ q_weight, const float* __restrict__ k_weight,
                     float eps, int n_seg, int seg) {
    extern __shared__ __align__(16) uint8_t ring_smem[];
    constexpr int E = Chunk16<T>::E;
    const int cph = head_dim / E;
    const int q_chunks = n_heads * cph;
    const int n_chunks = q_chunks + n_kv_heads * cph;
    const int lane = threadIdx.x & 31;
    if (!SEG) n_seg = 1, seg = n_chunks;  // one unit a token: the index arithmetic folds away
    const int slot_bytes = seg * 16;
    const int64_t n_units = total_tokens * n_seg;
    uint8_t* ring = ring_smem + (threadIdx.x >> 5) * R * slot_bytes;
    const int64_t warp0 = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int h0 = (lane % n_chunks) / cph;  // any chunk of this lane gives the columns
    const int col0 = ((paired && (h0 & 1)) ? stagger_offset : 0) + (lane % cph) * E;
    const int a_width = paired ? head_dim : head_dim >> 1;
    float wq[E], wk[E];  // NORM: this lane's weights (the same columns for every chunk)
    if (NORM) {
        const int off = (lane % cph) * E;
#pragma unroll
        for (int e = 0; e < E; e += 4) {
            const float4 a = q_weight ? __ldg(reinterpret_cast<const float4*>(q_weight + off + e))
                                      : make_float4(1.f, 1.f, 1.f, 1.f);
            const float4 b = k_weight ? __ldg(reinterpret_cast<const float4*>(k_weight + off + e))
                                      : make_float4(1.f, 1.f, 1.f, 1.f);
            wq[e] = a.x; wq[e + 1] = a.y; wq[e + 2] = a.z; wq[e + 3] = a.w;
            wk[e] = b.x; wk[e + 1] = b.y; wk[e + 2] = b.z; wk[e + 3] = b.w;
        }
    }
    // NORM: 1 / head_dim is exact (head_dim is a power of two here), so ss * inv_hd + eps rounds
    // once, as ss / head_dim + eps does
    const float inv_hd = 1.0f / static_cast<float>(head_dim);
    // unit u: token u / n_seg, chunks [c0, c1) with c0 = (u % n_seg) * seg
    auto token_of = [&](int64_t u) { return SEG ? u / n_seg : u; };
    auto issue = [&](int64_t u, int slot) {
        const int64_t t = token_of(u);
        const int c0 = SEG ? static_cast<int>(u - t * n_seg) * seg : 0;
        const int c1 = SEG ? min(c0 + seg, n_chunks) : n_chunks;
        const uint4* qrow = reinterpret_cast<const uint4*>(q + t * n_heads * static_cast<int64_t>(head_dim));
        const uint4* krow = reinterpret_cast<const uint4*>(k + t * n_kv_heads * static_cast<int64_t>(head_dim));
        uint8_t* dst = ring + slot * slot_bytes;
        for (int i = c0 + lane; i < c1; i += 32)
            cp_async_16(dst + (i - c0) * 16, i < q_chunks ? qrow + i : krow + (i - q_chunks));
    };
#pragma unroll
    for (int r = 0; r < R - 1; ++r) {
        const int64_t u = warp0 + r * n_warps;
        if (u < n_units) issue(u, r);
        cp_async_commit();
    }
    int pos_next = warp0 < n_units ? __ldg(positions + token_of(warp0)) : 0;
    int slot = 0;
    for (int64_t u = warp0; u < n_units; u += n_warps) {
        const int64_t ua = u + (R - 1) * n_warps;
        if (ua < n_units) issue(ua, (slot + R - 1) % R);  // the slot read last step
        cp_async_commit();
        const int64_t t = token_of(u);
        const int c0 = SEG ? static_cast<int>(u - t * n_seg) * seg : 0;
        const int c1 = SEG ? min(c0 + seg, n_chunks) : n_chunks;
        const int pos = pos_next;
        if (u + n_warps < n_units) pos_next = __ldg(positions + token_of(u + n_warps));
        const bool in_range = pos >= 0 && pos < tab_rows;
        float cu[E], su[E];
        if (in_range) {
            const double2* lo_row = fac + (pos % kRopeLoRows) * a_width;
            const double2* hi_row =
                fac + kRopeLoRows * a_width + static_cast<int64_t>(pos / kRopeLoRows) * (head_dim >> 1);
            table_cs<E, true, NEG>(nullptr, nullptr, lo_row, hi_row, col0, head_dim, cu, su);
        }
        cp_async_wait<R - 1>();  // this lane's chunks of unit u have landed
        uint4* qrow = reinterpret_cast<uint4*>(q + t * n_heads * static_cast<int64_t>(head_dim));
        uint4* krow = reinterpret_cast<uint4*>(k + t * n_kv_heads * static_cast<int64_t>(head_dim));
        const uint8_t* src = ring + slot * slot_bytes;
        if (NORM) {  // normalised, then rotated when the position is inside the table
#pragma unroll 2  // two rounds in flight (115.9 -> 114.3 us on the paired workload)
            for (int base = c0; base < c1; base += 32) {
                const int i = base + lane;
                const bool have = i < c1;
                float x[E];
                Chunk16<T>::to_floats(have ? *reinterpret_cast<const uint4*>(src + (i - c0) * 16)
                                           : make_uint4(0u, 0u, 0u, 0u), x);
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)  // offsets cph / 2 .. 1 (cph divides 32)
                    if (o < cph) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float inv = rsqrtf(fmaf(ss, inv_hd, eps));
                if (!have) continue;
                const bool is_q = i < q_chunks;
#pragma unroll
                for (int e = 0; e < E; ++e) x[e] = x[e] * inv * (is_q ? wq[e] : wk[e]);
                const uint4 y = in_range ? Chunk16<T>::template rotate_f<true>(x, cu, su)
                                         : Chunk16<T>::pack_f(x);
                if (is_q) qrow[i] = y; else krow[i - q_chunks] = y;
            }
        } else if (in_range) {  // a token outside the table is left unchanged
            // two chunks in flight per lane (three blocks per SM leave the registers for it:
            // 78.7 -> 76.6 us on the paired workload; by 3 or 6 it spills)
#pragma unroll 2
            for (int i = c0 + lane; i < c1; i += 32) {
                const uint4 y = Chunk16<T>::template rotate<true>(
                    *reinterpret_cast<const uint4*>(src + (i - c0) * 16), cu, su);
                if (i < q_chunks) qrow[i] = y; else krow[i - q_chunks] = y;
            }
        }
        slot = slot + 1 == R ? 0 : slot + 1;
    }
    cp_async_wait<0>();
}

cudaError_t launch_rope_tables(float* cos_tab, float* sin_tab, int rows, int head_dim, int paired,
                               double base, cudaStream_t stream) {
    const int64_t n = static_cast<int64_t>(rows) * (paired ? 2 : 1) * head_dim;
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (n + threads - 1) / threads;
    const int grid = static_cast<int>(blocks < 148 * 64 ? blocks : 148 * 64);
    rope_tables_kernel<<<grid, threads, 0, stream>>>(cos_tab, sin_tab, rows, head_dim, paired,
                                                     base);
    return cudaGetLastError();
}

cudaError_t launch_rope_factor_tables(double2* fac, int rows, int head_dim, int paired, double base,
                                      cudaStream_t stream) {
    const int64_t n = static_cast<int64_t>(kRopeLoRows) * (paired ? head_dim : head_dim / 2) +
                      static_cast<int64_t>(rope_hi_rows(rows)) * (head_dim / 2);
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (n + threads - 1) / threads;
    const int grid = static_cast<int>(blocks < 148 * 64 ? blocks : 148 * 64);
    rope_factor_tables_kernel<<<grid, threads, 0, stream>>>(fac, rows, head_dim, paired, base);
    return cudaGetLastError();
}

template <bool NORM, bool NEG = false, bool FACT = false>
static cudaError_t launch_rope_impl(void* q, void* k, const float* cos_tab, const float* sin_tab,
                                    int tab_rows, int tab_width, const int32_t* positions,
                                    int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                                    int is_bf16, int paired, int stagger_offset,
                                    const float* q_weight, const float* k_weight, float eps,
                                    cudaStream_t stream, const double2* fac = nullptr) {
    if (total_tokens == 0) return cudaSuccess;
    // Persistent grid: one wave of as many 256-thread blocks as are resident at once, each warp
    // striding over tokens, so no tail wave of partly filled SMs (at 1e5+ tokens this is ~7%
    // faster than one 8-token block per 8 tokens).
    const int threads = 256;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t blocks64 = (static_cast<int64_t>(total_tokens) + 7) / 8;
    const int64_t resident = static_cast<int64_t>(sms) *
                             (is_bf16 ? rope_min_blocks<__nv_bfloat16, NORM, FACT>()
                                      : rope_min_blocks<float, NORM, FACT>());
    const unsigned blocks = static_cast<unsigned>(blocks64 < resident ? blocks64 : resident);
    if (is_bf16)
        rope_kernel<__nv_bfloat16, NORM, NEG, FACT><<<blocks, threads, 0, stream>>>(
            static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), cos_tab, sin_tab,
            tab_rows, tab_width, positions, total_tokens, n_heads, n_kv_heads, head_dim, paired,
            stagger_offset, q_weight, k_weight, eps, fac);
    else
        rope_kernel<float, NORM, NEG, FACT><<<blocks, threads, 0, stream>>>(
            static_cast<float*>(q), static_cast<float*>(k), cos_tab, sin_tab, tab_rows, tab_width,
            positions, total_tokens, n_heads, n_kv_heads, head_dim, paired, stagger_offset,
            q_weight, k_weight, eps, fac);
    return cudaGetLastError();
}

// Ring depth and resident blocks of rope_ring_kernel: two slots per warp and three blocks per SM
// (up to 85 registers, which the rotation loop's unroll by two uses) for the rotation, three and
// three with the norm (measured on the paired workload: depth 2 at 4 blocks with 64 registers
// 80 us, 84 us once the packed rotation needed more registers than that; depth 2 at 3 blocks
// 78 us, 76.4 us unrolled; depth 3 at 3 blocks 78.2 us unrolled, 84 us with an earlier rotation;
// depth 4 at 2 blocks 98 us).
template <bool NORM>
constexpr int ring_depth() { return NORM ? 3 : 2; }
template <bool NORM>
constexpr int ring_blocks() { return 3; }

template <typename T, bool NEG, bool NORM, bool SEG>
static cudaError_t launch_rope_ring(void* q, void* k, const double2* fac, int rows,
                                   const int32_t* positions, int total_tokens, int n_heads,
                                   int n_kv_heads, int head_dim, int paired, int stagger_offset,
                                   const float* q_weight, const float* k_weight, float eps,
                                   int n_seg, int seg, int sms, cudaStream_t stream) {
    auto kern = rope_ring_kernel<T, NEG, NORM, SEG, ring_depth<NORM>(), ring_blocks<NORM>()>;
    const size_t smem = static_cast<size_t>(8) * ring_depth<NORM>() * seg * 16;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t blocks64 = (static_cast<int64_t>(total_tokens) * n_seg + 7) / 8;
    const int64_t resident = static_cast<int64_t>(sms) * ring_blocks<NORM>();
    const unsigned blocks = static_cast<unsigned>(blocks64 < resident ? blocks64 : resident);
    kern<<<blocks, 256, smem, stream>>>(static_cast<T*>(q), static_cast<T*>(k), positions,
                                        total_tokens, n_heads, n_kv_heads, head_dim, paired,
                                        stagger_offset, rows, fac, q_weight, k_weight, eps, n_seg,
                                        seg);
    return cudaGetLastError();
}

cudaError_t launch_rope_factored(void* q, void* k, const double2* fac, int rows,
                                 const int32_t* positions, int total_tokens, int n_heads,
                                 int n_kv_heads, int head_dim, int is_bf16, int paired,
                                 int stagger_offset, bool norm, bool neg, const float* q_weight,
                                 const float* k_weight, float eps, cudaStream_t stream) {
    const int width = paired ? 2 * head_dim : head_dim;
    // the ring kernel when a lane's chunks share table columns; a token wider than the ring's
    // slot (220 KB of shared memory per SM at the kernel's depth and blocks per SM) is split into
    // segments of a multiple of 32 chunks
    const int cph = head_dim / (is_bf16 ? 8 : 4);
    const bool uniform = (32 % cph == 0) && (!paired || ((32 / cph) % 2 == 0));
    if (uniform && total_tokens > 0) {
        const int n_chunks = (n_heads + n_kv_heads) * cph;
        const int per_chunk = 8 * 16 * (norm ? ring_depth<true>() * ring_blocks<true>()
                                             : ring_depth<false>() * ring_blocks<false>());
        const int seg_max = (220 * 1024 / per_chunk) / 32 * 32;
        int n_seg = 1, seg = n_chunks;
        if (n_chunks > seg_max) {
            n_seg = (n_chunks + seg_max - 1) / seg_max;
            seg = ((n_chunks + n_seg - 1) / n_seg + 31) / 32 * 32;
        }
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
#define PHA_RING(T_, NEG_, NORM_)                                                                \
    (n_seg > 1 ? launch_rope_ring<T_, NEG_, NORM_, true>(                                       \
                     q, k, fac, rows, positions, total_tokens, n_heads, n_kv_heads, head_dim,   \
                     paired, stagger_offset, q_weight, k_weight, eps, n_seg, seg, sms, stream)  \
               : launch_rope_ring<T_, NEG_, NORM_, false>(                                      \
                     q, k, fac, rows, positions, total_tokens, n_heads, n_kv_heads, head_dim,   \
                     paired, stagger_offset, q_weight, k_weight, eps, n_seg, seg, sms, stream))
        if (is_bf16)
            return norm ? PHA_RING(__nv_bfloat16, false, true)
                        : (neg ? PHA_RING(__nv_bfloat16, true, false)
                               : PHA_RING(__nv_bfloat16, false, false));
        return norm ? PHA_RING(float, false, true)
                    : (neg ? PHA_RING(float, true, false) : PHA_RING(float, false, false));
#undef PHA_RING
    }
    if (norm)
        return launch_rope_impl<true, false, true>(q, k, nullptr, nullptr, rows, width, positions,
                                                   total_tokens, n_heads, n_kv_heads, head_dim,
                                                   is_bf16, paired, stagger_offset, q_weight,
                                                   k_weight, eps, stream, fac);
    if (neg)
        return launch_rope_impl<false, true, true>(q, k, nullptr, nullptr, rows, width, positions,
                                                   total_tokens, n_heads, n_kv_heads, head_dim,
                                                   is_bf16, paired, stagger_offset, nullptr,
                                                   nullptr, 0.f, stream, fac);
    return launch_rope_impl<false, false, true>(q, k, nullptr, nullptr, rows, width, positions,
                                                total_tokens, n_heads, n_kv_heads, head_dim,
                                                is_bf16, paired, stagger_offset, nullptr, nullptr,
                                                0.f, stream, fac);
}

cudaError_t launch_rope(void* q, void* k, const float* cos_tab, const float* sin_tab, int tab_rows,
                        int tab_width, const int32_t* positions, int total_tokens, int n_heads,
                        int n_kv_heads, int head_dim, int is_bf16, int paired, int stagger_offset,
                        cudaStream_t stream) {
    return launch_rope_impl<false>(q, k, cos_tab, sin_tab, tab_rows, tab_width, positions,
                                   total_tokens, n_heads, n_kv_heads, head_dim, is_bf16, paired,
                                   stagger_offset, nullptr, nullptr, 0.f, stream);
}

cudaError_t launch_rope_bwd(void* dq, void* dk, const float* cos_tab, const float* sin_tab,
                            int tab_rows, int tab_width, const int32_t* positions, int total_tokens,
                            int n_heads, int n_kv_heads, int head_dim, int is_bf16, int paired,
                            int stagger_offset, cudaStream_t stream) {
    return launch_rope_impl<false, true>(dq, dk, cos_tab, sin_tab, tab_rows, tab_width, positions,
                                         total_tokens, n_heads, n_kv_heads, head_dim, is_bf16,
                                         paired, stagger_offset, nullptr, nullptr, 0.f, stream);
}

cudaError_t launch_qk_norm_rope(void* q, void* k, const float* q_weight, const float* k_weight,
                                float eps, const float* cos_tab, const float* sin_tab,
                                int tab_rows, int tab_width, const int32_t* positions,
                                int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                                int is_bf16, int paired, int stagger_offset, cudaStream_t stream) {
    return launch_rope_impl<true>(q, k, cos_tab, sin_tab, tab_rows, tab_width, positions,
                                  total_tokens, n_heads, n_kv_heads, head_dim, is_bf16, paired,
                                  stagger_offset, q_weight, k_weight, eps, stream);
}

}  // namespace pha
