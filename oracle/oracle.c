/*
 * oracle.c -- float64 CPU oracle for rotary embedding and causal / windowed varlen attention,
 * including the paired-head variant.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference leg may load this library. The product path (paired_heads_b200) never calls it,
 * and this file shares no code, header, table or constant with the CUDA library.
 *
 * Sources followed (web pages; cited by title and section):
 *   [PHA]  "modded-nanogpt Paired Head Attention record" (hncyxsy.com/news/170276):
 *          "core idea" (interleave two heads by position into a 2T sequence with H/2 heads),
 *          "interleave semantics under the causal mask", "zero-copy RoPE and delayed reshape",
 *          "staggered rotary", "sequence length and window handling" (seqlens and max_len doubled,
 *          window unchanged), "2. building the paired rotary table", "4. interleave index in the
 *          Triton kernel" (token t, head h -> slot 2t + h/(H/2), head h%(H/2); odd heads read the
 *          second half of the paired row).
 *   [RoPE] "Training an LLM from scratch (part 2): FlashAttention, GQA, RoPE, RMSNorm, SwiGLU"
 *          (juejin.cn), section "2. RoPE": inv_freq = 1 / base^(2i/d), rotation by +theta.
 *   [GQA]  same page, section "4. GQA & FlashAttention": query head h uses kv head h / (H/Hkv).
 *   [MASK] "ChatGPT" source notes (ranhao.site), section "SingleHeadAttention": lower-triangular
 *          causal mask, logits divided by sqrt(head_size), softmax over keys, weights times V.
 *   [SOFT] "mHC module" (lshu.cn/news/67890): softmax stabilised by subtracting the row max.
 *   [RMS]  "Training an LLM from scratch (part 2)", section "1. RMSNorm": y = x / sqrt(E[x^2] + eps)
 *          * gamma over the last dimension; [PHA] "4. interleave index in the Triton kernel": the
 *          rotary kernel also applies the QK RMS-norm (to each head row of q and k).
 *
 * Readings where the pages are silent or ambiguous (each is listed in the design notes):
 *   - rotation acts on adjacent pairs (x[2i], x[2i+1]) -- the [PHA] flip of a (..., D/2, 2) view;
 *   - the sine term enters with the standard sign: y0 = x0 cos - x1 sin, y1 = x0 sin + x1 cos
 *     ([RoPE] for one pair);
 *   - frequencies f_i = base^(-2i/hd), i = 0 .. hd/2-1, full rotary, no YaRN scaling;
 *   - paired phase of token t, head h: 2*pos[t] + (stagger ? h % 2 : 0);
 *   - window w > 0: key j visible from query slot i iff i - j < w (w slots counting i itself);
 *   - lse = natural log of the sum over visible keys of exp(scale * q.k).
 *
 * Everything is float64 with explicit loops in the order the definitions state. OpenMP only
 * distributes independent output rows; it does not change any row's arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL -1
#define ORACLE_ENOMEM -2

/* Rotary frequency of pair i: base^(-2i/hd)  ([RoPE] inv_freq). */
static double rope_freq(int i, int hd, double base)
{
    return pow(base, -2.0 * (double)i / (double)hd);
}

/* Rotary phase (in units of the frequency) of token t / head h. Standard: the token's position.
 * Paired: the paired table row p packs positions 2p and 2p+1, and odd heads read the second half
 * ([PHA] "staggered rotary", "2. building the paired rotary table"). */
static double rope_phase(int32_t pos, int h, int paired, int stagger)
{
    if (!paired) return (double)pos;
    return 2.0 * (double)pos + ((stagger && (h % 2)) ? 1.0 : 0.0);
}

/* In-place RoPE on x[n_tok][n_head][hd] (float64). table_f32 != 0 rounds each cosine and sine to
 * float32 before use, as the pipeline does when it keeps them in float32 tables ([PHA] "2. building
 * the paired rotary table": factor1 / factor2 are precomputed, stored tables); the rotation itself
 * stays float64. */
int oracle_rope(double* x, const int32_t* pos, int64_t n_tok, int n_head, int hd,
                int paired, int stagger, double base, int table_f32)
{
    if (!x || !pos || n_tok < 0 || n_head <= 0 || hd <= 0 || (hd % 2) != 0) return ORACLE_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int h = 0; h < n_head; ++h) {
            double* row = x + ((size_t)t * (size_t)n_head + (size_t)h) * (size_t)hd;
            double phase = rope_phase(pos[t], h, paired, stagger);
            for (int i = 0; i < hd / 2; ++i) {
                double theta = phase * rope_freq(i, hd, base);
                double c = cos(theta), s = sin(theta);
                if (table_f32) {
                    c = (double)(float)c;
                    s = (double)(float)s;
                }
                double a = row[2 * i], b = row[2 * i + 1];
                row[2 * i] = a * c - b * s;
                row[2 * i + 1] = a * s + b * c;
            }
        }
    }
    return ORACLE_OK;
}

/* RMS normalisation of each of the n_rows rows of x[n_rows][d] (in place), [RMS]:
 * y_j = x_j / sqrt((1/d) sum_k x_k^2 + eps) * gamma_j; gamma == NULL stands for all ones. */
int oracle_rms_norm(double* x, int64_t n_rows, int d, const double* gamma, double eps)
{
    if (!x || n_rows < 0 || d <= 0 || !(eps >= 0.0)) return ORACLE_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        double* row = x + (size_t)r * (size_t)d;
        double ms = 0.0;
        for (int j = 0; j < d; ++j) ms += row[j] * row[j];
        ms /= (double)d;
        double scale = 1.0 / sqrt(ms + eps);
        for (int j = 0; j < d; ++j) row[j] = row[j] * scale * (gamma ? gamma[j] : 1.0);
    }
    return ORACLE_OK;
}

/* Round every element to the nearest bfloat16 value (ties to even), in place. Used where the
 * pipeline stores a result in a bf16 buffer: RoPE rotates the bf16 q and k tensors in place
 * ([PHA] "zero-copy RoPE and delayed reshape": the rotated q, k are the tensors attention reads).
 * bfloat16 keeps 8 significant bits; the smallest normal value is 2^-126. */
static double round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    double m = frexp(x, &e); /* x = m * 2^e, 0.5 <= |m| < 1 */
    int bits = 8;
    if (e < -125) bits -= (-125 - e); /* subnormal range: fewer significant bits */
    if (bits < 0) return copysign(0.0, x);
    double r = nearbyint(ldexp(m, bits)); /* default rounding mode: to nearest, ties to even */
    double y = ldexp(r, e - bits);
    if (fabs(y) > 0x1.FEp127) return copysign(INFINITY, x); /* beyond the largest bf16 value */
    return y;
}

int oracle_round_bf16(double* x, int64_t n)
{
    if (!x || n < 0) return ORACLE_EINVAL;
    for (int64_t i = 0; i < n; ++i) x[i] = round_bf16(x[i]);
    return ORACLE_OK;
}

/* ---- e4m3 ("float8_e4m3fn"): the 8-bit floating point format of the packed FP8 Q/K/V path
 * ([PHA] "5. interactions with other mechanisms": on paired layers the FP8 QKV projection is
 * issued as separate column-slice GEMMs, so attention may receive Q, K, V in FP8).
 * Format (the OCP FP8 E4M3 definition, the one torch.float8_e4m3fn implements): 1 sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits. Exponent field 0 holds the subnormals
 * m/8 * 2^-6 = m * 2^-9; exponent field E in 1..15 holds (1 + m/8) * 2^(E-7); the two codes with
 * all exponent and mantissa bits set are NaN; there is no infinity, and the largest finite value
 * is 1.75 * 2^8 = 448. A tensor of codes b with per-tensor float32 scale s stands for s * value(b). */
static double decode_e4m3(uint8_t b)
{
    const int sign = b >> 7, E = (b >> 3) & 15, m = b & 7;
    if (E == 15 && m == 7) return NAN;
    const double v = E == 0 ? ldexp((double)m, -9) : ldexp(8.0 + (double)m, E - 10);
    return sign ? -v : v;
}

int oracle_decode_e4m3(const uint8_t* b, double* y, int64_t n)
{
    if ((!b || !y) && n > 0) return ORACLE_EINVAL;
    for (int64_t i = 0; i < n; ++i) y[i] = decode_e4m3(b[i]);
    return ORACLE_OK;
}

/* Nearest e4m3 code of x, ties to even (the mantissa code with its low bit clear). A magnitude
 * that rounds past 448 (above the midpoint 464 between 448 and the next step, 480), an infinity
 * or a NaN gives NaN: the format cannot hold it (torch's float8_e4m3fn cast behaves the same). */
static uint8_t encode_e4m3(double x)
{
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs(x);
    if (isinf(a)) return sign | 0x7F;
    if (a < ldexp(1.0, -6)) {                       /* subnormal grid, step 2^-9 */
        const double q = nearbyint(a * 512.0);      /* 0 .. 8; 8 is the smallest normal 2^-6 */
        return sign | (uint8_t)q;
    }
    int e;
    frexp(a, &e);                                   /* a in [2^(e-1), 2^e) */
    int E = e - 1;
    double q = nearbyint(ldexp(a, 3 - E));          /* 8 .. 16 significand steps of 2^(E-3) */
    if (q == 16.0) {
        E += 1;
        q = 8.0;
    }
    if (E > 8 || (E == 8 && q > 14.0)) return sign | 0x7F; /* past 448 */
    return sign | (uint8_t)(((E + 7) << 3) | ((int)q - 8));
}

int oracle_encode_e4m3(const double* x, uint8_t* b, int64_t n)
{
    if ((!b || !x) && n > 0) return ORACLE_EINVAL;
    for (int64_t i = 0; i < n; ++i) b[i] = encode_e4m3(x[i]);
    return ORACLE_OK;
}

/* Explicit paired interleave ([PHA] "core idea", "4. interleave index"): token t, head h of
 * x[T][H][d] moves to slot 2t + h/(H/2), head h % (H/2) of y[2T][H/2][d]. A copy loop, not a view. */
int oracle_interleave(const double* x, double* y, int64_t T, int H, int d)
{
    if (!x || !y || T < 0 || H <= 0 || (H % 2) != 0 || d <= 0) return ORACLE_EINVAL;
    const int Hp = H / 2;
    for (int64_t t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            int64_t slot = 2 * t + h / Hp;
            int hp = h % Hp;
            for (int e = 0; e < d; ++e)
                y[((size_t)slot * Hp + hp) * d + e] = x[((size_t)t * H + h) * d + e];
        }
    return ORACLE_OK;
}

/* Inverse of oracle_interleave: y[2T][H/2][d] -> x[T][H][d]. */
int oracle_deinterleave(const double* y, double* x, int64_t T, int H, int d)
{
    if (!x || !y || T < 0 || H <= 0 || (H % 2) != 0 || d <= 0) return ORACLE_EINVAL;
    const int Hp = H / 2;
    for (int64_t t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            int64_t slot = 2 * t + h / Hp;
            int hp = h % Hp;
            for (int e = 0; e < d; ++e)
                x[((size_t)t * H + h) * d + e] = y[((size_t)slot * Hp + hp) * d + e];
        }
    return ORACLE_OK;
}

/* Is key slot j visible from query slot i of a document spanning [lo, hi)? ([MASK] tril;
 * [PHA] window kept as is on the 2T sequence). */
static int visible(int64_t i, int64_t j, int64_t lo, int64_t hi, int causal, int window)
{
    if (j < lo || j >= hi) return 0;
    if (causal && j > i) return 0;
    if (window > 0 && i - j >= window) return 0;
    return 1;
}

/* One output row: query slot i, head h of a document [lo, hi). Plain two-pass stable softmax
 * ([SOFT]): m = max_j s_j; l = sum_j exp(s_j - m); o = sum_j exp(s_j - m) v_j / l; lse = m + ln l. */
static void attend_row(const double* q, const double* k, const double* v, int64_t i, int h,
                       int64_t lo, int64_t hi, int H, int Hkv, int hd, int causal, int window,
                       double scale, double* o_row, double* lse_out)
{
    const int g = h / (H / Hkv); /* [GQA] */
    const double* qi = q + ((size_t)i * H + h) * hd;
    double m = -INFINITY;
    for (int64_t j = lo; j < hi; ++j) {
        if (!visible(i, j, lo, hi, causal, window)) continue;
        const double* kj = k + ((size_t)j * Hkv + g) * hd;
        double s = 0.0;
        for (int e = 0; e < hd; ++e) s += qi[e] * kj[e];
        s *= scale;
        if (s > m) m = s;
    }
    for (int e = 0; e < hd; ++e) o_row[e] = 0.0;
    if (m == -INFINITY) { /* no visible key: defined as zero output, lse = -inf */
        *lse_out = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int64_t j = lo; j < hi; ++j) {
        if (!visible(i, j, lo, hi, causal, window)) continue;
        const double* kj = k + ((size_t)j * Hkv + g) * hd;
        const double* vj = v + ((size_t)j * Hkv + g) * hd;
        double s = 0.0;
        for (int e = 0; e < hd; ++e) s += qi[e] * kj[e];
        s *= scale;
        double p = exp(s - m);
        l += p;
        for (int e = 0; e < hd; ++e) o_row[e] += p * vj[e];
    }
    for (int e = 0; e < hd; ++e) o_row[e] /= l;
    *lse_out = m + log(l);
}

static int check_cu(const int64_t* cu, int B)
{
    if (cu[0] < 0) return 0;
    for (int b = 0; b < B; ++b)
        if (cu[b + 1] < cu[b]) return 0;
    return 1;
}

/* Attention over slot-major buffers q[S][H][hd], k,v[S][Hkv][hd]; documents are the slot ranges
 * [cu[b], cu[b+1]). o[S][H][hd], lse[S][H]. */
int oracle_attention(const double* q, const double* k, const double* v, const int64_t* cu, int B,
                     int H, int Hkv, int hd, int causal, int window, double scale, double* o,
                     double* lse)
{
    if (!q || !k || !v || !cu || !o || !lse || B < 0 || H <= 0 || Hkv <= 0 || (H % Hkv) != 0 ||
        hd <= 0 || !check_cu(cu, B))
        return ORACLE_EINVAL;
    for (int b = 0; b < B; ++b) {
        const int64_t lo = cu[b], hi = cu[b + 1];
        const int64_t n = (hi - lo) * (int64_t)H;
#pragma omp parallel for schedule(dynamic, 16)
        for (int64_t r = 0; r < n; ++r) {
            int64_t i = lo + r / H;
            int h = (int)(r % H);
            attend_row(q, k, v, i, h, lo, hi, H, Hkv, hd, causal, window, scale,
                       o + ((size_t)i * H + h) * hd, lse + (size_t)i * H + h);
        }
    }
    return ORACLE_OK;
}

/* Selected rows only: rows[r] = slot * H + head. Same arithmetic as oracle_attention. */
int oracle_attention_rows(const double* q, const double* k, const double* v, const int64_t* cu,
                          int B, int H, int Hkv, int hd, int causal, int window, double scale,
                          const int64_t* rows, int64_t n_rows, double* o_rows, double* lse_rows)
{
    if (!q || !k || !v || !cu || !rows || !o_rows || !lse_rows || B <= 0 || H <= 0 || Hkv <= 0 ||
        (H % Hkv) != 0 || hd <= 0 || n_rows < 0 || !check_cu(cu, B))
        return ORACLE_EINVAL;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows[r] / H;
        int h = (int)(rows[r] % H);
        if (rows[r] < 0 || i >= cu[B]) { bad = 1; continue; }
        /* document containing slot i: the last b with cu[b] <= i (binary search) */
        int a = 0, z = B; /* invariant: cu[a] <= i < cu[z] */
        while (z - a > 1) {
            int mid = (a + z) / 2;
            if (cu[mid] <= i) a = mid; else z = mid;
        }
        while (a + 1 < B && cu[a + 1] <= i) ++a; /* skip empty documents */
        attend_row(q, k, v, i, h, cu[a], cu[a + 1], H, Hkv, hd, causal, window, scale,
                   o_rows + (size_t)r * hd, lse_rows + r);
    }
    return bad ? ORACLE_EINVAL : ORACLE_OK;
}

/* Full forward in the caller's layout: q[T][H][hd], k,v[T][Hkv][hd], cu_seqlens in tokens.
 * Paired: explicitly interleave q, k, v into [2T][H/2][hd], double cu_seqlens ([PHA] "sequence
 * length and window handling"), attend with H/2 and Hkv/2 heads and the unchanged window, then
 * de-interleave o and lse back to [T][H]. */
int oracle_attn_fwd(const double* q, const double* k, const double* v, const int32_t* cu_seqlens,
                    int B, int H, int Hkv, int hd, int causal, int window, int paired,
                    double scale, double* o, double* lse)
{
    if (!q || !k || !v || !cu_seqlens || !o || !lse || B < 0 || H <= 0 || Hkv <= 0 ||
        (H % Hkv) != 0 || hd <= 0)
        return ORACLE_EINVAL;
    if (paired && ((H % 2) != 0 || (Hkv % 2) != 0)) return ORACLE_EINVAL;
    const int64_t T = cu_seqlens[B];
    int64_t* cu = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
    if (!cu) return ORACLE_ENOMEM;
    for (int b = 0; b <= B; ++b) cu[b] = (paired ? 2 : 1) * (int64_t)cu_seqlens[b];
    int rc;
    if (!paired) {
        rc = oracle_attention(q, k, v, cu, B, H, Hkv, hd, causal, window, scale, o, lse);
        free(cu);
        return rc;
    }
    const int Hp = H / 2, Hkvp = Hkv / 2;
    const size_t nq = (size_t)T * H * hd, nk = (size_t)T * Hkv * hd;
    double* qi = (double*)malloc(nq * sizeof(double));
    double* ki = (double*)malloc(nk * sizeof(double));
    double* vi = (double*)malloc(nk * sizeof(double));
    double* oi = (double*)malloc(nq * sizeof(double));
    double* li = (double*)malloc((size_t)T * H * sizeof(double));
    if (!qi || !ki || !vi || !oi || !li) {
        free(qi); free(ki); free(vi); free(oi); free(li); free(cu);
        return ORACLE_ENOMEM;
    }
    oracle_interleave(q, qi, T, H, hd);
    oracle_interleave(k, ki, T, Hkv, hd);
    oracle_interleave(v, vi, T, Hkv, hd);
    rc = oracle_attention(qi, ki, vi, cu, B, Hp, Hkvp, hd, causal, window, scale, oi, li);
    if (rc == ORACLE_OK) {
        oracle_deinterleave(oi, o, T, H, hd);
        oracle_deinterleave(li, lse, T, H, 1);
    }
    free(qi); free(ki); free(vi); free(oi); free(li); free(cu);
    return rc;
}

/* ------------------------------------------------------------------ backward (gradients)
 * The gradients of the attention above with respect to q, k, v for an upstream gradient dO, by
 * the chain rule through the row softmax (the standard identity: with P_ij the softmax weights,
 * dP_ij = dO_i . v_j, dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik), dQ_i = scale sum_j dS_ij k_j,
 * dK_j = scale sum_i dS_ij q_i, dV_j = sum_i P_ij dO_i). P is recomputed here from q and k with
 * the same two-pass softmax as attend_row; nothing saved by the forward is used. */

/* Slot-major buffers as oracle_attention; dq[S][H][hd], dk, dv[S][Hkv][hd] (overwritten). */
int oracle_attention_bwd(const double* q, const double* k, const double* v, const double* dout,
                         const int64_t* cu, int B, int H, int Hkv, int hd, int causal, int window,
                         double scale, double* dq, double* dk, double* dv)
{
    if (!q || !k || !v || !dout || !cu || !dq || !dk || !dv || B < 0 || H <= 0 || Hkv <= 0 ||
        (H % Hkv) != 0 || hd <= 0 || !check_cu(cu, B))
        return ORACLE_EINVAL;
    const int G = H / Hkv;
    const int64_t S = cu[B];
    memset(dq, 0, sizeof(double) * (size_t)S * H * hd);
    memset(dk, 0, sizeof(double) * (size_t)S * Hkv * hd);
    memset(dv, 0, sizeof(double) * (size_t)S * Hkv * hd);
    for (int b = 0; b < B; ++b) {
        const int64_t lo = cu[b], hi = cu[b + 1];
        const int64_t L = hi - lo;
        if (L <= 0) continue;
        /* one kv head per task: its dk, dv rows receive every query head of its group */
#pragma omp parallel for schedule(dynamic, 1)
        for (int g = 0; g < Hkv; ++g) {
            double* p = (double*)malloc(sizeof(double) * (size_t)L);
            double* dp = (double*)malloc(sizeof(double) * (size_t)L);
            for (int h = g * G; h < (g + 1) * G; ++h) {
                for (int64_t i = lo; i < hi; ++i) {
                    const double* qi = q + ((size_t)i * H + h) * hd;
                    const double* gi = dout + ((size_t)i * H + h) * hd;
                    double m = -INFINITY;
                    for (int64_t j = lo; j < hi; ++j) {
                        p[j - lo] = -INFINITY;
                        if (!visible(i, j, lo, hi, causal, window)) continue;
                        const double* kj = k + ((size_t)j * Hkv + g) * hd;
                        double sc = 0.0;
                        for (int e = 0; e < hd; ++e) sc += qi[e] * kj[e];
                        p[j - lo] = sc * scale;
                        if (p[j - lo] > m) m = p[j - lo];
                    }
                    if (m == -INFINITY) continue;
                    double l = 0.0;
                    for (int64_t j = lo; j < hi; ++j) {
                        p[j - lo] = (p[j - lo] == -INFINITY) ? 0.0 : exp(p[j - lo] - m);
                        l += p[j - lo];
                    }
                    double dsum = 0.0;
                    for (int64_t j = lo; j < hi; ++j) {
                        p[j - lo] /= l;
                        dp[j - lo] = 0.0;
                        if (p[j - lo] == 0.0) continue;
                        const double* vj = v + ((size_t)j * Hkv + g) * hd;
                        for (int e = 0; e < hd; ++e) dp[j - lo] += gi[e] * vj[e];
                        dsum += p[j - lo] * dp[j - lo];
                    }
                    double* dqi = dq + ((size_t)i * H + h) * hd;
                    for (int64_t j = lo; j < hi; ++j) {
                        if (p[j - lo] == 0.0) continue;
                        const double ds = p[j - lo] * (dp[j - lo] - dsum);
                        const double* kj = k + ((size_t)j * Hkv + g) * hd;
                        double* dkj = dk + ((size_t)j * Hkv + g) * hd;
                        double* dvj = dv + ((size_t)j * Hkv + g) * hd;
                        for (int e = 0; e < hd; ++e) {
                            dqi[e] += scale * ds * kj[e];
                            dkj[e] += scale * ds * qi[e];
                            dvj[e] += p[j - lo] * gi[e];
                        }
                    }
                }
            }
            free(p);
            free(dp);
        }
    }
    return ORACLE_OK;
}

/* Token-major wrapper like oracle_attn_fwd: paired = 1 interleaves q, k, v, dout explicitly, runs
 * the slot-major backward on the doubled documents and de-interleaves dq, dk, dv. */
int oracle_attn_bwd(const double* q, const double* k, const double* v, const double* dout,
                    const int32_t* cu_seqlens, int B, int H, int Hkv, int hd, int causal,
                    int window, int paired, double scale, double* dq, double* dk, double* dv)
{
    if (!q || !k || !v || !dout || !cu_seqlens || !dq || !dk || !dv || B < 0 || H <= 0 ||
        Hkv <= 0 || (H % Hkv) != 0 || hd <= 0)
        return ORACLE_EINVAL;
    if (paired && ((H % 2) != 0 || (Hkv % 2) != 0)) return ORACLE_EINVAL;
    const int64_t T = cu_seqlens[B];
    int64_t* cu = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
    if (!cu) return ORACLE_ENOMEM;
    for (int b = 0; b <= B; ++b) cu[b] = (paired ? 2 : 1) * (int64_t)cu_seqlens[b];
    int rc;
    if (!paired) {
        rc = oracle_attention_bwd(q, k, v, dout, cu, B, H, Hkv, hd, causal, window, scale, dq, dk,
                                  dv);
        free(cu);
        return rc;
    }
    const size_t nq = (size_t)T * H * hd, nk = (size_t)T * Hkv * hd;
    double* buf = (double*)malloc(sizeof(double) * (4 * nq + 4 * nk));
    if (!buf) { free(cu); return ORACLE_ENOMEM; }
    double *qi = buf, *gi = qi + nq, *dqi = gi + nq, *ki = dqi + nq, *vi = ki + nk, *dki = vi + nk,
           *dvi = dki + nk;
    oracle_interleave(q, qi, T, H, hd);
    oracle_interleave(dout, gi, T, H, hd);
    oracle_interleave(k, ki, T, Hkv, hd);
    oracle_interleave(v, vi, T, Hkv, hd);
    rc = oracle_attention_bwd(qi, ki, vi, gi, cu, B, H / 2, Hkv / 2, hd, causal, window, scale,
                              dqi, dki, dvi);
    if (rc == ORACLE_OK) {
        oracle_deinterleave(dqi, dq, T, H, hd);
        oracle_deinterleave(dki, dk, T, Hkv, hd);
        oracle_deinterleave(dvi, dv, T, Hkv, hd);
    }
    free(buf);
    free(cu);
    return rc;
}

/* Gradient of oracle_rope with respect to its input: the transposed rotation of every pair,
 * dx0 = c dy0 + s dy1, dx1 = -s dy0 + c dy1 (in place on dy[n_tok][n_head][hd]). */
int oracle_rope_bwd(double* dy, const int32_t* pos, int64_t n_tok, int n_head, int hd,
                    int paired, int stagger, double base, int table_f32)
{
    if (!dy || !pos || n_tok < 0 || n_head <= 0 || hd <= 0 || (hd % 2) != 0) return ORACLE_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int h = 0; h < n_head; ++h) {
            double* row = dy + ((size_t)t * (size_t)n_head + (size_t)h) * (size_t)hd;
            double phase = rope_phase(pos[t], h, paired, stagger);
            for (int i = 0; i < hd / 2; ++i) {
                double theta = phase * rope_freq(i, hd, base);
                double c = cos(theta), s = sin(theta);
                if (table_f32) {
                    c = (double)(float)c;
                    s = (double)(float)s;
                }
                double a = row[2 * i], b = row[2 * i + 1];
                row[2 * i] = a * c + b * s;
                row[2 * i + 1] = -a * s + b * c;
            }
        }
    }
    return ORACLE_OK;
}
