/*
 * CPU oracle for the FP8 "fast-math" linear layer, its W8A16 default path and
 * its routed-expert variant.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or constant with the CUDA library.
 *
 * Everything here is written for a reader who checks it against the model
 * cards by eye: plain loops, float64 accumulation, one rounding at the end.
 * The only liberty taken is an OpenMP "parallel for" over independent output
 * rows, which changes no result.
 *
 * Sources (model cards of the Metis-1.6 family):
 *  - "Lernex/Metis-1.6-Logos-FP8", section "What --fast-math does": each
 *    layer's input is rounded to FP8 per token and multiplied with the FP8
 *    weights on FP8 tensor cores; the default instead widens the FP8 weights
 *    to 16 bits and does BF16 maths, so only the weights are rounded.
 *  - same card, section "What is in FP8": E4M3 weights with one scale per
 *    output channel, activations quantized per token at run time, routed
 *    experts among the FP8 tensors.
 *  - "Lernex/Metis-1.6-Praxis-NVFP4", section "What --fast-math does": the
 *    same two ways of multiplying; single-stream decode always takes the
 *    default maths.
 *  - The E4M3 number format itself is the OCP 8-bit floating point
 *    specification (OFP8), "E4M3" encoding: bias 7, no infinities, one NaN
 *    mantissa pattern (S.1111.111), largest finite magnitude 448.
 *
 * Readings where the cards are silent (they print no formula):
 *  - scale s = amax/448 in binary32; the element is multiplied by
 *    inv = 448/amax (binary32, clamped to FLT_MAX, 0 when amax = 0) and the
 *    binary32 product is rounded once to E4M3, nearest-even, saturating.
 *  - GEMM results are s_tok[m]*s_w[n]*sum_k D(a)*D(b) in float64, rounded
 *    once to BF16, nearest-even.
 *  - W8A16: s_w[n] is applied to the float64 sum, not to the weights.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (see build.py).
 * -ffp-contract=off keeps every binary32 multiply a separate rounding.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_NONFINITE 1
#define ORACLE_BAD_INDEX 2

/* ---------------------------------------------------------------- helpers */

/* BF16 bit pattern -> binary32 value (the BF16 bits are the high half). */
static float bf16_bits_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a non-negative real r (exactly representable as a double) to the
 * nearest integer, ties to even. */
static double round_half_even(double r) {
    double fl = floor(r);
    double diff = r - fl; /* exact: r and fl share the binade or fl = 0 */
    if (diff > 0.5) return fl + 1.0;
    if (diff < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* ------------------------------------------------------------ E4M3 codec */

/* D(b): the exact real value of an E4M3 byte (OFP8 E4M3: bias 7,
 * subnormals m * 2^-9, S.1111.111 is NaN). */
double metis_oracle_e4m3_decode(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return sign ? -NAN : NAN;
    if (e == 0)
        v = ldexp((double)m, -9);              /* subnormal: 0.m * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);    /* 1.m * 2^(e-7) */
    return sign ? -v : v;
}

/* Q(v): binary32 -> E4M3 byte, round to nearest even on the E4M3 grid,
 * saturating to +-448 (the "satfinite" behaviour). NaN -> S.1111.111. */
uint8_t metis_oracle_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a, q, r, res;
    int e2, E;
    if (isnan(v)) return sign | 0x7F;
    a = fabs((double)v);
    /* Everything at or beyond the largest finite value saturates: (448,464]
     * rounds to 448 (464 is the tie with the would-be 480, whose mantissa
     * 111 is odd) and above 464 it would round past 448, which satfinite
     * clamps back to 448. Infinities saturate as well. */
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    frexp(a, &e2);
    E = e2 - 1;                 /* a in [2^E, 2^(E+1)) */
    if (E < -6) E = -6;         /* subnormals share the quantum of binade -6 */
    q = ldexp(1.0, E - 3);      /* three fraction bits */
    r = a / q;                  /* exact: q is a power of two */
    res = round_half_even(r) * q;
    if (res == 0.0) return sign;
    if (res < ldexp(1.0, -6)) {
        int mant = (int)(res / ldexp(1.0, -9));  /* 1..7 */
        return sign | (uint8_t)mant;
    }
    frexp(res, &e2);
    E = e2 - 1;                  /* res may have moved up one binade */
    {
        int mant = (int)(res / ldexp(1.0, E - 3)) - 8; /* 0..7 */
        int field = E + 7;                              /* 1..15 */
        return sign | (uint8_t)(field << 3) | (uint8_t)mant;
    }
}

/* --------------------------------------------------------------- BF16 RNE */

/* A real value (given as a double) rounded once to BF16, nearest-even,
 * overflow to infinity; returns the BF16 bit pattern. */
uint16_t metis_oracle_bf16_from_double(double v) {
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a, q, res;
    int e2, E;
    float f;
    uint32_t u;
    if (isnan(v)) return 0x7FC0;
    a = fabs(v);
    if (isinf(a)) return sign | 0x7F80;
    if (a == 0.0) return sign;
    frexp(a, &e2);
    E = e2 - 1;
    if (E < -126) E = -126;      /* BF16 subnormals: quantum 2^-133 */
    q = ldexp(1.0, E - 7);       /* seven fraction bits */
    res = round_half_even(a / q) * q;
    if (res >= ldexp(1.0, 128)) return sign | 0x7F80;
    f = (float)res;              /* exact: at most 8 significant bits */
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

/* ------------------------------------------------ per-row FP8 quantization */

/* One row: amax, s = amax/448, inv = 448/amax (clamped), codes Q(x*inv). */
static void quant_one_row(const float* row, int64_t K, uint8_t* q, float* s) {
    float amax = 0.0f, sc, inv;
    int64_t k;
    for (k = 0; k < K; ++k) {
        float a = fabsf(row[k]);
        if (a > amax) amax = a;
    }
    sc = amax / 448.0f;
    inv = (amax > 0.0f) ? fminf(448.0f / amax, FLT_MAX) : 0.0f;
    *s = sc;
    for (k = 0; k < K; ++k) {
        float prod = row[k] * inv;   /* one binary32 rounding */
        q[k] = metis_oracle_e4m3_encode(prod);
    }
}

/* Per-token quantization of BF16 activations x[M][ldx] (each layer's input
 * rounded to FP8 per token at run time). */
int metis_oracle_quant_rows_bf16(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                 uint8_t* q, int64_t ldq, float* s) {
    int64_t m;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (m = 0; m < M; ++m) {
        float* row = (float*)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
        int64_t k;
        for (k = 0; k < K; ++k) {
            row[k] = bf16_bits_to_float(x[m * ldx + k]);  /* exact widening */
            if (!isfinite(row[k])) bad = 1;
        }
        quant_one_row(row, K, q + m * ldq, s + m);
        free(row);
    }
    return bad ? ORACLE_NONFINITE : ORACLE_OK;
}

/* Per-output-channel quantization of binary32 weights w[N][ldw] (the
 * checkpoint format: E4M3 weights with one scale per output channel). */
int metis_oracle_quant_rows_f32(const float* w, int64_t N, int64_t K, int64_t ldw,
                                uint8_t* q, int64_t ldq, float* s) {
    int64_t n;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (n = 0; n < N; ++n) {
        int64_t k;
        for (k = 0; k < K; ++k)
            if (!isfinite(w[n * ldw + k])) bad = 1;
        quant_one_row(w + n * ldw, K, q + n * ldq, s + n);
    }
    return bad ? ORACLE_NONFINITE : ORACLE_OK;
}

/* ------------------------------------------------------------------ GEMMs */

/* W8A8: y[r][n] = bf16( s_tok[m] * s_w[n] * sum_k D(xq[m][k]) * D(wq[n][k]) )
 * for m = rows[r] (or m = r when rows is NULL). The float64 sum is exact
 * for K <= 8192: every product is an integer multiple of 2^-18 below 2^18. */
int metis_oracle_gemm_w8a8(const uint8_t* xq, int64_t ldq, const float* s_tok,
                           const uint8_t* wq, int64_t ldw, const float* s_w,
                           int64_t M, int64_t N, int64_t K,
                           const int64_t* rows, int64_t nrows,
                           uint16_t* y, double* y64) {
    double dec[256];
    int64_t r;
    int i, bad = 0;
    for (i = 0; i < 256; ++i) dec[i] = metis_oracle_e4m3_decode((uint8_t)i);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (r = 0; r < nrows; ++r) {
        int64_t m = rows ? rows[r] : r;
        int64_t n, k;
        if (m < 0 || m >= M) { bad = 1; continue; }
        for (n = 0; n < N; ++n) {
            double acc = 0.0, v;
            for (k = 0; k < K; ++k)
                acc += dec[xq[m * ldq + k]] * dec[wq[n * ldw + k]];
            v = (double)s_tok[m] * (double)s_w[n] * acc;
            if (y64) y64[r * N + n] = v;
            y[r * N + n] = metis_oracle_bf16_from_double(v);
        }
    }
    return bad ? ORACLE_BAD_INDEX : ORACLE_OK;
}

/* W8A16 (the default maths): y[m][n] = bf16( s_w[n] * sum_k x[m][k] * D(wq[n][k]) ),
 * x in BF16, the weights widened exactly, the per-channel scale applied to
 * the sum, float64 accumulation. */
int metis_oracle_gemm_w8a16(const uint16_t* x, int64_t ldx,
                            const uint8_t* wq, int64_t ldw, const float* s_w,
                            int64_t M, int64_t N, int64_t K,
                            uint16_t* y, double* y64) {
    double dec[256];
    int64_t n;
    int i;
    for (i = 0; i < 256; ++i) dec[i] = metis_oracle_e4m3_decode((uint8_t)i);
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        int64_t m, k;
        for (m = 0; m < M; ++m) {
            double acc = 0.0, v;
            for (k = 0; k < K; ++k)
                acc += (double)bf16_bits_to_float(x[m * ldx + k]) * dec[wq[n * ldw + k]];
            v = (double)s_w[n] * acc;
            if (y64) y64[m * N + n] = v;
            y[m * N + n] = metis_oracle_bf16_from_double(v);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------- routed experts */

/* Routing bookkeeping for slots s = t*topk + j (token t, choice j):
 * counts[e] = number of slots routed to e; offsets = exclusive prefix sum
 * (E+1 entries); slot_to_row[s] = offsets[e] + number of earlier slots (in
 * slot order) routed to the same expert, i.e. a stable sort by expert. */
int metis_oracle_moe_route(const int32_t* ids, int64_t T, int64_t topk, int64_t E,
                           int32_t* counts, int32_t* offsets, int32_t* slot_to_row,
                           int32_t* row_to_slot) {
    int64_t s, e, S = T * topk;
    for (e = 0; e < E; ++e) counts[e] = 0;
    for (s = 0; s < S; ++s) {
        if (ids[s] < 0 || ids[s] >= E) return ORACLE_BAD_INDEX;
        counts[ids[s]] += 1;
    }
    offsets[0] = 0;
    for (e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (e = 0; e < E; ++e) counts[e] = 0; /* reuse as per-expert fill */
    for (s = 0; s < S; ++s) {
        int32_t x = ids[s];
        int32_t row = offsets[x] + counts[x];
        counts[x] += 1;
        slot_to_row[s] = row;
        if (row_to_slot) row_to_slot[row] = (int32_t)s;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ NVFP4
 * "Lernex/Metis-1.6-Praxis-NVFP4", "What is in NVFP4": the routed experts are
 * "4-bit E2M1 values with one FP8 (E4M3) scale per 16 inputs and an FP32
 * scale per expert"; with --fast-math "the 4-bit experts multiply in FP4",
 * their inputs rounded to FP4 too (section "What --fast-math does"). The card
 * prints no rounding rule. Reading, for a row (a token, or an output channel
 * of an expert) and its scale owner (the token itself, or the whole expert):
 *   g     = amax_owner / 2688            (binary32; 2688 = 6 * 448)
 *   inv_g = 2688 / amax_owner, 0 if amax_owner = 0 (binary32, FLT_MAX clamp)
 *   per 16-element block with block amax b:
 *     sb  = E4M3( (b * inv_g) / 6 )      (each step binary32, nearest-even,
 *                                         saturating; a non-negative code)
 *     q_i = E2M1( (x_i * inv_g) * (1 / D(sb)) ), 0 when sb decodes to 0
 *   value_i = D2(q_i) * D(sb) * g.
 * E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit: magnitudes
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6; nearest-even, saturating to 6, no NaN. */
double metis_oracle_e2m1_decode(uint8_t c) {
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = mag[c & 7];
    return (c & 8) ? -v : v;
}

uint8_t metis_oracle_e2m1_encode(float v) {
    /* nearest of the 8 magnitudes, ties to the even mantissa (codes 0, 2, 4, 6) */
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    uint8_t best = 0;
    int i;
    if (a >= 6.0) return sign | 7; /* saturate */
    for (i = 1; i < 8; ++i) {
        double d_best = fabs(a - mag[best]), d = fabs(a - mag[i]);
        if (d < d_best || (d == d_best && (i & 1) == 0)) best = (uint8_t)i;
    }
    return sign | best;
}

/* Quantizes rows [R, K] (K % 16 == 0) to NVFP4: codes [R, K] one per byte,
 * block scales [R, K/16] E4M3 codes, and the global scale(s): one per row
 * when per_row != 0, else one for all rows (written to g[0]). */
int metis_oracle_nvfp4_quant(const float* x, int64_t R, int64_t K, int per_row, uint8_t* q,
                             uint8_t* sb, float* g) {
    int64_t r, k, b;
    float amax_all = 0.0f;
    if (K % 16 != 0) return ORACLE_BAD_INDEX;
    if (!per_row) {
        for (r = 0; r < R * K; ++r) {
            float a = fabsf(x[r]);
            if (a > amax_all) amax_all = a;
        }
    }
    for (r = 0; r < R; ++r) {
        const float* row = x + r * K;
        float amax = amax_all, inv_g;
        if (per_row) {
            amax = 0.0f;
            for (k = 0; k < K; ++k)
                if (fabsf(row[k]) > amax) amax = fabsf(row[k]);
        }
        inv_g = amax > 0.0f ? 2688.0f / amax : 0.0f;
        if (inv_g > FLT_MAX) inv_g = FLT_MAX;
        if (per_row) g[r] = amax / 2688.0f;
        else if (r == 0) g[0] = amax / 2688.0f;
        for (b = 0; b < K / 16; ++b) {
            float bamax = 0.0f, t, ds, inv_s;
            uint8_t code;
            for (k = 0; k < 16; ++k)
                if (fabsf(row[b * 16 + k]) > bamax) bamax = fabsf(row[b * 16 + k]);
            t = bamax * inv_g;
            t = t / 6.0f;
            code = metis_oracle_e4m3_encode(t);
            sb[r * (K / 16) + b] = code;
            ds = (float)metis_oracle_e4m3_decode(code);
            inv_s = ds > 0.0f ? 1.0f / ds : 0.0f;
            for (k = 0; k < 16; ++k) {
                float v = row[b * 16 + k] * inv_g;
                v = v * inv_s;
                q[r * K + b * 16 + k] = ds > 0.0f ? metis_oracle_e2m1_encode(v) : (uint8_t)(signbit(row[b * 16 + k]) ? 8 : 0);
            }
        }
    }
    return ORACLE_OK;
}

/* NVFP4 GEMM: y[m, n] = bf16( ga[m] * gb * sum_k V(a)[m, k] * V(b)[n, k] ) with
 * V = D2(q) * D(sb) per 16-element block, float64 sum, one final rounding.
 * ga [M] per token, gb one scale for B (the expert's). */
int metis_oracle_nvfp4_gemm(const uint8_t* qa, const uint8_t* sa, const float* ga,
                            const uint8_t* qb, const uint8_t* sbb, float gb, int64_t M,
                            int64_t N, int64_t K, uint16_t* y, double* y64) {
    int64_t m;
    if (K % 16 != 0) return ORACLE_BAD_INDEX;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        int64_t n, k;
        for (n = 0; n < N; ++n) {
            double acc = 0.0, v;
            for (k = 0; k < K; ++k) {
                double av = metis_oracle_e2m1_decode(qa[m * K + k]) *
                            metis_oracle_e4m3_decode(sa[m * (K / 16) + k / 16]);
                double bv = metis_oracle_e2m1_decode(qb[n * K + k]) *
                            metis_oracle_e4m3_decode(sbb[n * (K / 16) + k / 16]);
                acc += av * bv;
            }
            v = (double)ga[m] * (double)gb * acc;
            y64[m * N + n] = v;
            y[m * N + n] = metis_oracle_bf16_from_double(v);
        }
    }
    return ORACLE_OK;
}

/* Router top-k. The cards keep "the routers and their balance bias" in FP32
 * ("Lernex/Metis-1.6-Logos-FP8", "What is in FP8") and route each token to
 * a few experts; they print no formula. Reading: the balance bias only
 * decides which experts are chosen, and the chosen experts' weights are a
 * softmax over their own (unbiased) logits. Choice j of token t is the j-th
 * largest binary32 score logit + bias (the binary32 sum decides, as the
 * logits are binary32), ties going to the lower expert index; its weight is
 * exp(l_j - m) / sum_i exp(l_i - m) over the chosen experts, m their largest
 * logit, evaluated in float64. bias may be NULL (no bias). */
int metis_oracle_route_topk(const float* logits, const float* bias, int64_t T, int64_t E,
                            int64_t topk, int32_t* ids, double* w) {
    int64_t t;
    if (topk < 1 || topk > E) return ORACLE_BAD_INDEX;
    for (t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        int64_t j, e;
        double m, sum;
        for (j = 0; j < topk; ++j) {
            int64_t best = -1;
            float best_s = 0.0f;
            for (e = 0; e < E; ++e) {
                int64_t i, taken = 0;
                float s;
                for (i = 0; i < j; ++i)
                    if (ids[t * topk + i] == e) taken = 1;
                if (taken) continue;
                s = bias ? l[e] + bias[e] : l[e];
                if (best < 0 || s > best_s) { /* strict: ties keep the lower index */
                    best = e;
                    best_s = s;
                }
            }
            ids[t * topk + j] = (int32_t)best;
        }
        m = l[ids[t * topk]];
        for (j = 1; j < topk; ++j)
            if (l[ids[t * topk + j]] > m) m = l[ids[t * topk + j]];
        sum = 0.0;
        for (j = 0; j < topk; ++j) sum += exp((double)l[ids[t * topk + j]] - m);
        for (j = 0; j < topk; ++j) w[t * topk + j] = exp((double)l[ids[t * topk + j]] - m) / sum;
    }
    return ORACLE_OK;
}

/* Routing-weighted combine: y[t][n] = bf16( sum_j w[t][j] * o[t][j][n] ),
 * o given in slot order as BF16, float64 sum over j in order 0..topk-1. */
int metis_oracle_moe_combine(const uint16_t* o, const float* w, int64_t T, int64_t topk,
                             int64_t H, uint16_t* y, double* y64) {
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        int64_t n, j;
        for (n = 0; n < H; ++n) {
            double acc = 0.0;
            for (j = 0; j < topk; ++j)
                acc += (double)w[t * topk + j] *
                       (double)bf16_bits_to_float(o[(t * topk + j) * H + n]);
            if (y64) y64[t * H + n] = acc;
            y[t * H + n] = metis_oracle_bf16_from_double(acc);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------- shared expert
 * "Lernex/Metis-1.6-Praxis" card, "Architecture": every layer ends in routed
 * experts and one shared expert; the FP8 cards ("What is in FP8") keep the
 * shared expert as trained, in BF16. Reading: the shared expert runs on every
 * token with weight 1 and the same two projections as a routed expert (no
 * activation, h rounded to BF16); the layer output adds its BF16 output to
 * the routed weighted sum before the one final rounding. */

/* y[m, n] = bf16( sum_k x[m, k] w[n, k] ), BF16 operands, float64 sum. */
int metis_oracle_gemm_bf16(const uint16_t* x, int64_t ldx, const uint16_t* w, int64_t ldw,
                           int64_t M, int64_t N, int64_t K, uint16_t* y, double* y64) {
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        int64_t n, k;
        for (n = 0; n < N; ++n) {
            double acc = 0.0;
            for (k = 0; k < K; ++k)
                acc += (double)bf16_bits_to_float(x[m * ldx + k]) *
                       (double)bf16_bits_to_float(w[n * ldw + k]);
            if (y64) y64[m * N + n] = acc;
            y[m * N + n] = metis_oracle_bf16_from_double(acc);
        }
    }
    return ORACLE_OK;
}

/* y[t, n] = bf16( s[t, n] + sum_j w[t, j] o[t, j, n] ), s the shared
 * expert's BF16 output [T, H], o the routed outputs in slot order [T, topk, H]. */
int metis_oracle_shared_combine(const uint16_t* s, const uint16_t* o, const float* w, int64_t T,
                                int64_t topk, int64_t H, uint16_t* y, double* y64) {
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        int64_t n, j;
        for (n = 0; n < H; ++n) {
            double acc = (double)bf16_bits_to_float(s[t * H + n]);
            for (j = 0; j < topk; ++j)
                acc += (double)w[t * topk + j] *
                       (double)bf16_bits_to_float(o[(t * topk + j) * H + n]);
            if (y64) y64[t * H + n] = acc;
            y[t * H + n] = metis_oracle_bf16_from_double(acc);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------- array forms of the codec */

void metis_oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = metis_oracle_e4m3_encode(v[i]);
}

void metis_oracle_e4m3_decode_array(const uint8_t* b, int64_t n, double* out) {
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = metis_oracle_e4m3_decode(b[i]);
}

void metis_oracle_bf16_from_double_array(const double* v, int64_t n, uint16_t* out) {
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = metis_oracle_bf16_from_double(v[i]);
}
