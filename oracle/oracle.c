/*
 * oracle.c -- plain, slow CPU oracle for the quantized W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links, loads or
 * calls this file; only the tests, the package's smoke check and the bench's
 * CPU-baseline leg do. It shares no code with the CUDA path.
 *
 * What it computes, and where each definition comes from:
 *   - LLM.int8 mixed-precision decomposition with outlier threshold 6.0, the
 *     outlier part in floating point: Image21-INT8 page, section
 *     "Quantization".
 *   - vector-wise int8 (per-token absmax / 127 for activations, per-output-
 *     channel absmax / 127 for weights, int32 accumulation, dequant by the
 *     outer product of the two scale vectors): the bitsandbytes LLM.int8
 *     scheme the same page names; the formula is the plainest reading
 *     (absmax / QMAX, multiply by the reciprocal, round half to even).
 *   - FP8 E4M3 W8A8 with static per-tensor fp32 weight_scale and
 *     input_scale: Darkstar ModelOpt-FP8 page, "Precision map"; the scales
 *     come from max calibration ("Provenance").
 *   - FP8 E4M3 weights with one bf16 scale per output channel ([out,1]) and
 *     dynamic per-token FP8 activations: Text-Encoder-FP8 page, "Format".
 *   - weight dequant weight.to(bf16) * weight_scale: Text-Encoder-FP8 page,
 *     "Format"; the ModelOpt-FP8 page, "Consumption", states the same.
 *   - E4M3 has a 3-bit mantissa: Text-Encoder-FP8 page, "How it was tested".
 *     The OCP e4m3fn layout (bias 7, no infinities, max 448) is the reading.
 *   - int4 per-group weights with int8 activations and fp32 scales:
 *     Qwen-Image-fni8 page, "Format". Group size 128 is the workload's.
 *
 * Arithmetic conventions (the pages fix none of them; these are the
 * readings):
 *   - inputs (fp16 / bf16) are widened exactly to fp32;
 *   - a scale is s = absmax / QMAX (one IEEE fp32 division), its reciprocal
 *     inv = 1 / s (one IEEE fp32 division) and the scaled value t = v * inv
 *     (one fp32 multiply); all quantisation decisions are taken in fp32, the
 *     precision the CUDA kernels take them in;
 *   - a zero input maps to a zero code even when inv overflows (0 * inf is
 *     never formed); absmax == 0 gives s = 0 and all-zero codes;
 *   - int8 codes: round half to even, clamp to [-127, 127]; int4: [-7, 7];
 *   - e4m3 codes: round to nearest even in the e4m3 grid, saturating to
 *     +-448 (a negative value that rounds to zero keeps its sign: 0x80);
 *   - contractions and dequantised outputs are formed in fp64 (int8 sums are
 *     formed in int64 and checked to fit int32).
 *
 * Every function that writes an output array takes a nullable pointer: pass
 * NULL to skip that output. Sizes are int64_t; arrays are row-major.
 * Compiled with -O2 -ffp-contract=off so that no fp32 multiply is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_F16 0
#define ORC_BF16 1

/* ------------------------------------------------------------------ */
/* Scalar formats, written from their bit-level definitions.           */
/* ------------------------------------------------------------------ */

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_to_double(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m | 0x400), e - 25);
    return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double orc_bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double widen(uint16_t h, int dt) {
    return dt == ORC_BF16 ? orc_bf16_to_double(h) : orc_f16_to_double(h);
}

/* Round x to the nearest number with p significant bits whose exponent is
 * at least emin (below it the quantum is fixed: the subnormal range); ties
 * go to the even neighbour. x / quantum is exact (a power-of-two scaling),
 * and nearbyint rounds half to even in the default rounding mode. Overflow
 * is left to the caller. */
static double round_to_grid(double x, int p, int emin) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(fabs(x), &e);               /* |x| = f * 2^e, f in [0.5, 1) */
    int lead = e - 1;                 /* exponent of the leading bit */
    if (lead < emin) lead = emin;
    double quantum = ldexp(1.0, lead - (p - 1));
    return nearbyint(x / quantum) * quantum;
}

/* double -> bfloat16 bits, round to nearest even (8 significant bits,
 * emin -126, max finite (2 - 2^-7) * 2^127, overflow -> inf). */
uint16_t orc_double_to_bf16(double x) {
    if (isnan(x)) return 0x7fc0;
    double r = round_to_grid(x, 8, -126);
    float f = (float)r;               /* exact: r has 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* double -> binary16 bits, round to nearest even (11 significant bits,
 * emin -14, max finite 65504, overflow -> inf). */
uint16_t orc_double_to_f16(double x) {
    if (isnan(x)) return 0x7e00;
    double r = round_to_grid(x, 11, -14);
    uint16_t s = signbit(r) ? 0x8000 : 0;
    double a = fabs(r);
    if (a > 65504.0) return s | 0x7c00;
    if (a == 0.0) return s;
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < -14) {                 /* subnormal: a = m * 2^-24 */
        return s | (uint16_t)(a / ldexp(1.0, -24));
    }
    uint16_t m = (uint16_t)(a / ldexp(1.0, lead - 10)) - 0x400;
    return s | (uint16_t)((lead + 15) << 10) | m;
}

static uint16_t narrow(double x, int dt) {
    return dt == ORC_BF16 ? orc_double_to_bf16(x) : orc_double_to_f16(x);
}

/* E4M3 (OCP e4m3fn): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; max finite S.1111.110 = 448; subnormals
 * m * 2^-9. */
double orc_e4m3_decode(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 0xf, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return s ? -v : v;
}

/* fp32 -> E4M3 code: round to nearest even on the e4m3 grid (4 significant
 * bits, emin -6), then saturate to +-448 (satfinite). NaN -> 0x7f. */
uint8_t orc_e4m3_encode(float t) {
    if (isnan(t)) return 0x7f;
    double r = round_to_grid((double)t, 4, -6);
    uint8_t s = signbit(r) ? 0x80 : 0;
    double a = fabs(r);
    if (a > 448.0) a = 448.0;         /* also catches +-inf */
    if (a == 0.0) return s;
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < -6) return s | (uint8_t)(a / ldexp(1.0, -9));
    uint8_t m = (uint8_t)(a / ldexp(1.0, lead - 3)) - 8;
    return s | (uint8_t)((lead + 7) << 3) | m;
}

/* A second, independent E4M3 encoder used only to pin the first: search
 * the 127 non-negative finite code values for the nearest one; on a tie
 * take the code with an even mantissa; above 448 saturate. */
uint8_t orc_e4m3_encode_search(float t) {
    if (isnan(t)) return 0x7f;
    double a = fabs((double)t);
    uint8_t sign = signbit(t) ? 0x80 : 0;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        double d = fabs(orc_e4m3_decode((uint8_t)c) - a);
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    if (a >= 448.0) best = 0x7e;
    return sign | (uint8_t)best;
}

/* A third E4M3 encoder, integer arithmetic on the fp32 bit fields (round
 * to nearest even by shifting the 24-bit significand with a round bit and a
 * sticky bit), used only to pin orc_e4m3_encode over all 2^32 inputs. */
static uint32_t rne_shift(uint32_t x, int s) {
    if (s <= 0) return x;
    if (s > 31) return 0;
    uint32_t q = x >> s;
    uint32_t r = (x >> (s - 1)) & 1u;
    uint32_t sticky = x & ((1u << (s - 1)) - 1u);
    if (r && (sticky || (q & 1u))) ++q;
    return q;
}

uint8_t orc_e4m3_encode_bits(float t) {
    uint32_t u;
    memcpy(&u, &t, 4);
    const uint8_t sign = (uint8_t)((u >> 24) & 0x80u);
    const uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) return 0x7f;           /* NaN */
    if (a >= 0x7f800000u) return sign | 0x7e;   /* +-inf saturates */
    const int E = (int)(a >> 23) - 127;         /* fp32 subnormals have E = -127 */
    const uint32_t sig = (a >> 23) ? ((a & 0x7fffffu) | 0x800000u) : (a & 0x7fffffu);
    if (E > 8) return sign | 0x7e;
    if (E < -6) {
        /* e4m3 subnormal: the code is round(|t| / 2^-9), |t| = sig * 2^(E - 23) */
        const int sh = (E == -127) ? 23 + 126 - 9 : 23 - (E + 9);
        const uint32_t q = rne_shift(sig, sh);   /* 0..8; 8 is the smallest normal, code 0x08 */
        return sign | (uint8_t)q;
    }
    uint32_t q = rne_shift(sig, 20);            /* 4 significant bits: 8..16 */
    int e = E;
    if (q == 16u) { q = 8u; ++e; }
    const int field = e + 7;
    if (field > 15 || (field == 15 && q - 8u == 7u)) return sign | 0x7e;   /* above 448 */
    return sign | (uint8_t)((field << 3) | (int)(q - 8u));
}

/* Mismatches between orc_e4m3_encode and orc_e4m3_encode_bits over the fp32
 * bit patterns [lo, lo + count). */
int64_t orc_e4m3_compare_encoders(uint64_t lo, uint64_t count) {
    int64_t bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        const uint32_t bits = (uint32_t)(lo + (uint64_t)i);
        float t;
        memcpy(&t, &bits, 4);
        if (orc_e4m3_encode(t) != orc_e4m3_encode_bits(t)) ++bad;
    }
    return bad;
}

/* codes[i] = orc_e4m3_encode(float with bit pattern lo + i), i < count. */
void orc_e4m3_encode_range(uint64_t lo, uint64_t count, uint8_t *codes) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        const uint32_t bits = (uint32_t)(lo + (uint64_t)i);
        float t;
        memcpy(&t, &bits, 4);
        codes[i] = orc_e4m3_encode(t);
    }
}

/* ------------------------------------------------------------------ */
/* Quantiser Q(v, s): s = absmax / QMAX, inv = 1 / s, t = v * inv.     */
/* ------------------------------------------------------------------ */

static float scale_of(float absmax, float qmax) { return absmax / qmax; }

static float recip(float s) { return 1.0f / s; }

/* integer code: round half to even, clamp to [-qmax, qmax] */
static int q_int(float v, float inv, int qmax) {
    if (v == 0.0f) return 0;
    float t = v * inv;
    if (isnan(t)) return 0;
    if (t >= (float)qmax) return qmax;
    if (t <= -(float)qmax) return -qmax;
    return (int)nearbyintf(t);
}

int orc_q_int8(float v, float inv) { return q_int(v, inv, 127); }
int orc_q_int4(float v, float inv) { return q_int(v, inv, 7); }

uint8_t orc_q_e4m3(float v, float inv) {
    float t = (v == 0.0f) ? v : v * inv;
    return orc_e4m3_encode(t);
}

float orc_int8_scale(float absmax) { return scale_of(absmax, 127.0f); }
float orc_e4m3_scale(float absmax) { return scale_of(absmax, 448.0f); }
float orc_recip(float s) { return recip(s); }

static float *widen_all(const uint16_t *X, int dt, int64_t n) {
    float *f = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) f[i] = (float)widen(X[i], dt);
    return f;
}

static float absmax_range(const float *v, int64_t n) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > m) m = a;
    }
    return m;
}

/* ------------------------------------------------------------------ */
/* Offline weight quantisation and calibration.                        */
/* ------------------------------------------------------------------ */

/* Max calibration: absmax over a tensor / qmax (fp32). */
float orc_absmax_scale(const uint16_t *X, int dt, int64_t n, float qmax) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf((float)widen(X[i], dt));
        if (a > m) m = a;
    }
    return scale_of(m, qmax);
}

/* int8, one scale per output channel: s_w[j] = absmax_k |W[j,k]| / 127. */
void orc_quantize_weight_int8(const uint16_t *W, int dt, int64_t N, int64_t K,
                              int8_t *Wq, float *s_w) {
    float *w = widen_all(W, dt, N * K);
    for (int64_t j = 0; j < N; ++j) {
        float s = scale_of(absmax_range(w + j * K, K), 127.0f);
        float inv = recip(s);
        s_w[j] = s;
        for (int64_t k = 0; k < K; ++k)
            Wq[j * K + k] = (int8_t)(s == 0.0f ? 0 : q_int(w[j * K + k], inv, 127));
    }
    free(w);
}

/* FP8 E4M3, one fp32 scale per tensor: s = absmax(W) / 448. */
void orc_quantize_weight_fp8_tensor(const uint16_t *W, int dt, int64_t N, int64_t K,
                                    uint8_t *Wq, float *s_out) {
    float *w = widen_all(W, dt, N * K);
    float s = scale_of(absmax_range(w, N * K), 448.0f);
    float inv = recip(s);
    *s_out = s;
    for (int64_t i = 0; i < N * K; ++i) Wq[i] = s == 0.0f ? 0 : orc_q_e4m3(w[i], inv);
    free(w);
}

/* FP8 E4M3, one bf16 scale per output channel (shape [out,1]):
 * s_w[j] = bf16(absmax_j / 448); the codes divide by that stored bf16
 * value so that weight.to(bf16) * weight_scale reproduces W. */
void orc_quantize_weight_fp8_channel(const uint16_t *W, int dt, int64_t N, int64_t K,
                                     uint8_t *Wq, uint16_t *s_bf16) {
    float *w = widen_all(W, dt, N * K);
    for (int64_t j = 0; j < N; ++j) {
        float s32 = scale_of(absmax_range(w + j * K, K), 448.0f);
        uint16_t sb = orc_double_to_bf16((double)s32);
        float s = (float)orc_bf16_to_double(sb);
        float inv = recip(s);
        s_bf16[j] = sb;
        for (int64_t k = 0; k < K; ++k)
            Wq[j * K + k] = s == 0.0f ? 0 : orc_q_e4m3(w[j * K + k], inv);
    }
    free(w);
}

/* int4, symmetric, one fp32 scale per (output channel, group of G along K):
 * s = absmax_group / 7, codes in [-7, 7]. Packing (the page fixes no byte
 * layout): each row is cut into blocks of 32 consecutive k stored in 16
 * bytes; byte b of a block holds its element b in the low nibble and its
 * element b + 16 in the high nibble, two's complement. K % 32 == 0. */
void orc_quantize_weight_int4(const uint16_t *W, int dt, int64_t N, int64_t K, int64_t G,
                              uint8_t *Wq4, float *s_w) {
    float *w = widen_all(W, dt, N * K);
    int64_t ng = K / G;
    for (int64_t j = 0; j < N; ++j) {
        for (int64_t g = 0; g < ng; ++g) {
            const float *wg = w + j * K + g * G;
            float s = scale_of(absmax_range(wg, G), 7.0f);
            float inv = recip(s);
            s_w[j * ng + g] = s;
            for (int64_t k = 0; k < G; ++k) {
                int q = s == 0.0f ? 0 : q_int(wg[k], inv, 7);
                int64_t kk = g * G + k;
                int64_t e = kk % 32;   /* position in its block of 32 */
                uint8_t *b = Wq4 + j * (K / 2) + (kk / 32) * 16 + e % 16;
                if (e < 16) *b = (uint8_t)((*b & 0xf0) | (q & 0xf));
                else *b = (uint8_t)((*b & 0x0f) | ((q & 0xf) << 4));
            }
        }
    }
    free(w);
}

static int int4_at(const uint8_t *Wq4, int64_t K, int64_t j, int64_t k) {
    int64_t e = k % 32;
    uint8_t b = Wq4[j * (K / 2) + (k / 32) * 16 + e % 16];
    int nib = e >= 16 ? (b >> 4) : (b & 0xf);
    return nib >= 8 ? nib - 16 : nib;
}

int orc_int4_unpack(const uint8_t *Wq4, int64_t K, int64_t j, int64_t k) {
    return int4_at(Wq4, K, j, k);
}

/* ------------------------------------------------------------------ */
/* LLM.int8 mixed-precision decomposition.                             */
/* ------------------------------------------------------------------ */

/* Decomposition is off when the threshold is <= 0 or +inf. */
static int decomposition_on(float thr) { return thr > 0.0f && !isinf(thr); }

/* Activation side of LLM.int8 for all M rows:
 *   O       = { k : exists i with |X[i,k]| > thr }, ascending;
 *   s_x[i]  = absmax over k not in O of |X[i,k]|, / 127;
 *   Xq[i,k] = 0 for k in O, else clamp(rne(X[i,k] / s_x[i]), +-127);
 *   X_O[i,o]= X[i, O[o]] (an exact copy), stored with row stride ostride.
 * Outputs are nullable. */
void orc_int8_outlier_prep(const uint16_t *X, int dt, int64_t M, int64_t K, float thr,
                           int8_t *Xq, float *s_x, uint8_t *is_outlier, int32_t *O,
                           int32_t *count, uint16_t *X_O, int64_t ostride) {
    float *x = widen_all(X, dt, M * K);
    uint8_t *flag = (uint8_t *)calloc((size_t)(K > 0 ? K : 1), 1);
    if (decomposition_on(thr)) {
        for (int64_t i = 0; i < M; ++i)
            for (int64_t k = 0; k < K; ++k)
                if (fabsf(x[i * K + k]) > thr) flag[k] = 1;
    }
    int32_t n = 0;
    for (int64_t k = 0; k < K; ++k) {
        if (flag[k]) {
            if (O) O[n] = (int32_t)k;
            ++n;
        }
    }
    if (count) *count = n;
    if (is_outlier) memcpy(is_outlier, flag, (size_t)K);
    for (int64_t i = 0; i < M; ++i) {
        const float *row = x + i * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            if (!flag[k] && fabsf(row[k]) > amax) amax = fabsf(row[k]);
        float s = scale_of(amax, 127.0f);
        float inv = recip(s);
        if (s_x) s_x[i] = s;
        if (Xq)
            for (int64_t k = 0; k < K; ++k)
                Xq[i * K + k] = (int8_t)((flag[k] || s == 0.0f) ? 0 : q_int(row[k], inv, 127));
        if (X_O) {
            int32_t o = 0;
            for (int64_t k = 0; k < K; ++k)
                if (flag[k]) X_O[i * ostride + (o++)] = X[i * K + k];
        }
    }
    free(flag);
    free(x);
}

/* Dequantised weight columns for the floating-point outlier part, by the
 * weight.to(dtype) * weight_scale rule: W_O[j,o] = dtype(fp32(Wq[j,O[o]]) *
 * s_w[j]), one fp32 multiply, then rounded to the activation dtype. */
void orc_outlier_weights(const int8_t *Wq, const float *s_w, int64_t N, int64_t K,
                         const int32_t *O, int32_t count, int dt, uint16_t *W_O, int64_t ostride) {
    for (int64_t j = 0; j < N; ++j)
        for (int32_t o = 0; o < count; ++o) {
            float p = (float)Wq[j * K + O[o]] * s_w[j];
            W_O[j * ostride + o] = narrow((double)p, dt);
        }
}

/* Full LLM.int8 linear for the rows listed in `rows` (all rows if NULL):
 *   C[r,j]   = sum_k Xq[i,k] * Wq[j,k]            (int64, checked to fit int32)
 *   F[r,j]   = sum_o X_O[i,o] * W_O[j,o]          (fp64; the floating-point part)
 *   Y64[r,j] = C * s_x[i] * s_w[j] + F + bias[j]  (fp64, before rounding)
 *   Y[r,j]   = Y64 rounded to the activation dtype.
 * The outlier set and the row scales are always taken over all M rows: the
 * outlier test is per call, over every token of the call.
 * Returns 0, or -1 if some |C| does not fit int32. */
int orc_int8_outlier_forward(const uint16_t *X, int dt, int64_t M, int64_t K,
                             const int8_t *Wq, const float *s_w, int64_t N, float thr,
                             const uint16_t *bias, const int64_t *rows, int64_t nrows,
                             int32_t *C, double *Y64, uint16_t *Y) {
    int8_t *Xq = (int8_t *)malloc((size_t)(M * K > 0 ? M * K : 1));
    float *s_x = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
    int32_t *O = (int32_t *)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
    int32_t cnt = 0;
    int64_t ostr = K > 0 ? K : 1;
    uint16_t *X_O = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(M * ostr > 0 ? M * ostr : 1));
    uint16_t *W_O = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(N * ostr > 0 ? N * ostr : 1));
    orc_int8_outlier_prep(X, dt, M, K, thr, Xq, s_x, NULL, O, &cnt, X_O, ostr);
    orc_outlier_weights(Wq, s_w, N, K, O, cnt, dt, W_O, ostr);
    if (!rows) nrows = M;
    int overflow = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : overflow)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            int64_t c = 0;
            for (int64_t k = 0; k < K; ++k) c += (int64_t)Xq[i * K + k] * (int64_t)Wq[j * K + k];
            if (c > INT32_MAX || c < INT32_MIN) overflow = 1;
            double f = 0.0;
            for (int32_t o = 0; o < cnt; ++o)
                f += widen(X_O[i * ostr + o], dt) * widen(W_O[j * ostr + o], dt);
            double y = (double)c * (double)s_x[i] * (double)s_w[j] + f;
            if (bias) y += widen(bias[j], dt);
            if (C) C[r * N + j] = (int32_t)c;
            if (Y64) Y64[r * N + j] = y;
            if (Y) Y[r * N + j] = narrow(y, dt);
        }
    }
    free(Xq);
    free(s_x);
    free(O);
    free(X_O);
    free(W_O);
    return overflow ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 W8A8.                                                      */
/* ------------------------------------------------------------------ */

/* Static per-tensor activation codes: Xq = e4m3(X * (1 / input_scale)). */
void orc_fp8_static_prep(const uint16_t *X, int dt, int64_t M, int64_t K, float input_scale,
                         uint8_t *Xq) {
    float inv = recip(input_scale);
    for (int64_t i = 0; i < M * K; ++i) {
        float v = (float)widen(X[i], dt);
        Xq[i] = input_scale == 0.0f ? 0 : orc_q_e4m3(v, inv);
    }
}

/* Dynamic per-token activation codes: s_x[i] = absmax_i / 448,
 * Xq[i,k] = e4m3(X[i,k] * (1 / s_x[i])). */
void orc_fp8_dynamic_prep(const uint16_t *X, int dt, int64_t M, int64_t K, uint8_t *Xq,
                          float *s_x) {
    float *x = widen_all(X, dt, M * K);
    for (int64_t i = 0; i < M; ++i) {
        float s = scale_of(absmax_range(x + i * K, K), 448.0f);
        float inv = recip(s);
        if (s_x) s_x[i] = s;
        for (int64_t k = 0; k < K; ++k)
            Xq[i * K + k] = s == 0.0f ? 0 : orc_q_e4m3(x[i * K + k], inv);
    }
    free(x);
}

/* FP8 linear over the listed rows. acc = sum_k dec(Xq[i,k]) * dec(Wq[j,k])
 * is exact in fp64 (each product has at most 8 significant bits and the
 * sum stays below 2^49 ulps). Then
 *   static:  Y64 = acc * input_scale * weight_scale + bias
 *   dynamic: Y64 = acc * s_x[i] * float(bf16 s_w[j]) + bias
 * x_scale_static < 0 selects the dynamic per-token mode; w_scale_bf16 != NULL
 * selects per-channel bf16 weight scales, else w_scale_tensor is used. */
void orc_fp8_forward(const uint16_t *X, int dt, int64_t M, int64_t K, const uint8_t *Wq,
                     float w_scale_tensor, const uint16_t *w_scale_bf16, int64_t N,
                     float x_scale_static, const uint16_t *bias, const int64_t *rows,
                     int64_t nrows, uint8_t *Xq_out, float *s_x_out, double *acc_out,
                     double *Y64, uint16_t *Y) {
    uint8_t *Xq = (uint8_t *)malloc((size_t)(M * K > 0 ? M * K : 1));
    float *s_x = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
    int dynamic = x_scale_static < 0.0f;
    if (dynamic) orc_fp8_dynamic_prep(X, dt, M, K, Xq, s_x);
    else {
        orc_fp8_static_prep(X, dt, M, K, x_scale_static, Xq);
        for (int64_t i = 0; i < M; ++i) s_x[i] = x_scale_static;
    }
    if (Xq_out) memcpy(Xq_out, Xq, (size_t)(M * K));
    if (s_x_out) memcpy(s_x_out, s_x, sizeof(float) * (size_t)M);
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += orc_e4m3_decode(Xq[i * K + k]) * orc_e4m3_decode(Wq[j * K + k]);
            double sw = w_scale_bf16 ? orc_bf16_to_double(w_scale_bf16[j]) : (double)w_scale_tensor;
            double y = acc * (double)s_x[i] * sw;
            if (bias) y += widen(bias[j], dt);
            if (acc_out) acc_out[r * N + j] = acc;
            if (Y64) Y64[r * N + j] = y;
            if (Y) Y[r * N + j] = narrow(y, dt);
        }
    }
    free(Xq);
    free(s_x);
}

/* ------------------------------------------------------------------ */
/* Weight-only FP8 (Qwen-Image-2.1-Text-Encoder-FP8, section "Format":  */
/* E4M3 weights with a bf16 scale per output channel, [out,1], and the  */
/* dequant rule weight.to(bf16) * weight_scale; the activations stay    */
/* in their 16-bit dtype).                                              */
/* ------------------------------------------------------------------ */

/* W_deq[j,k] = bf16(decode(Wq[j,k]) * s_w[j]): the e4m3 value widens to
 * bf16 exactly (3 mantissa bits), the bf16 x bf16 product is exact in
 * double, and the bf16 multiply rounds it once, to nearest even. */
void orc_fp8_weight_only_dequant(const uint8_t *Wq, const uint16_t *s_w_bf16, int64_t N, int64_t K,
                                 uint16_t *W_deq) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
        double s = orc_bf16_to_double(s_w_bf16[j]);
        for (int64_t k = 0; k < K; ++k) W_deq[j * K + k] = orc_double_to_bf16(orc_e4m3_decode(Wq[j * K + k]) * s);
    }
}

/* Y64[i,j] = sum_k X[i,k] * W_deq[j,k] + bias[j] in double (each product of
 * two 16-bit values is exact); Y = Y64 rounded once to the activation dtype.
 * W_deq is bf16 and X is bf16 or fp16, as the page's rule leaves them. */
void orc_fp8_weight_only_forward(const uint16_t *X, int dt, int64_t M, int64_t K, const uint8_t *Wq,
                                 const uint16_t *s_w_bf16, int64_t N, const uint16_t *bias,
                                 const int64_t *rows, int64_t nrows, double *Y64, uint16_t *Y) {
    uint16_t *Wd = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(N * K > 0 ? N * K : 1));
    orc_fp8_weight_only_dequant(Wq, s_w_bf16, N, K, Wd);
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += widen(X[i * K + k], dt) * orc_bf16_to_double(Wd[j * K + k]);
            if (bias) acc += widen(bias[j], dt);
            if (Y64) Y64[r * N + j] = acc;
            if (Y) Y[r * N + j] = narrow(acc, dt);
        }
    }
    free(Wd);
}

/* ------------------------------------------------------------------ */
/* Unquantised 16-bit linear: the layers kept in fp16 because they write */
/* or cancel massive activations (Image21-Turbo-OrbitQuant-W4A4,        */
/* section "What 4-bit breaks here and what stays in fp16").            */
/* ------------------------------------------------------------------ */

/* Y64[i,j] = sum_k X[i,k] * W[j,k] + bias[j] in double (each product of two
 * 16-bit values is exact); Y = Y64 rounded once to the dtype of X and W. */
void orc_fp_linear_forward(const uint16_t *X, int dt, int64_t M, int64_t K, const uint16_t *W, int64_t N,
                           const uint16_t *bias, const int64_t *rows, int64_t nrows, double *Y64, uint16_t *Y) {
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += widen(X[i * K + k], dt) * widen(W[j * K + k], dt);
            if (bias) acc += widen(bias[j], dt);
            if (Y64) Y64[r * N + j] = acc;
            if (Y) Y[r * N + j] = narrow(acc, dt);
        }
    }
}

/* ------------------------------------------------------------------ */
/* W4A8: int4 per-group weights, int8 per-token activations.           */
/* ------------------------------------------------------------------ */

/* Activations: per-token int8 over all K (no outlier split), i.e. the
 * vector-wise int8 row quantiser. Per group g of G columns:
 *   C_g[i,j] = sum_{k in g} Xq[i,k] * Wq4[j,k]  (int32)
 *   Y64[i,j] = s_x[i] * sum_g s_w[j,g] * C_g[i,j] + bias[j]. */
void orc_w4a8_forward(const uint16_t *X, int dt, int64_t M, int64_t K, const uint8_t *Wq4,
                      const float *s_w, int64_t N, int64_t G, const uint16_t *bias,
                      const int64_t *rows, int64_t nrows, int8_t *Xq_out, float *s_x_out,
                      int32_t *Cg, double *Y64, uint16_t *Y) {
    int8_t *Xq = (int8_t *)malloc((size_t)(M * K > 0 ? M * K : 1));
    float *s_x = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
    orc_int8_outlier_prep(X, dt, M, K, 0.0f, Xq, s_x, NULL, NULL, NULL, NULL, 0);
    if (Xq_out) memcpy(Xq_out, Xq, (size_t)(M * K));
    if (s_x_out) memcpy(s_x_out, s_x, sizeof(float) * (size_t)M);
    int64_t ng = K / G;
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t g = 0; g < ng; ++g) {
                int64_t c = 0;
                for (int64_t k = g * G; k < (g + 1) * G; ++k)
                    c += (int64_t)Xq[i * K + k] * (int64_t)int4_at(Wq4, K, j, k);
                if (Cg) Cg[(r * N + j) * ng + g] = (int32_t)c;
                acc += (double)s_w[j * ng + g] * (double)c;
            }
            double y = (double)s_x[i] * acc;
            if (bias) y += widen(bias[j], dt);
            if (Y64) Y64[r * N + j] = y;
            if (Y) Y[r * N + j] = narrow(y, dt);
        }
    }
    free(Xq);
    free(s_x);
}

/* ------------------------------------------------------------------ */
/* Block-scaled int8 weights (Qwen-Image-2.1-Text-Encoder-FP8, section  */
/* "How it was tested", where GGUF Q8_0 is compared: int8 codes, one    */
/* scale for each run of 32 weights). The page fixes only the block of  */
/* 32 along a weight row and the 8-bit codes; the scale and code rules  */
/* are the quantiser Q above (s = absmax_block / 127, fp32), and the    */
/* activations take the W4A8 mode's per-token int8 rows.                */
/* ------------------------------------------------------------------ */

/* One fp32 scale per (output channel j, block b of B consecutive k):
 * s_w[j,b] = absmax_{k in b} |W[j,k]| / 127, Wq[j,k] = Q(W[j,k], s_w[j,b]). */
void orc_quantize_weight_int8_block(const uint16_t *W, int dt, int64_t N, int64_t K, int64_t B,
                                    int8_t *Wq, float *s_w) {
    float *w = widen_all(W, dt, N * K);
    int64_t nb = K / B;
    for (int64_t j = 0; j < N; ++j) {
        for (int64_t b = 0; b < nb; ++b) {
            const float *wb = w + j * K + b * B;
            float s = scale_of(absmax_range(wb, B), 127.0f);
            float inv = recip(s);
            s_w[j * nb + b] = s;
            for (int64_t k = 0; k < B; ++k) Wq[j * K + b * B + k] = (int8_t)(s == 0.0f ? 0 : q_int(wb[k], inv, 127));
        }
    }
    free(w);
}

/* Per block b of B columns:
 *   C_b[i,j] = sum_{k in b} Xq[i,k] * Wq[j,k]  (int32)
 *   Y64[i,j] = s_x[i] * sum_b s_w[j,b] * C_b[i,j] + bias[j],
 * with Xq, s_x the per-token int8 rows over all K. */
void orc_int8_block_forward(const uint16_t *X, int dt, int64_t M, int64_t K, const int8_t *Wq,
                            const float *s_w, int64_t N, int64_t B, const uint16_t *bias,
                            const int64_t *rows, int64_t nrows, int8_t *Xq_out, float *s_x_out,
                            int32_t *Cb, double *Y64, uint16_t *Y) {
    int8_t *Xq = (int8_t *)malloc((size_t)(M * K > 0 ? M * K : 1));
    float *s_x = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
    orc_int8_outlier_prep(X, dt, M, K, 0.0f, Xq, s_x, NULL, NULL, NULL, NULL, 0);
    if (Xq_out) memcpy(Xq_out, Xq, (size_t)(M * K));
    if (s_x_out) memcpy(s_x_out, s_x, sizeof(float) * (size_t)M);
    int64_t nb = K / B;
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t b = 0; b < nb; ++b) {
                int64_t c = 0;
                for (int64_t k = b * B; k < (b + 1) * B; ++k) c += (int64_t)Xq[i * K + k] * (int64_t)Wq[j * K + k];
                if (Cb) Cb[(r * N + j) * nb + b] = (int32_t)c;
                acc += (double)s_w[j * nb + b] * (double)c;
            }
            double y = (double)s_x[i] * acc;
            if (bias) y += widen(bias[j], dt);
            if (Y64) Y64[r * N + j] = y;
            if (Y) Y[r * N + j] = narrow(y, dt);
        }
    }
    free(Xq);
    free(s_x);
}

/* ------------------------------------------------------------------ */
/* NVFP4 weights, 16-bit activations. The Darkstar pages name NVFP4 as */
/* the family's primary release format and give no layout; this is the */
/* plainest reading of the name: E2M1 codes, one E4M3 scale per 16     */
/* consecutive weights of a row, one fp32 scale per tensor.            */
/* ------------------------------------------------------------------ */

/* E2M1: sign bit 3, 2 exponent bits (bias 1), 1 mantissa bit, no inf or
 * NaN. Exponent 0 is subnormal: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double orc_e2m1_decode(uint8_t c) {
    int e = (c >> 1) & 3, m = c & 1;
    double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (c & 8) ? -mag : mag;
}

/* Nearest E2M1 value, ties to the even mantissa bit, saturating at 6; the
 * sign of t (also of -0) goes to bit 3. Found by searching the 8
 * magnitudes. */
uint8_t orc_e2m1_encode(float t) {
    uint8_t sign = signbit(t) ? 8 : 0;
    double a = fabs((double)t);
    if (a >= 6.0) return sign | 7;   /* saturation (far above 6 the distances to 4 and 6 round equal) */
    uint8_t best = 0;
    double bd = INFINITY;
    for (uint8_t c = 0; c < 8; ++c) {
        double d = fabs(orc_e2m1_decode(c) - a);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return sign | best;
}

/* W [N,K] (K % 32 == 0) -> codes Wq [N,K/2] packed like the int4 format
 * (each block of 32 k in 16 bytes, byte b holding element b in its low
 * nibble and element b + 16 in its high nibble), block scales s_b e4m3
 * [N,K/16], tensor scale s_t:
 *   s_t  = absmax(W) / 2688                  (2688 = 6 * 448)
 *   s_b  = e4m3(absmax(block) / (6 * s_t))   (rne, saturating at 448; 0 if s_t == 0)
 *   code = e2m1(w / (decode(s_b) * s_t))     (0 where that divisor is 0)
 * each division and product one IEEE fp32 operation. */
void orc_quantize_weight_nvfp4(const uint16_t *W, int dt, int64_t N, int64_t K, uint8_t *Wq, uint8_t *s_b,
                               float *s_t) {
    float *w = widen_all(W, dt, N * K);
    const float st = absmax_range(w, N * K) / 2688.0f;
    const float six_st = 6.0f * st;
    *s_t = st;
    memset(Wq, 0, (size_t)(N * K / 2));
    for (int64_t j = 0; j < N; ++j) {
        for (int64_t b = 0; b < K / 16; ++b) {
            const float *wb = w + j * K + b * 16;
            const uint8_t sc = six_st == 0.0f ? 0 : orc_e4m3_encode(absmax_range(wb, 16) / six_st);
            s_b[j * (K / 16) + b] = sc;
            const float d = (float)orc_e4m3_decode(sc) * st;
            for (int64_t e = 0; e < 16; ++e) {
                const int64_t k = b * 16 + e;
                const uint8_t c = d == 0.0f ? 0 : orc_e2m1_encode(wb[e] / d);
                const int64_t pos = k % 32;
                uint8_t *byte = Wq + j * (K / 2) + (k / 32) * 16 + pos % 16;
                if (pos < 16) *byte = (uint8_t)((*byte & 0xf0) | (c & 0xf));
                else *byte = (uint8_t)((*byte & 0x0f) | ((c & 0xf) << 4));
            }
        }
    }
    free(w);
}

/* The E2M1 code of weight (j, k) in the packed layout above. */
uint8_t orc_nvfp4_code(const uint8_t *Wq, int64_t K, int64_t j, int64_t k) {
    const int64_t pos = k % 32;
    const uint8_t byte = Wq[j * (K / 2) + (k / 32) * 16 + pos % 16];
    return pos < 16 ? (byte & 0xf) : (byte >> 4);
}

/* Y64[i,j] = s_t * sum_k X[i,k] * decode(code[j,k]) * decode(s_b[j,k/16]) + bias[j]
 * in double (each product exact); Y = Y64 rounded once to the dtype of X. */
void orc_nvfp4_weight_only_forward(const uint16_t *X, int dt, int64_t M, int64_t K, const uint8_t *Wq,
                                   const uint8_t *s_b, float s_t, int64_t N, const uint16_t *bias,
                                   const int64_t *rows, int64_t nrows, double *Y64, uint16_t *Y) {
    double *Wd = (double *)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k)
            Wd[j * K + k] = orc_e2m1_decode(orc_nvfp4_code(Wq, K, j, k)) * orc_e4m3_decode(s_b[j * (K / 16) + k / 16]);
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += widen(X[i * K + k], dt) * Wd[j * K + k];
            acc *= (double)s_t;
            if (bias) acc += widen(bias[j], dt);
            if (Y64) Y64[r * N + j] = acc;
            if (Y) Y[r * N + j] = narrow(acc, dt);
        }
    }
    free(Wd);
}

/* NVFP4 activations and weights (W4A4; the next step of the NVFP4 reading):
 * X [M,K] is quantised per call exactly like a weight (orc_quantize_weight_nvfp4
 * applied to X: its tensor scale from this call's absmax, one E4M3 scale per
 * 16 values of a row), then
 *   Y64[i,j] = s_tx * s_tw * sum_k (e2m1(cx[i,k]) * e4m3(sbx[i,k/16]))
 *                                * (e2m1(cw[j,k]) * e4m3(sbw[j,k/16])) + bias[j]
 * in double (each product exact). Xq [M,K/2], s_bx [M,K/16], s_tx [1] are
 * written out (codes for every row; Y64/Y only for `rows`). */
void orc_nvfp4_forward(const uint16_t *X, int dt, int64_t M, int64_t K, const uint8_t *Wq, const uint8_t *s_bw,
                       float s_tw, int64_t N, const uint16_t *bias, const int64_t *rows, int64_t nrows,
                       uint8_t *Xq, uint8_t *s_bx, float *s_tx, double *Y64, uint16_t *Y) {
    orc_quantize_weight_nvfp4(X, dt, M, K, Xq, s_bx, s_tx);
    double *Wd = (double *)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k)
            Wd[j * K + k] = orc_e2m1_decode(orc_nvfp4_code(Wq, K, j, k)) * orc_e4m3_decode(s_bw[j * (K / 16) + k / 16]);
    const double st = (double)*s_tx * (double)s_tw;
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        double *xd = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
        for (int64_t k = 0; k < K; ++k)
            xd[k] = orc_e2m1_decode(orc_nvfp4_code(Xq, K, i, k)) * orc_e4m3_decode(s_bx[i * (K / 16) + k / 16]);
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += xd[k] * Wd[j * K + k];
            acc *= st;
            if (bias) acc += widen(bias[j], dt);
            if (Y64) Y64[r * N + j] = acc;
            if (Y) Y[r * N + j] = narrow(acc, dt);
        }
        free(xd);
    }
    free(Wd);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
