/*
 * qlinear_oracle.c -- plain, slow, fp64 CPU oracle for the group-scaled
 * quantized linear layer y = x . dequant(W)^T and its MoE gate_up use.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA library; it is written
 * from the format definitions on the model cards:
 *
 *   "gemma4-26b-a4b-dflash-i8" README, table "Weights" and the recipe in
 *     "How this file was made": int8 codes -127..127, a bf16 scale per row
 *     and 128 of K, 128-wide Hadamard domain (transform=fwht128, clamp=sym);
 *     the drafter's linears use an f16 scale instead.
 *   "gemma4-26b-a4b-dflash-fp8" README, table "Weights" and its recipe:
 *     FP8 E4M3 codes per 128x128 block with bf16 block scales.
 *   "Gemma4-26B-CIRU-AMD-STRIX-vLLM", "What is in the release": symmetric
 *     int4, group 64, bf16 scales, 4.25 bits per quantized weight.
 *   "keptn/gemma4-31b-w5", table "Format" and "How it was made" step 4:
 *     int5 codes with a u8 zero point and one f16 scale per 128 weights;
 *     activations 16-bit up to 64 rows, int8 per token and 128 above.
 *   The i8 card's recipe marks the experts' quantiser "rule=search" (round to
 *     nearest with a scale search); the candidates and the measure are a
 *     reading of this build, stated at qo_scale_search_group.
 *   "keptn/gemma4-12b-i8g", table "Format": int8 weights with a bf16 scale
 *     per 128, activations int8 with one scale per token and 128 values.
 *   The FP8-activation variant of the fp8 container (format 7) takes the
 *     weights of "gemma4-26b-a4b-dflash-fp8" unchanged and quantises the
 *     activations as the int8 cards do -- one fp32 scale per token and 128
 *     values -- but to E4M3 codes: a reading of this build, not a card's.
 *   The experts' down projections and the router stay bf16 ("gemma4-26b-
 *     a4b-dflash-i8" README, table "Weights"); the activation between the
 *     gate and up halves and the routing-weighted combine are not on the
 *     cards: qo_moe_down_combine states the reading taken.
 *
 * Where the cards leave the arithmetic open, the oracle takes one plain
 * reading and states it at the function that implements it.  Everything is
 * evaluated in fp64 except the steps whose result is an integer code (the
 * quantisers), which run in fp32 exactly as their definition states, so that
 * a device implementation can reproduce the same codes bit for bit.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (no -ffast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Format identifiers: the numeric values of the library's public enum. */
enum {
    QO_I8_G128_BF16 = 1,   /* int8, bf16 scale per row per 128 K, bf16 x  */
    QO_I8_G128_F16 = 2,    /* int8, f16 scale per row per 128 K, bf16 x   */
    QO_I8A8_G128_BF16 = 3, /* int8 weights and int8 activations (W8A8)    */
    QO_I4_G64_BF16 = 4,    /* int4 [-8,7], bf16 scale per row per 64 K    */
    QO_I5Z_G128_F16 = 5,   /* int5 [0,31], u8 zero + f16 scale per 128 K  */
    QO_FP8_B128_BF16 = 6,  /* e4m3, bf16 scale per 128x128 block          */
    QO_FP8A8_B128_BF16 = 7 /* the same weights, e4m3 activations          */
};
enum { QO_HADAMARD = 1 };

/* ------------------------------------------------------------------------ */
/* Number formats, from their definitions (not from any bit trick).          */
/* ------------------------------------------------------------------------ */

/* Round v to the nearest value of a binary floating-point format with
 * `sig` significant bits, minimum normal exponent `emin` (subnormals below),
 * ties to even.  Returns the rounded value; +-INFINITY when the rounded
 * magnitude exceeds `maxfinite` (IEEE overflow), or +-maxfinite when
 * `saturate` is set.  All steps are exact in fp64 for the inputs used here
 * (fp32 or fp64 values rounded to at most 11 significant bits). */
static double round_to_format(double v, int sig, int emin, double maxfinite, int saturate)
{
    if (isnan(v)) return v;
    if (v == 0.0) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1): exponent of a is e-1 */
    int ex = e - 1;
    if (ex < emin) ex = emin;                    /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, ex - (sig - 1));
    double r = a / quantum;                      /* exact: power-of-two divide */
    double lo = floor(r);
    double frac = r - lo;
    double n = lo;
    if (frac > 0.5 || (frac == 0.5 && fmod(lo, 2.0) != 0.0)) n = lo + 1.0;
    double out = n * quantum;
    if (out > maxfinite) out = saturate ? maxfinite : INFINITY;
    return v < 0 ? -out : out;
}

/* bfloat16: 8 significant bits, exponent range of fp32. */
static const double BF16_MAX = 3.3895313892515355e38; /* (2 - 2^-7) * 2^127 */

double qo_bf16_decode(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;     /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

uint16_t qo_bf16_encode(double v)
{
    double r = round_to_format(v, 8, -126, BF16_MAX, 0);
    float f = (float)r;                  /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(r)) return (uint16_t)(0x7FC0 | ((u >> 16) & 0x8000));
    return (uint16_t)(u >> 16);
}

/* IEEE binary16: 11 significant bits, emin = -14, max 65504. */
double qo_f16_decode(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

uint16_t qo_f16_encode(double v)
{
    if (isnan(v)) return 0x7E00;
    double r = round_to_format(v, 11, -14, 65504.0, 0);
    uint16_t s = (r < 0 || (r == 0 && signbit(r))) ? 0x8000 : 0;
    double a = fabs(r);
    if (isinf(a)) return s | 0x7C00;
    if (a == 0) return s;
    if (a < ldexp(1.0, -14)) return s | (uint16_t)(a / ldexp(1.0, -24));
    int e;
    frexp(a, &e);
    int ex = e - 1;
    uint16_t m = (uint16_t)((a / ldexp(1.0, ex) - 1.0) * 1024.0);
    return s | (uint16_t)((ex + 15) << 10) | m;
}

/* OCP FP8 E4M3 (the "fn" variant): bias 7, no infinities, S.1111.111 is NaN,
 * largest finite 448, subnormals m * 2^-9. */
double qo_e4m3_decode(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round to nearest even, saturating to +-448 (the "satfinite" behaviour). */
uint8_t qo_e4m3_encode(double v)
{
    if (isnan(v)) return 0x7F;
    double r = round_to_format(v, 4, -6, 448.0, 1);
    uint8_t s = (r < 0 || (r == 0 && signbit(r))) ? 0x80 : 0;
    double a = fabs(r);
    if (a == 0) return s;
    if (a < ldexp(1.0, -6)) return s | (uint8_t)(a / ldexp(1.0, -9));
    int e;
    frexp(a, &e);
    int ex = e - 1;
    uint8_t m = (uint8_t)((a / ldexp(1.0, ex) - 1.0) * 8.0);
    return s | (uint8_t)((ex + 7) << 3) | m;
}

/* ------------------------------------------------------------------------ */
/* Walsh-Hadamard transform over 128 values (transform=fwht128).             */
/* ------------------------------------------------------------------------ */

/* Exact fp64 transform with the Sylvester-ordered matrix H_128
 * (H_1 = [1], H_2n = [[H, H], [H, -H]]), unnormalised: out = H . v. */
void qo_fwht128_f64(const double* v, double* out)
{
    double t[128];
    memcpy(t, v, sizeof t);
    for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = t[j], b = t[j + h];
                t[j] = a + b;
                t[j + h] = a - b;
            }
    memcpy(out, t, sizeof t);
}

/* The transform as the quantisers evaluate it, fixed so that the codes it
 * leads to are reproducible: fp32 radix-2 butterflies (a, b) -> (a + b, a - b)
 * with strides 1, 2, 4, ..., 64 in that order, each rounded to nearest, then
 * one multiply by fp32(1/sqrt(128)) = 0x3DB504F3.  This orthonormal scaling
 * keeps (H x) . (H w) = x . w, so a rotated weight row still multiplies a
 * rotated activation row to the same product. */
static float fwht_scale_f32(void)
{
    uint32_t u = 0x3DB504F3u;
    float c;
    memcpy(&c, &u, 4);
    return c;
}

void qo_fwht128_spec_f32(const float* v, float* out)
{
    volatile float t[128]; /* volatile: keep every rounding in fp32 */
    for (int i = 0; i < 128; ++i) t[i] = v[i];
    for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float a = t[j], b = t[j + h];
                float s = a + b, d = a - b;
                t[j] = s;
                t[j + h] = d;
            }
    const float c = fwht_scale_f32();
    for (int i = 0; i < 128; ++i) {
        float p = t[i] * c;
        out[i] = p;
    }
}

/* hadamard128_rotate: bf16 x [M,K] -> bf16 y [M,K], each 128-block of each
 * row transformed by qo_fwht128_spec_f32, the fp32 result rounded to bf16. */
void qo_hadamard128_rotate(const uint16_t* x, int M, int K, uint16_t* y)
{
    float v[128], r[128];
    for (int m = 0; m < M; ++m)
        for (int g = 0; g < K / 128; ++g) {
            const uint16_t* src = x + (size_t)m * K + (size_t)g * 128;
            for (int i = 0; i < 128; ++i) v[i] = (float)qo_bf16_decode(src[i]);
            qo_fwht128_spec_f32(v, r);
            uint16_t* dst = y + (size_t)m * K + (size_t)g * 128;
            for (int i = 0; i < 128; ++i) dst[i] = qo_bf16_encode((double)r[i]);
        }
}

/* ------------------------------------------------------------------------ */
/* Activation quantiser: int8, one scale per token per 128 values            */
/* ("keptn/gemma4-12b-i8g", Format).  The card gives no arithmetic; the     */
/* reading taken: on the fp32 group v (rotated by the spec transform when    */
/* `rotate` is set, never rounded to bf16 in between):                       */
/*   amax = max |v|;  s = fp32(amax / 127);  inv = fp32(127 / amax);         */
/*   q = clamp(round_half_even(fp32(v * inv)), -127, 127);                   */
/*   amax == 0 gives s = 0 and q = 0.  The scale is kept in fp32.            */
/* ------------------------------------------------------------------------ */

static int rint_even_f32(float f) /* nearest integer, ties to even; |f| small */
{
    double d = (double)f;
    double lo = floor(d);
    double fr = d - lo;
    double n = lo;
    if (fr > 0.5 || (fr == 0.5 && fmod(lo, 2.0) != 0.0)) n = lo + 1.0;
    return (int)n;
}

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

void qo_act_quant_group(const float* v, int8_t* q, float* s)
{
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s = 0.0f;
        for (int i = 0; i < 128; ++i) q[i] = 0;
        return;
    }
    volatile float sv = amax / 127.0f;
    volatile float inv = 127.0f / amax;
    *s = sv;
    for (int i = 0; i < 128; ++i) {
        volatile float p = v[i] * inv;
        q[i] = (int8_t)clampi(rint_even_f32(p), -127, 127);
    }
}

/* E4M3 activations, per token per 128 values, in the same steps as the int8
 * quantiser with 448 (the largest finite E4M3 value) in place of 127:
 *   amax = max |v|;  s = fp32(amax / 448);  inv = fp32(448 / amax);
 *   q[i] = e4m3_rne_satfinite(fp32(v[i] * inv)).
 *   amax == 0 gives s = 0 and q = 0.  The scale is kept in fp32. */
void qo_act_quant_e4m3_group(const float* v, uint8_t* q, float* s)
{
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s = 0.0f;
        for (int i = 0; i < 128; ++i) q[i] = 0;
        return;
    }
    volatile float sv = amax / 448.0f;
    volatile float inv = 448.0f / amax;
    *s = sv;
    for (int i = 0; i < 128; ++i) {
        volatile float p = v[i] * inv;
        q[i] = qo_e4m3_encode((double)p);
    }
}

void qo_act_quant_e4m3_g128(const uint16_t* x, int M, int K, int rotate, uint8_t* q, float* s)
{
    float v[128], r[128];
    for (int m = 0; m < M; ++m)
        for (int g = 0; g < K / 128; ++g) {
            const uint16_t* src = x + (size_t)m * K + (size_t)g * 128;
            for (int i = 0; i < 128; ++i) v[i] = (float)qo_bf16_decode(src[i]);
            if (rotate) qo_fwht128_spec_f32(v, r);
            else memcpy(r, v, sizeof r);
            qo_act_quant_e4m3_group(r, q + (size_t)m * K + (size_t)g * 128, s + (size_t)m * (K / 128) + g);
        }
}

void qo_act_quant_i8_g128(const uint16_t* x, int M, int K, int rotate, int8_t* q, float* s)
{
    float v[128], r[128];
    for (int m = 0; m < M; ++m)
        for (int g = 0; g < K / 128; ++g) {
            const uint16_t* src = x + (size_t)m * K + (size_t)g * 128;
            for (int i = 0; i < 128; ++i) v[i] = (float)qo_bf16_decode(src[i]);
            if (rotate) qo_fwht128_spec_f32(v, r);
            else memcpy(r, v, sizeof r);
            qo_act_quant_group(r, q + (size_t)m * K + (size_t)g * 128, s + (size_t)m * (K / 128) + g);
        }
}

/* ------------------------------------------------------------------------ */
/* Weight quantisers (round to nearest, "rtn ... clamp=sym" in the recipes). */
/* ------------------------------------------------------------------------ */

/* Row n of W as the quantiser sees it: fp32, rotated block by block by the
 * spec transform when QO_HADAMARD is set. */
static void weight_row(const float* W, int K, int n, int flags, float* row)
{
    const float* src = W + (size_t)n * K;
    if (flags & QO_HADAMARD)
        for (int g = 0; g < K / 128; ++g) qo_fwht128_spec_f32(src + g * 128, row + g * 128);
    else
        memcpy(row, src, sizeof(float) * (size_t)K);
}

/* int8, group 128 along K: s = scale_fmt(fp32(amax / 127)) with the scale
 * format bf16 or f16; q = clamp(round_half_even(fp32(w / s)), -127, 127);
 * the clamp absorbs a scale that rounded down.  amax == 0 (or a scale that
 * rounds to 0) gives s = 0 and q = 0. */
void qo_quant_i8_g128(const float* W, int N, int K, int flags, int scale_f16, int8_t* q, uint16_t* s)
{
    int G = K / 128;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        float* row = (float*)malloc(sizeof(float) * (size_t)K);
        weight_row(W, K, n, flags, row);
        for (int g = 0; g < G; ++g) {
            const float* v = row + g * 128;
            float amax = 0.0f;
            for (int i = 0; i < 128; ++i)
                if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
            volatile float raw = amax / 127.0f;
            uint16_t sb = scale_f16 ? qo_f16_encode(raw) : qo_bf16_encode(raw);
            float sf = (float)(scale_f16 ? qo_f16_decode(sb) : qo_bf16_decode(sb));
            s[(size_t)n * G + g] = sb;
            for (int i = 0; i < 128; ++i) {
                int code = 0;
                if (sf != 0.0f) {
                    volatile float t = v[i] / sf;
                    code = clampi(rint_even_f32(t), -127, 127);
                }
                q[(size_t)n * K + g * 128 + i] = (int8_t)code;
            }
        }
        free(row);
    }
}

/* int8 group 128 with a scale search ("round to nearest with a scale search",
 * rule=search, in the "gemma4-26b-a4b-dflash-i8" README's "Weights" table and
 * recipe).  The card names the search but not its candidates or its measure;
 * the reading taken here:
 *   r = fp32(amax / 127) (the round-to-nearest scale before rounding);
 *   candidate i = 0..20: raw_i = fp32(r * c_i), c_i = fp32((100 - i) / 100),
 *     s_i = scale_fmt(raw_i), codes q = clamp(rne(fp32(w / s_i)), -127, 127)
 *     (s_i == 0: every code 0), exactly as round to nearest does with s_i;
 *   error_i = sum over the group, k = 0..127 in order, of (w_k - s_i * q_k)^2,
 *     each product, difference and sum rounded to fp64 (no fused operations);
 *   the group keeps the candidate with the smallest error, the smaller i on a tie.
 * c_0 = 1, so candidate 0 is the round-to-nearest result and the search never
 * does worse than it.  v is the group as the quantiser sees it (rotated when
 * the weights live in the Hadamard domain); *i_out (may be NULL) gets the
 * chosen i. */
void qo_scale_search_group(const float* v, int scale_f16, int8_t* q, uint16_t* s_out, int* i_out)
{
    float amax = 0.0f;
    for (int k = 0; k < 128; ++k)
        if (fabsf(v[k]) > amax) amax = fabsf(v[k]);
    volatile float r = amax / 127.0f;
    int best = 0;
    double best_err = 0.0;
    uint16_t best_s = 0;
    for (int i = 0; i <= 20; ++i) {
        volatile float c = (float)(100 - i) / 100.0f;
        volatile float raw = r * c;
        uint16_t sb = scale_f16 ? qo_f16_encode(raw) : qo_bf16_encode(raw);
        float sf = (float)(scale_f16 ? qo_f16_decode(sb) : qo_bf16_decode(sb));
        double err = 0.0;
        for (int k = 0; k < 128; ++k) {
            int code = 0;
            if (sf != 0.0f) {
                volatile float t = v[k] / sf;
                code = clampi(rint_even_f32(t), -127, 127);
            }
            double d = (double)v[k] - (double)sf * (double)code;
            err = err + d * d;
        }
        if (i == 0 || err < best_err) {
            best = i;
            best_err = err;
            best_s = sb;
        }
    }
    float sf = (float)(scale_f16 ? qo_f16_decode(best_s) : qo_bf16_decode(best_s));
    for (int k = 0; k < 128; ++k) {
        int code = 0;
        if (sf != 0.0f) {
            volatile float t = v[k] / sf;
            code = clampi(rint_even_f32(t), -127, 127);
        }
        q[k] = (int8_t)code;
    }
    *s_out = best_s;
    if (i_out) *i_out = best;
}

/* The scale search over a whole [N, K] weight (rows rotated first when
 * QO_HADAMARD is set); chosen (may be NULL) gets each group's i, [N][K/128]. */
void qo_quant_i8_g128_search(const float* W, int N, int K, int flags, int scale_f16, int8_t* q, uint16_t* s,
                             int32_t* chosen)
{
    int G = K / 128;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        float* row = (float*)malloc(sizeof(float) * (size_t)K);
        weight_row(W, K, n, flags, row);
        for (int g = 0; g < G; ++g) {
            int ci;
            qo_scale_search_group(row + g * 128, scale_f16, q + (size_t)n * K + g * 128, s + (size_t)n * G + g, &ci);
            if (chosen) chosen[(size_t)n * G + g] = ci;
        }
        free(row);
    }
}

/* Symmetric int4, group 64: s = bf16(fp32(amax / 7)),
 * q = clamp(round_half_even(fp32(w / s)), -8, 7); s == 0 gives q = 0. */
void qo_quant_i4_g64(const float* W, int N, int K, int flags, int8_t* q, uint16_t* s)
{
    int G = K / 64;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        float* row = (float*)malloc(sizeof(float) * (size_t)K);
        weight_row(W, K, n, flags, row);
        for (int g = 0; g < G; ++g) {
            const float* v = row + g * 64;
            float amax = 0.0f;
            for (int i = 0; i < 64; ++i)
                if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
            volatile float raw = amax / 7.0f;
            uint16_t sb = qo_bf16_encode(raw);
            float sf = (float)qo_bf16_decode(sb);
            s[(size_t)n * G + g] = sb;
            for (int i = 0; i < 64; ++i) {
                int code = 0;
                if (sf != 0.0f) {
                    volatile float t = v[i] / sf;
                    code = clampi(rint_even_f32(t), -8, 7);
                }
                q[(size_t)n * K + g * 64 + i] = (int8_t)code;
            }
        }
        free(row);
    }
}

/* FP8 E4M3 per 128 (rows) x 128 (K) block: amax over the block,
 * s = bf16(fp32(amax / 448)), q = e4m3_rne_satfinite(fp32(w / s)).  A ragged
 * last row block (N % 128 != 0) takes the rows that exist. */
void qo_quant_fp8_b128(const float* W, int N, int K, int flags, uint8_t* q, uint16_t* s)
{
    int G = K / 128, NB = (N + 127) / 128;
    float* rows = (float*)malloc(sizeof(float) * (size_t)N * K);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) weight_row(W, K, n, flags, rows + (size_t)n * K);
#pragma omp parallel for collapse(2) schedule(static)
    for (int nb = 0; nb < NB; ++nb)
        for (int g = 0; g < G; ++g) {
            int n1 = (nb + 1) * 128 < N ? (nb + 1) * 128 : N;
            float amax = 0.0f;
            for (int n = nb * 128; n < n1; ++n)
                for (int i = 0; i < 128; ++i) {
                    float a = fabsf(rows[(size_t)n * K + g * 128 + i]);
                    if (a > amax) amax = a;
                }
            volatile float raw = amax / 448.0f;
            uint16_t sb = qo_bf16_encode(raw);
            float sf = (float)qo_bf16_decode(sb);
            s[(size_t)nb * G + g] = sb;
            for (int n = nb * 128; n < n1; ++n)
                for (int i = 0; i < 128; ++i) {
                    size_t idx = (size_t)n * K + g * 128 + i;
                    uint8_t code = 0;
                    if (sf != 0.0f) {
                        volatile float t = rows[idx] / sf;
                        code = qo_e4m3_encode((double)t);
                    }
                    q[idx] = code;
                }
        }
    free(rows);
}

/* ------------------------------------------------------------------------ */
/* Bit packing ("codes packed little-endian along K").                       */
/* ------------------------------------------------------------------------ */

/* int4: offset-binary nibble u = q + 8; code k of a row sits in byte k/2,
 * the low nibble for even k and the high nibble for odd k (equivalently,
 * nibble k%8 of the little-endian 32-bit word k/8, low nibble first). */
void qo_pack_i4(const int8_t* q, int N, int K, uint8_t* out)
{
    for (size_t n = 0; n < (size_t)N; ++n)
        for (int b = 0; b < K / 2; ++b) {
            unsigned lo = (unsigned)(q[n * K + 2 * b] + 8) & 15u;
            unsigned hi = (unsigned)(q[n * K + 2 * b + 1] + 8) & 15u;
            out[n * (K / 2) + b] = (uint8_t)(lo | (hi << 4));
        }
}

void qo_unpack_i4(const uint8_t* p, int N, int K, int8_t* q)
{
    for (size_t n = 0; n < (size_t)N; ++n)
        for (int k = 0; k < K; ++k) {
            uint8_t byte = p[n * (K / 2) + k / 2];
            int u = (k & 1) ? (byte >> 4) : (byte & 15);
            q[n * K + k] = (int8_t)(u - 8);
        }
}

/* int5: each row is one least-significant-bit-first bit stream; code k
 * occupies stream bits 5k .. 5k+4, bit b of the stream being bit b%8 of
 * byte b/8.  A row of K codes takes 5K/8 bytes. */
void qo_pack_i5(const uint8_t* q, int N, int K, uint8_t* out)
{
    size_t rb = (size_t)K * 5 / 8;
    memset(out, 0, rb * (size_t)N);
    for (size_t n = 0; n < (size_t)N; ++n)
        for (int k = 0; k < K; ++k)
            for (int bit = 0; bit < 5; ++bit)
                if ((q[n * K + k] >> bit) & 1) {
                    size_t b = (size_t)k * 5 + bit;
                    out[n * rb + b / 8] |= (uint8_t)(1u << (b % 8));
                }
}

void qo_unpack_i5(const uint8_t* p, int N, int K, uint8_t* q)
{
    size_t rb = (size_t)K * 5 / 8;
    for (size_t n = 0; n < (size_t)N; ++n)
        for (int k = 0; k < K; ++k) {
            unsigned v = 0;
            for (int bit = 0; bit < 5; ++bit) {
                size_t b = (size_t)k * 5 + bit;
                v |= (unsigned)((p[n * rb + b / 8] >> (b % 8)) & 1) << bit;
            }
            q[n * K + k] = (uint8_t)v;
        }
}

/* Byte sizes of the three packed buffers of an [N, K] weight. */
int qo_packed_sizes(int fmt, int N, int K, size_t* codes, size_t* scales, size_t* zeros)
{
    size_t n = (size_t)N, k = (size_t)K;
    *zeros = 0;
    switch (fmt) {
    case QO_I8_G128_BF16:
    case QO_I8_G128_F16:
    case QO_I8A8_G128_BF16:
        *codes = n * k;
        *scales = n * (k / 128) * 2;
        return 0;
    case QO_I4_G64_BF16:
        *codes = n * k / 2;
        *scales = n * (k / 64) * 2;
        return 0;
    case QO_I5Z_G128_F16:
        *codes = n * k * 5 / 8;
        *scales = n * (k / 128) * 2;
        *zeros = n * (k / 128);
        return 0;
    case QO_FP8_B128_BF16:
    case QO_FP8A8_B128_BF16:
        *codes = n * k;
        *scales = ((n + 127) / 128) * (k / 128) * 2;
        return 0;
    }
    return 1;
}

/* ------------------------------------------------------------------------ */
/* Dequantisation: W~[n,k] in fp64.                                          */
/*   int8 (any scale format): s[n, k/128] * q                                */
/*   int4:                    s[n, k/64] * q,  q in [-8, 7]                   */
/*   int5:                    s[n, k/128] * (q - z[n, k/128])                 */
/*   fp8:                     s[n/128, k/128] * e4m3(q)                       */
/* ------------------------------------------------------------------------ */

static double scale_of(int fmt, const uint16_t* s, size_t idx)
{
    return (fmt == QO_I8_G128_F16 || fmt == QO_I5Z_G128_F16) ? qo_f16_decode(s[idx]) : qo_bf16_decode(s[idx]);
}

static void dequant_row(int fmt, const uint8_t* codes, const uint16_t* s, const uint8_t* z, int n, int K,
                        double* out)
{
    size_t N0 = (size_t)n;
    switch (fmt) {
    case QO_I8_G128_BF16:
    case QO_I8_G128_F16:
    case QO_I8A8_G128_BF16:
        for (int k = 0; k < K; ++k)
            out[k] = scale_of(fmt, s, N0 * (K / 128) + k / 128) * (double)(int8_t)codes[N0 * K + k];
        break;
    case QO_I4_G64_BF16:
        for (int k = 0; k < K; ++k) {
            uint8_t byte = codes[N0 * (K / 2) + k / 2];
            int q = ((k & 1) ? (byte >> 4) : (byte & 15)) - 8;
            out[k] = scale_of(fmt, s, N0 * (K / 64) + k / 64) * (double)q;
        }
        break;
    case QO_I5Z_G128_F16: {
        size_t rb = (size_t)K * 5 / 8;
        for (int k = 0; k < K; ++k) {
            unsigned v = 0;
            for (int bit = 0; bit < 5; ++bit) {
                size_t b = (size_t)k * 5 + bit;
                v |= (unsigned)((codes[N0 * rb + b / 8] >> (b % 8)) & 1) << bit;
            }
            size_t gi = N0 * (K / 128) + k / 128;
            out[k] = scale_of(fmt, s, gi) * ((double)v - (double)z[gi]);
        }
        break;
    }
    case QO_FP8_B128_BF16:
    case QO_FP8A8_B128_BF16:
        for (int k = 0; k < K; ++k)
            out[k] = scale_of(fmt, s, (N0 / 128) * (K / 128) + k / 128) * qo_e4m3_decode(codes[N0 * K + k]);
        break;
    }
}

void qo_dequant(int fmt, const uint8_t* codes, const uint16_t* scales, const uint8_t* zeros, int N, int K,
                double* W)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) dequant_row(fmt, codes, scales, zeros, n, K, W + (size_t)n * K);
}

/* ------------------------------------------------------------------------ */
/* The linear layer.                                                         */
/*                                                                           */
/*   y[m,n] = sum_k x~[m,k] * W~[n,k]   (fp64)                               */
/*                                                                           */
/* x~ is x itself (bf16, exact) for the weight-only formats, or, with        */
/* QO_HADAMARD, the bf16 output of qo_hadamard128_rotate.  For W8A8 the      */
/* activation is quantised per token per 128 (rotated first with            */
/* QO_HADAMARD); each group's integer dot product                            */
/*   acc[m,n,g] = sum_{k in g} qx[m,k] * qw[n,k]                             */
/* is kept exactly (int32), and y = sum_g sx[m,g] * sw[n,g] * acc[m,n,g].    */
/* The int5 format does the same above 64 rows ("keptn/gemma4-31b-w5",      */
/* table "Format": activations up to 64 rows f16, above that int8 with one  */
/* scale per token and 128 values), with qw = q - z, the zero-point-        */
/* corrected code, and its f16 scale for sw.                                 */
/* ------------------------------------------------------------------------ */
enum { QO_W5A8_MIN_M = 65 };

int qo_forward(const uint16_t* x, int M, int K, const uint8_t* codes, const uint16_t* scales,
               const uint8_t* zeros, int fmt, int flags, int N, double* y, int32_t* acc_out)
{
    if (fmt < QO_I8_G128_BF16 || fmt > QO_FP8A8_B128_BF16) return 1;
    int G = K / 128;
    if (fmt == QO_FP8A8_B128_BF16) {
        /* E4M3 activations: y = sum_g sx[m,g] * sw[n/128,g] * sum_{k in g} e4m3(qx) * e4m3(qw).
         * Every product of two E4M3 values and every partial sum here is exact in fp64. */
        uint8_t* qx = (uint8_t*)malloc((size_t)M * K);
        float* sx = (float*)malloc(sizeof(float) * (size_t)M * G);
        qo_act_quant_e4m3_g128(x, M, K, flags & QO_HADAMARD, qx, sx);
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            const uint8_t* qw = codes + (size_t)n * K;
            for (int m = 0; m < M; ++m) {
                double sum = 0.0;
                for (int g = 0; g < G; ++g) {
                    double part = 0.0;
                    for (int i = 0; i < 128; ++i)
                        part += qo_e4m3_decode(qx[(size_t)m * K + g * 128 + i]) * qo_e4m3_decode(qw[g * 128 + i]);
                    sum += (double)sx[(size_t)m * G + g] * qo_bf16_decode(scales[(size_t)(n / 128) * G + g]) * part;
                }
                y[(size_t)m * N + n] = sum;
            }
        }
        free(qx);
        free(sx);
        return 0;
    }
    if (fmt == QO_I5Z_G128_F16 && M >= QO_W5A8_MIN_M) {
        int8_t* qx = (int8_t*)malloc((size_t)M * K);
        float* sx = (float*)malloc(sizeof(float) * (size_t)M * G);
        qo_act_quant_i8_g128(x, M, K, flags & QO_HADAMARD, qx, sx);
        size_t rb = (size_t)K * 5 / 8;
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            int32_t* qw = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
            for (int k = 0; k < K; ++k) {
                unsigned v = 0;
                for (int bit = 0; bit < 5; ++bit) {
                    size_t b = (size_t)k * 5 + bit;
                    v |= (unsigned)((codes[(size_t)n * rb + b / 8] >> (b % 8)) & 1) << bit;
                }
                qw[k] = (int32_t)v - (int32_t)zeros[(size_t)n * G + k / 128];
            }
            for (int m = 0; m < M; ++m) {
                double sum = 0.0;
                for (int g = 0; g < G; ++g) {
                    int32_t acc = 0;
                    for (int i = 0; i < 128; ++i) acc += (int32_t)qx[(size_t)m * K + g * 128 + i] * qw[g * 128 + i];
                    if (acc_out) acc_out[((size_t)m * N + n) * G + g] = acc;
                    sum += (double)sx[(size_t)m * G + g] * qo_f16_decode(scales[(size_t)n * G + g]) * (double)acc;
                }
                y[(size_t)m * N + n] = sum;
            }
            free(qw);
        }
        free(qx);
        free(sx);
        return 0;
    }
    if (fmt == QO_I8A8_G128_BF16) {
        int8_t* qx = (int8_t*)malloc((size_t)M * K);
        float* sx = (float*)malloc(sizeof(float) * (size_t)M * G);
        qo_act_quant_i8_g128(x, M, K, flags & QO_HADAMARD, qx, sx);
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            const int8_t* qw = (const int8_t*)codes + (size_t)n * K;
            for (int m = 0; m < M; ++m) {
                double sum = 0.0;
                for (int g = 0; g < G; ++g) {
                    int32_t acc = 0;
                    for (int i = 0; i < 128; ++i)
                        acc += (int32_t)qx[(size_t)m * K + g * 128 + i] * (int32_t)qw[g * 128 + i];
                    if (acc_out) acc_out[((size_t)m * N + n) * G + g] = acc;
                    sum += (double)sx[(size_t)m * G + g] * qo_bf16_decode(scales[(size_t)n * G + g]) * (double)acc;
                }
                y[(size_t)m * N + n] = sum;
            }
        }
        free(qx);
        free(sx);
        return 0;
    }
    double* xt = (double*)malloc(sizeof(double) * (size_t)M * K);
    if (flags & QO_HADAMARD) {
        uint16_t* xr = (uint16_t*)malloc(2 * (size_t)M * K);
        qo_hadamard128_rotate(x, M, K, xr);
        for (size_t i = 0; i < (size_t)M * K; ++i) xt[i] = qo_bf16_decode(xr[i]);
        free(xr);
    } else {
        for (size_t i = 0; i < (size_t)M * K; ++i) xt[i] = qo_bf16_decode(x[i]);
    }
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
        dequant_row(fmt, codes, scales, zeros, n, K, w);
        for (int m = 0; m < M; ++m) {
            double sum = 0.0;
            for (int k = 0; k < K; ++k) sum += xt[(size_t)m * K + k] * w[k];
            y[(size_t)m * N + n] = sum;
        }
        free(w);
    }
    free(xt);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MoE gate_up ("gemma4-26b-a4b-dflash-i8", Weights: the routed experts'    */
/* gate_up projections, int8 in the Hadamard domain).                        */
/* ------------------------------------------------------------------------ */

/* Group the T*topk (token, slot) pairs by expert.  counts[e] = pairs routed
 * to e; offsets = exclusive prefix sum (E+1 entries); perm lists the flat
 * pair index t*topk + j in order of (expert, t, j), so each expert's segment
 * keeps the tokens' order.  Ids outside [0, E) are dropped and counted in
 * the return value. */
int qo_moe_permute(const int32_t* ids, int T, int topk, int E, int32_t* counts, int32_t* offsets,
                   int32_t* perm)
{
    int bad = 0;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int i = 0; i < T * topk; ++i) {
        if (ids[i] < 0 || ids[i] >= E) ++bad;
        else ++counts[ids[i]];
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int pos = 0;
    for (int e = 0; e < E; ++e)
        for (int i = 0; i < T * topk; ++i)
            if (ids[i] == e) perm[pos++] = i;
    return bad;
}

/* out[t, j, :] = x~[t, :] . W~_{ids[t,j]}^T for every pair, where the expert
 * weights are stacked [E, N, K] (codes) and [E, N, K/128] (scales), and x~ is
 * x rotated once per token (bf16, as qo_hadamard128_rotate) when QO_HADAMARD
 * is set.  The routing weights are not applied: they belong after the down
 * projection, which this layer does not compute.  Pairs with an invalid id
 * leave their output row untouched.
 * Format 7 experts (the fp8 container's E4M3 weights with E4M3 activations,
 * "gemma4-26b-a4b-dflash-fp8" README, table "Weights", with the activation
 * rule of "keptn/gemma4-12b-i8g" applied to E4M3 codes -- a reading of this
 * build): each token is quantised once, per 128 values (rotated first with
 * QO_HADAMARD), and every pair's output is the format-7 sum
 * sum_g sx[t,g] * sw_e[n/128,g] * sum_{k in g} e4m3(qx) * e4m3(qw). */
int qo_moe_gate_up(const uint16_t* x, const int32_t* ids, int T, int topk, int E, int N, int K, int fmt,
                   int flags, const uint8_t* codes, const uint16_t* scales, double* out)
{
    if (fmt != QO_I8_G128_BF16 && fmt != QO_I8_G128_F16 && fmt != QO_FP8_B128_BF16 && fmt != QO_FP8A8_B128_BF16)
        return 1;
    size_t cs, ss, zs;
    qo_packed_sizes(fmt, N, K, &cs, &ss, &zs);
    if (fmt == QO_FP8A8_B128_BF16) {
        const int G = K / 128;
        uint8_t* qx = (uint8_t*)malloc((size_t)T * K);
        float* sx = (float*)malloc(sizeof(float) * (size_t)T * G);
        qo_act_quant_e4m3_g128(x, T, K, flags & QO_HADAMARD, qx, sx);
#pragma omp parallel for schedule(dynamic)
        for (int p = 0; p < T * topk; ++p) {
            const int e = ids[p], t = p / topk;
            if (e < 0 || e >= E) continue;
            const uint8_t* ce = codes + (size_t)e * cs;
            const uint16_t* se = scales + (size_t)e * (ss / 2);
            for (int n = 0; n < N; ++n) {
                double sum = 0.0;
                for (int g = 0; g < G; ++g) {
                    double part = 0.0;
                    for (int i = 0; i < 128; ++i)
                        part += qo_e4m3_decode(qx[(size_t)t * K + g * 128 + i]) *
                                qo_e4m3_decode(ce[(size_t)n * K + g * 128 + i]);
                    sum += (double)sx[(size_t)t * G + g] * qo_bf16_decode(se[(size_t)(n / 128) * G + g]) * part;
                }
                out[(size_t)p * N + n] = sum;
            }
        }
        free(qx);
        free(sx);
        return 0;
    }
    double* xt = (double*)malloc(sizeof(double) * (size_t)T * K);
    uint16_t* xr = (uint16_t*)malloc(2 * (size_t)T * K);
    if (flags & QO_HADAMARD) qo_hadamard128_rotate(x, T, K, xr);
    else memcpy(xr, x, 2 * (size_t)T * K);
    for (size_t i = 0; i < (size_t)T * K; ++i) xt[i] = qo_bf16_decode(xr[i]);
    free(xr);
#pragma omp parallel for schedule(dynamic)
    for (int e = 0; e < E; ++e) {
        const uint8_t* ce = codes + (size_t)e * cs;
        const uint16_t* se = scales + (size_t)e * (ss / 2);
        double* w = NULL;
        for (int p = 0; p < T * topk; ++p) {
            if (ids[p] != e) continue;
            if (!w) { /* dequantise expert e once, on its first routed pair */
                w = (double*)malloc(sizeof(double) * (size_t)N * K);
                for (int n = 0; n < N; ++n) dequant_row(fmt, ce, se, NULL, n, K, w + (size_t)n * K);
            }
            int t = p / topk;
            for (int n = 0; n < N; ++n) {
                double sum = 0.0;
                for (int k = 0; k < K; ++k) sum += xt[(size_t)t * K + k] * w[(size_t)n * K + k];
                out[(size_t)p * N + n] = sum;
            }
        }
        free(w);
    }
    free(xt);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MoE down projection and combine ("gemma4-26b-a4b-dflash-i8", Weights:     */
/* the routed experts' down projections bf16 as the checkpoint ships them).  */
/* ------------------------------------------------------------------------ */

/* GELU with the tanh approximation, the activation of the Gemma family's
 * gated MLP (the cards name no activation; this is the reading taken):
 * gelu(v) = 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), in fp64. */
double qo_gelu_tanh(double v)
{
    const double c = sqrt(2.0 / 3.14159265358979323846);
    return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

/* For every (token, slot) pair p = t * topk + j routed to expert e = ids[p]:
 * h[p] is its gate_up output (fp32, [2I]: the gate half first, then the up
 * half, the row order of the packed experts), a_i = gelu(h[p][i]) * h[p][I + i]
 * (fp64), d[n] = sum_i a_i * wd_e[n][i] with the expert's bf16 down weight
 * wd_e [K][I] decoded exactly, and out[t][n] = sum_j w[t][j] * d_(t,j)[n],
 * the routing weights as given (not renormalised), summed in slot order.
 * Pairs with an id outside [0, E) add nothing.  out fp64 [T][K]. */
int qo_moe_down_combine(const float* h, const int32_t* ids, const float* w, int T, int topk, int E, int I, int K,
                        const uint16_t* wd, double* out)
{
#pragma omp parallel for schedule(dynamic)
    for (int t = 0; t < T; ++t) {
        double* a = (double*)malloc(sizeof(double) * (size_t)I);
        for (int n = 0; n < K; ++n) out[(size_t)t * K + n] = 0.0;
        for (int j = 0; j < topk; ++j) {
            const int p = t * topk + j, e = ids[p];
            if (e < 0 || e >= E) continue;
            const float* hp = h + (size_t)p * 2 * I;
            for (int i = 0; i < I; ++i) a[i] = qo_gelu_tanh((double)hp[i]) * (double)hp[I + i];
            const uint16_t* we = wd + (size_t)e * K * I;
            for (int n = 0; n < K; ++n) {
                double d = 0.0;
                for (int i = 0; i < I; ++i) d += a[i] * qo_bf16_decode(we[(size_t)n * I + i]);
                out[(size_t)t * K + n] += (double)w[p] * d;
            }
        }
        free(a);
    }
    return 0;
}
