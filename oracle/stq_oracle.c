/*
 * stq_oracle.c -- the oracle: a plain, slow, single-threaded fp64 CPU implementation of
 * what the quantized-state decode path computes.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this code. The product library never links, loads or calls it, and it shares
 * no code, header, helper, table or constant with the CUDA path.
 *
 * Sources (pages, cited by title and section):
 *   [P1]  "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), sections 背景 / 方法 / 實驗結果
 *   [P5]  "线性注意力状态量化难题:Qwen状态池70并发就超模型权重" (aitest123.com/news/n1kj09),
 *         sections 直接量化为什么会翻车 / 时间维度 / 空间维度 / 工程落地
 * The pages name the method (gated delta rule state, per-step read -> update -> requantize ->
 * store, key-row x value-column dual scales, impact-weighted column fit, per-head bit widths
 * from a few discrete candidates, a small set of FP16 "pivot" heads) but print no formula.
 * The exact formulas below are this library's specification; every place where the pages
 * leave a step open is marked READING and listed in the design notes.
 *
 * Conventions: a head state S is d_k x d_v, row-major, S[i*dv + j]; i is the key row, j the
 * value column. All arithmetic is IEEE fp64 with round-to-nearest-even, compiled without
 * FMA contraction. Stored scales are fp32, stored pivots fp16, emitted outputs o fp32.
 *
 * Byte layout of one head block (READING: the pages give no layout):
 *   bits in {4,6,8}: packed codes, code (i,j) occupies bits [b*n, b*n+b) of a little-endian
 *     bitstream, n = i*dv + j, bit k of the stream is bit (k mod 8) of byte k/8; each code is
 *     stored offset-binary u = Q + 2^(b-1); then zero padding to a 16-byte boundary; then
 *     r[dk], then c[dv], each fp32 (or bf16 in the 16-bit scale format); then zero padding to
 *     a 128-byte boundary.
 *   bits == 16 (pivot): S as fp16 row-major, padded to 128 bytes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "stq_oracle.h"

/* ------------------------------------------------------------------------------------------ */
/* Small helpers                                                                              */
/* ------------------------------------------------------------------------------------------ */

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int orc_qmax(int bits) { return (1 << (bits - 1)) - 1; }

static int valid_bits(int bits) { return bits == 4 || bits == 6 || bits == 8 || bits == 16; }

/* Round half to even, written out from its definition: the nearest integer, and of two
 * equally near integers the even one. Valid for |y| < 2^52 (always the case here). */
double orc_round_half_even(double y)
{
    double a = fabs(y);
    double f = floor(a);
    double d = a - f; /* exact: a and f share the exponent range, a < 2^52 */
    double n;
    if (d > 0.5)
        n = f + 1.0;
    else if (d < 0.5)
        n = f;
    else
        n = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
    return y < 0 ? -n : n;
}

/* Distance of y from the nearest rounding tie n + 1/2, i.e. | |y - floor(y)| - 1/2 |. */
static double tie_distance(double y)
{
    double fr = y - floor(y);
    return fabs(fr - 0.5);
}

/* ------------------------------------------------------------------------------------------ */
/* Layout                                                                                     */
/* ------------------------------------------------------------------------------------------ */

size_t orc_codes_bytes(int bits, int dk, int dv)
{
    size_t nbits = (size_t)bits * (size_t)dk * (size_t)dv;
    return (nbits + 7) / 8;
}

size_t orc_scale_offset(int bits, int dk, int dv)
{
    return round_up(orc_codes_bytes(bits, dk, dv), 16);
}

static int valid_sfmt(int sfmt) { return sfmt == ORC_SCALE_F32 || sfmt == ORC_SCALE_BF16; }
static size_t scale_bytes(int sfmt) { return sfmt == ORC_SCALE_BF16 ? 2 : 4; }

size_t orc_block_bytes_s(int bits, int sfmt, int dk, int dv)
{
    if (!valid_bits(bits) || !valid_sfmt(sfmt) || dk < 1 || dv < 1) return 0;
    if (bits == 16) return round_up((size_t)2 * dk * dv, 128);
    return round_up(orc_scale_offset(bits, dk, dv) + scale_bytes(sfmt) * ((size_t)dk + (size_t)dv), 128);
}

size_t orc_block_bytes(int bits, int dk, int dv) { return orc_block_bytes_s(bits, ORC_SCALE_F32, dk, dv); }

/* ------------------------------------------------------------------------------------------ */
/* Packing: offset-binary codes into a little-endian bitstream                                */
/* ------------------------------------------------------------------------------------------ */

void orc_pack(int bits, size_t n, const int32_t *u, uint8_t *out)
{
    size_t nbytes = ((size_t)bits * n + 7) / 8;
    memset(out, 0, nbytes);
    for (size_t idx = 0; idx < n; ++idx) {
        for (int t = 0; t < bits; ++t) {
            size_t bit = (size_t)bits * idx + (size_t)t;
            if ((u[idx] >> t) & 1) out[bit / 8] |= (uint8_t)(1u << (bit % 8));
        }
    }
}

void orc_unpack(int bits, size_t n, const uint8_t *in, int32_t *u)
{
    for (size_t idx = 0; idx < n; ++idx) {
        int32_t val = 0;
        for (int t = 0; t < bits; ++t) {
            size_t bit = (size_t)bits * idx + (size_t)t;
            if ((in[bit / 8] >> (bit % 8)) & 1) val |= (int32_t)1 << t;
        }
        u[idx] = val;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* IEEE binary16, from the format's definition (1 sign, 5 exponent bits biased by 15, 10      */
/* fraction bits; exponent 0 = subnormal with quantum 2^-24; exponent 31 = inf/NaN).          */
/* ------------------------------------------------------------------------------------------ */

double orc_half_to_double(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return s ? -v : v;
}

uint16_t orc_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    if (a >= 65520.0) return sign | 0x7c00; /* 65504 + half an ulp (16) and above -> inf */
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: integer multiple of 2^-24 (may round up into the smallest normal) */
        double r = orc_round_half_even(ldexp(a, 24));
        return sign | (uint16_t)r;
    }
    int E;
    frexp(a, &E);  /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1; /* a in [2^e, 2^(e+1)) */
    double r = orc_round_half_even(ldexp(a, 10 - e)); /* significand in [1024, 2048] */
    if (r == 2048.0) {
        r = 1024.0;
        e += 1;
    }
    if (e > 15) return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)r - 1024));
}

/* Position of a real value between two neighbouring fp16 values, in units of the fp16 quantum
 * at that magnitude: used only to flag fp16 rounding near-ties. */
static double half_units(double a)
{
    a = fabs(a);
    if (a < ldexp(1.0, -14)) return ldexp(a, 24);
    int E;
    frexp(a, &E);
    return ldexp(a, 10 - (E - 1));
}

/* ------------------------------------------------------------------------------------------ */
/* bfloat16, from the format's definition (1 sign, 8 exponent bits biased by 127, 7 fraction  */
/* bits; exponent 0 = subnormal with quantum 2^-133; exponent 255 = inf/NaN): the upper half  */
/* of an IEEE binary32 pattern.                                                               */
/* ------------------------------------------------------------------------------------------ */

double orc_bf16_to_double(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int m = h & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133);
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), e - 134); /* (1 + m/128) * 2^(e-127) */
    return s ? -v : v;
}

uint16_t orc_double_to_bf16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7fc0;
    /* the largest finite value is (2 - 2^-7) 2^127; half an ulp above it rounds to inf */
    if (a >= ldexp(255.0 + 0.5, 120)) return sign | 0x7f80;
    if (a < ldexp(1.0, -126)) {
        double r = orc_round_half_even(ldexp(a, 133)); /* subnormal: multiple of 2^-133 */
        return sign | (uint16_t)r;
    }
    int E;
    frexp(a, &E);  /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1; /* a in [2^e, 2^(e+1)) */
    double r = orc_round_half_even(ldexp(a, 7 - e)); /* significand in [128, 256] */
    if (r == 256.0) {
        r = 128.0;
        e += 1;
    }
    if (e > 127) return sign | 0x7f80;
    return sign | (uint16_t)(((e + 127) << 7) | ((int)r - 128));
}

/* Position of a positive value on the bf16 grid in units of the quantum at that magnitude:
 * used only to flag scale rounding near-ties. */
static double bf16_units(double a)
{
    a = fabs(a);
    if (a < ldexp(1.0, -126)) return ldexp(a, 133);
    int E;
    frexp(a, &E);
    return ldexp(a, 7 - (E - 1));
}

/* ------------------------------------------------------------------------------------------ */
/* Little-endian fp32 / u16 storage                                                           */
/* ------------------------------------------------------------------------------------------ */

static void store_f32(uint8_t *p, float f) { memcpy(p, &f, 4); }
static float load_f32(const uint8_t *p)
{
    float f;
    memcpy(&f, p, 4);
    return f;
}
static void store_u16(uint8_t *p, uint16_t h) { memcpy(p, &h, 2); }
static uint16_t load_u16(const uint8_t *p)
{
    uint16_t h;
    memcpy(&h, p, 2);
    return h;
}

/* The value a scale takes once stored in format sfmt (fp32 or bf16, round half to even). */
static double stored_scale(int sfmt, double v)
{
    if (sfmt == ORC_SCALE_BF16) return orc_bf16_to_double(orc_double_to_bf16(v));
    return (double)(float)v;
}
/* Distance of v from the nearest rounding tie of format sfmt, in quanta of that format. */
static double scale_tie_distance(int sfmt, double v)
{
    if (sfmt == ORC_SCALE_BF16) return tie_distance(bf16_units(v));
    int E;
    frexp(fabs(v), &E);
    return tie_distance(ldexp(fabs(v), 23 - (E - 1)));
}
static void store_scale(int sfmt, uint8_t *p, double v)
{
    if (sfmt == ORC_SCALE_BF16)
        store_u16(p, orc_double_to_bf16(v));
    else
        store_f32(p, (float)v);
}
static double load_scale(int sfmt, const uint8_t *p)
{
    return sfmt == ORC_SCALE_BF16 ? orc_bf16_to_double(load_u16(p)) : (double)load_f32(p);
}

/* ------------------------------------------------------------------------------------------ */
/* Quantizer: impact-weighted column scale, row scale from the column-normalised max,         */
/* round-half-to-even codes.                                                                  */
/*                                                                                            */
/* [P1 方法] and [P5 空间维度]: one scale per key row and one per value column, their product   */
/* sets the quantization step; the column scale is fitted by weighted least squares in which  */
/* high-impact rows weigh more; the two are fitted jointly.                                   */
/* Specification (READING c5/c6/c8: column first, then the row from the stored column scale,  */
/* one pass; fp32 storage, or bf16 in the 16-bit scale format):                               */
/*   W     = sum_i w_i                                                                        */
/*   c_j   = sqrt( sum_i w_i S_ij^2 / W ),   c_j := 1 if it is 0,   c~_j = stored(c_j)         */
/*   t_ij  = S_ij / c~_j                                                                      */
/*   r_i   = max_j |t_ij| / qmax,            r_i := 1 if it is 0,   r~_i = stored(r_i)         */
/*   x_ij  = t_ij / r~_i,  Q_ij = clamp(round_half_even(x_ij), -qmax, qmax)                   */
/* stored() rounds half to even to the format. With bf16 scales r~_i may sit just below r_i,  */
/* so |x| may pass qmax by a fraction of a step: the clamp takes it back.                     */
/* Pivot heads ([P1 方法], [P5 时间维度]: the highest-risk heads stay FP16): S -> fp16, RNE.    */
/* ------------------------------------------------------------------------------------------ */

static int check_weights(int dk, const double *w)
{
    for (int i = 0; i < dk; ++i)
        if (!(w[i] > 0.0) || !isfinite(w[i])) return ORC_EINVAL;
    return ORC_OK;
}

/* Quantize one head. sfmt: ORC_SCALE_F32 or ORC_SCALE_BF16. c_given / r_given (optional):
 * stored column / row scale values to use instead of fitting them (used by the tests to
 * requantize with the scales another implementation chose at a scale rounding near-tie).
 * stie_out (optional, dk + dv flags: rows, then columns): the fitted scale lay within `delta`
 * quanta of a rounding tie of the storage format. */
int orc_quantize_s(int bits, int sfmt, int dk, int dv, const double *S, const double *w,
                   const double *c_given, const double *r_given, uint8_t *block, double *x_out,
                   uint8_t *tie_out, uint8_t *stie_out, double delta)
{
    if (!valid_bits(bits) || !valid_sfmt(sfmt) || dk < 1 || dv < 1) return ORC_EINVAL;
    size_t n = (size_t)dk * dv;
    int nonfinite = 0;
    for (size_t e = 0; e < n; ++e)
        if (!isfinite(S[e])) nonfinite = 1;
    memset(block, 0, orc_block_bytes_s(bits, sfmt, dk, dv));
    if (stie_out) memset(stie_out, 0, (size_t)dk + (size_t)dv);

    if (bits == 16) {
        for (size_t e = 0; e < n; ++e) {
            uint16_t h = orc_double_to_half(S[e]);
            if ((h & 0x7c00) == 0x7c00) nonfinite = 1; /* overflow to inf, or NaN */
            store_u16(block + 2 * e, h);
            if (x_out) x_out[e] = half_units(S[e]);
            if (tie_out) tie_out[e] = tie_distance(half_units(S[e])) <= delta;
        }
        return nonfinite ? ORC_ENONFINITE : ORC_OK;
    }

    if (check_weights(dk, w) != ORC_OK) return ORC_EINVAL;
    int qmax = orc_qmax(bits);
    size_t soff = orc_scale_offset(bits, dk, dv);
    size_t sb = scale_bytes(sfmt);
    double *cs = (double *)malloc(sizeof(double) * dv);
    double *rs = (double *)malloc(sizeof(double) * dk);
    int32_t *u = (int32_t *)malloc(sizeof(int32_t) * n);

    double W = 0.0;
    for (int i = 0; i < dk; ++i) W += w[i];

    for (int j = 0; j < dv; ++j) {
        if (c_given) {
            cs[j] = c_given[j];
        } else {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += w[i] * S[(size_t)i * dv + j] * S[(size_t)i * dv + j];
            double c = sqrt(acc / W);
            if (c == 0.0) c = 1.0;
            cs[j] = stored_scale(sfmt, c);
            if (stie_out) stie_out[dk + j] = isfinite(c) && scale_tie_distance(sfmt, c) <= delta;
        }
        if (!isfinite(cs[j])) nonfinite = 1;
    }
    for (int i = 0; i < dk; ++i) {
        if (r_given) {
            rs[i] = r_given[i];
        } else {
            double m = 0.0;
            for (int j = 0; j < dv; ++j) {
                double t = fabs(S[(size_t)i * dv + j] / cs[j]);
                if (t > m) m = t;
            }
            double r = m / (double)qmax;
            if (r == 0.0) r = 1.0;
            rs[i] = stored_scale(sfmt, r);
            if (stie_out) stie_out[i] = isfinite(r) && scale_tie_distance(sfmt, r) <= delta;
        }
        if (!isfinite(rs[i]) || rs[i] == 0.0) nonfinite = 1;
    }
    for (int i = 0; i < dk; ++i) {
        for (int j = 0; j < dv; ++j) {
            size_t e = (size_t)i * dv + j;
            double x = (S[e] / cs[j]) / rs[i];
            double qv = orc_round_half_even(x);
            if (qv > qmax) qv = qmax;
            if (qv < -qmax) qv = -qmax;
            if (!isfinite(x)) qv = 0.0;
            u[e] = (int32_t)qv + (1 << (bits - 1));
            if (x_out) x_out[e] = x;
            if (tie_out) tie_out[e] = isfinite(x) ? (tie_distance(x) <= delta) : 0;
        }
    }
    orc_pack(bits, n, u, block);
    for (int i = 0; i < dk; ++i) store_scale(sfmt, block + soff + sb * (size_t)i, rs[i]);
    for (int j = 0; j < dv; ++j) store_scale(sfmt, block + soff + sb * ((size_t)dk + (size_t)j), cs[j]);
    free(cs);
    free(rs);
    free(u);
    return nonfinite ? ORC_ENONFINITE : ORC_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Impact-aware joint refinement of the two scales                                            */
/*                                                                                            */
/* [P5 空间维度]: the output error is the sum over key rows of each row's error weighted by a   */
/* coefficient whose mean square is the row impact score; the column scale is fitted by       */
/* weighted least squares in which high-impact rows weigh more; the row scale reflects the     */
/* row's magnitude and its impact; [P1 方法]: the two scales are fitted jointly.               */
/* READING c23: after the one-pass fit above, `rounds` rounds of alternating least squares on  */
/* the impact-weighted reconstruction error  E = sum_i w_i sum_j (S_ij - r_i c_j Q_ij)^2:      */
/*   c_j <- sum_i w_i r~_i Q_ij S_ij / sum_i w_i (r~_i Q_ij)^2        (codes Q of the last round) */
/*   r_i <- sum_j c~_j Q_ij S_ij / sum_j (c~_j Q_ij)^2                (new stored c~, same Q)    */
/*   Q_ij <- clamp(round_half_even((S_ij / c~_j) / r~_i), -qmax, qmax)                         */
/* each new scale stored (fp32 or bf16) before it is used; a scale whose denominator is 0, or  */
/* whose new value is not finite and positive, keeps its previous value. The weight of a row   */
/* multiplies all of that row's terms, so the row step does not depend on w_i: impact reaches */
/* the row scales through the jointly fitted column scales. With rounds = 0 this is the       */
/* one-pass quantizer.                                                                        */
/* ------------------------------------------------------------------------------------------ */

static void codes_with(int bits, int dk, int dv, const double *S, const double *cs, const double *rs, int32_t *Q)
{
    int qmax = orc_qmax(bits);
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) {
            size_t e = (size_t)i * dv + j;
            double x = (S[e] / cs[j]) / rs[i];
            double qv = orc_round_half_even(x);
            if (qv > qmax) qv = qmax;
            if (qv < -qmax) qv = -qmax;
            if (!isfinite(x)) qv = 0.0;
            Q[e] = (int32_t)qv;
        }
}

int orc_quantize_fit(int bits, int sfmt, int rounds, int dk, int dv, const double *S, const double *w,
                     uint8_t *block, double *x_out, uint8_t *tie_out, uint8_t *stie_out, double delta)
{
    if (rounds < 0) return ORC_EINVAL;
    int st = orc_quantize_s(bits, sfmt, dk, dv, S, w, NULL, NULL, block, x_out, tie_out, stie_out, delta);
    if (bits == 16 || rounds == 0 || st == ORC_EINVAL) return st;
    size_t n = (size_t)dk * dv;
    size_t soff = orc_scale_offset(bits, dk, dv);
    size_t sb = scale_bytes(sfmt);
    double *cs = (double *)malloc(sizeof(double) * dv);
    double *rs = (double *)malloc(sizeof(double) * dk);
    int32_t *Q = (int32_t *)malloc(sizeof(int32_t) * n);
    for (int i = 0; i < dk; ++i) rs[i] = load_scale(sfmt, block + soff + sb * (size_t)i);
    for (int j = 0; j < dv; ++j) cs[j] = load_scale(sfmt, block + soff + sb * ((size_t)dk + (size_t)j));
    if (stie_out) memset(stie_out, 0, (size_t)dk + (size_t)dv);
    for (int round = 0; round < rounds; ++round) {
        int last = round == rounds - 1;
        codes_with(bits, dk, dv, S, cs, rs, Q);
        for (int j = 0; j < dv; ++j) {
            double num = 0.0, den = 0.0;
            for (int i = 0; i < dk; ++i) {
                double a = rs[i] * (double)Q[(size_t)i * dv + j];
                num += w[i] * a * S[(size_t)i * dv + j];
                den += w[i] * a * a;
            }
            if (den > 0.0) {
                double c = stored_scale(sfmt, num / den);
                if (isfinite(c) && c > 0.0) cs[j] = c;
                if (last && stie_out) stie_out[dk + j] = scale_tie_distance(sfmt, num / den) <= delta;
            }
        }
        for (int i = 0; i < dk; ++i) {
            double num = 0.0, den = 0.0;
            for (int j = 0; j < dv; ++j) {
                double a = cs[j] * (double)Q[(size_t)i * dv + j];
                num += a * S[(size_t)i * dv + j];
                den += a * a;
            }
            if (den > 0.0) {
                double r = stored_scale(sfmt, num / den);
                if (isfinite(r) && r > 0.0) rs[i] = r;
                if (last && stie_out) stie_out[i] = scale_tie_distance(sfmt, num / den) <= delta;
            }
        }
    }
    st = orc_quantize_s(bits, sfmt, dk, dv, S, w, cs, rs, block, x_out, tie_out, NULL, delta);
    free(cs);
    free(rs);
    free(Q);
    return st;
}

int orc_quantize(int bits, int dk, int dv, const double *S, const double *w, uint8_t *block,
                 double *x_out, uint8_t *tie_out, double delta)
{
    return orc_quantize_s(bits, ORC_SCALE_F32, dk, dv, S, w, NULL, NULL, block, x_out, tie_out, NULL, delta);
}

/* Dequantize: S_ij = r~_i * c~_j * Q_ij (fp64), or the fp16 value of a pivot head. */
int orc_dequantize_s(int bits, int sfmt, int dk, int dv, const uint8_t *block, double *S)
{
    if (!valid_bits(bits) || !valid_sfmt(sfmt) || dk < 1 || dv < 1) return ORC_EINVAL;
    size_t n = (size_t)dk * dv;
    if (bits == 16) {
        for (size_t e = 0; e < n; ++e) S[e] = orc_half_to_double(load_u16(block + 2 * e));
        return ORC_OK;
    }
    size_t soff = orc_scale_offset(bits, dk, dv);
    int32_t *u = (int32_t *)malloc(sizeof(int32_t) * n);
    orc_unpack(bits, n, block, u);
    size_t sb = scale_bytes(sfmt);
    for (int i = 0; i < dk; ++i) {
        double r = load_scale(sfmt, block + soff + sb * (size_t)i);
        for (int j = 0; j < dv; ++j) {
            double c = load_scale(sfmt, block + soff + sb * ((size_t)dk + (size_t)j));
            size_t e = (size_t)i * dv + j;
            double qv = (double)(u[e] - (1 << (bits - 1)));
            S[e] = r * c * qv;
        }
    }
    free(u);
    return ORC_OK;
}

int orc_dequantize(int bits, int dk, int dv, const uint8_t *block, double *S)
{
    return orc_dequantize_s(bits, ORC_SCALE_F32, dk, dv, block, S);
}

/* ------------------------------------------------------------------------------------------ */
/* Gated delta rule update and readout                                                        */
/*                                                                                            */
/* [P5 intro] the models use the gated delta rule; [P5 直接量化为什么会翻车] every decode step  */
/* reads the previous state, updates it, requantizes and stores it. Specification:            */
/*   u   = k^T S                       (u_j = sum_i k_i S_ij)                                 */
/*   S'  = alpha (S - beta k u^T) + beta k v^T                                                */
/*   o   = S'^T q                      (o_j = sum_i q_i S'_ij; READING c3: after the update,   */
/*                                      before requantization)                                */
/* Channel gate ([P5 直接量化为什么会翻车] names Kimi's gating "KDA"; READING c2): alpha is a  */
/* vector over key rows. ORC_GATE_CHANNEL substitutes it literally, S'_ij = alpha_i (S_ij -   */
/* beta k_i u_j) + beta k_i v_j. ORC_GATE_CHANNEL_DECAY_FIRST decays first:                   */
/* u_j = sum_i k_i alpha_i S_ij, S'_ij = alpha_i S_ij - beta k_i u_j + beta k_i v_j.          */
/* ------------------------------------------------------------------------------------------ */

void orc_update(int dk, int dv, int gate, double *S, const double *q, const double *k,
                const double *v, double beta, const double *alpha, double *o)
{
    double *u = (double *)malloc(sizeof(double) * dv);
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) {
            double a = (gate == ORC_GATE_CHANNEL_DECAY_FIRST) ? alpha[i] : 1.0;
            acc += k[i] * a * S[(size_t)i * dv + j];
        }
        u[j] = acc;
    }
    for (int i = 0; i < dk; ++i) {
        double a = (gate == ORC_GATE_SCALAR) ? alpha[0] : alpha[i];
        for (int j = 0; j < dv; ++j) {
            size_t e = (size_t)i * dv + j;
            if (gate == ORC_GATE_CHANNEL_DECAY_FIRST)
                S[e] = a * S[e] - beta * k[i] * u[j] + beta * k[i] * v[j];
            else
                S[e] = a * (S[e] - beta * k[i] * u[j]) + beta * k[i] * v[j];
        }
    }
    if (o) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += q[i] * S[(size_t)i * dv + j];
            o[j] = acc;
        }
    }
    free(u);
}

/* One decode step on one head block, in place: dequantize -> update -> readout -> requantize.
 * o is emitted as fp32 (RNE of the fp64 value). S_new_out (optional) receives the fp64
 * updated state before requantization. x_out / tie_out (optional) receive the requantizer's
 * real-valued codes and near-tie flags. */
int orc_decode_step_s(int bits, int sfmt, int rounds, int dk, int dv, int gate, uint8_t *block, const double *q,
                      const double *k, const double *v, double beta, const double *alpha,
                      const double *w, float *o, double *S_new_out, double *x_out,
                      uint8_t *tie_out, uint8_t *stie_out, double delta)
{
    if (!valid_bits(bits) || !valid_sfmt(sfmt) || dk < 1 || dv < 1) return ORC_EINVAL;
    if (gate != ORC_GATE_SCALAR && gate != ORC_GATE_CHANNEL && gate != ORC_GATE_CHANNEL_DECAY_FIRST)
        return ORC_EINVAL;
    if (bits != 16 && check_weights(dk, w) != ORC_OK) return ORC_EINVAL;
    size_t n = (size_t)dk * dv;
    double *S = (double *)malloc(sizeof(double) * n);
    double *od = (double *)malloc(sizeof(double) * dv);
    orc_dequantize_s(bits, sfmt, dk, dv, block, S);
    orc_update(dk, dv, gate, S, q, k, v, beta, alpha, od);
    int nonfinite = 0;
    for (int j = 0; j < dv; ++j) {
        o[j] = (float)od[j];
        if (!isfinite(o[j])) nonfinite = 1;
    }
    if (S_new_out) memcpy(S_new_out, S, sizeof(double) * n);
    int st = orc_quantize_fit(bits, sfmt, rounds, dk, dv, S, w, block, x_out, tie_out, stie_out, delta);
    free(S);
    free(od);
    if (st != ORC_OK) return st;
    return nonfinite ? ORC_ENONFINITE : ORC_OK;
}

int orc_decode_step(int bits, int dk, int dv, int gate, uint8_t *block, const double *q,
                    const double *k, const double *v, double beta, const double *alpha,
                    const double *w, float *o, double *S_new_out, double *x_out,
                    uint8_t *tie_out, double delta)
{
    return orc_decode_step_s(bits, ORC_SCALE_F32, 0, dk, dv, gate, block, q, k, v, beta, alpha, w, o, S_new_out,
                             x_out, tie_out, NULL, delta);
}

/* ------------------------------------------------------------------------------------------ */
/* Chunked prefill, sequential form                                                           */
/*                                                                                            */
/* READING c16: tokens [0, T) of one call are cut into chunks [0,C), [C,2C), ... (the last may */
/* be short). Inside a chunk the state is not quantized; it is updated token by token with    */
/* the same rule as the decode step and o_t = S_t^T q_t is emitted for every token. At the    */
/* end of every chunk the state is requantized into the block.                                */
/* Layouts: q,k [T][dk], v [T][dv], beta [T], alpha [T] (scalar gate) or [T][dk], o [T][dv].  */
/* ------------------------------------------------------------------------------------------ */

int orc_prefill_seq_s(int bits, int sfmt, int rounds, int dk, int dv, int gate, uint8_t *block, int T, int chunk,
                      const double *q, const double *k, const double *v, const double *beta,
                      const double *alpha, const double *w, float *o, double *x_out,
                      uint8_t *tie_out, uint8_t *stie_out, double delta)
{
    if (!valid_bits(bits) || !valid_sfmt(sfmt) || dk < 1 || dv < 1 || T < 0 || chunk < 1) return ORC_EINVAL;
    if (bits != 16 && check_weights(dk, w) != ORC_OK) return ORC_EINVAL;
    size_t n = (size_t)dk * dv;
    int na = (gate == ORC_GATE_SCALAR) ? 1 : dk;
    double *S = (double *)malloc(sizeof(double) * n);
    double *od = (double *)malloc(sizeof(double) * dv);
    int status = ORC_OK;
    for (int c0 = 0; c0 < T; c0 += chunk) {
        int c1 = c0 + chunk < T ? c0 + chunk : T;
        orc_dequantize_s(bits, sfmt, dk, dv, block, S);
        for (int t = c0; t < c1; ++t) {
            orc_update(dk, dv, gate, S, q + (size_t)t * dk, k + (size_t)t * dk,
                       v + (size_t)t * dv, beta[t], alpha + (size_t)t * na, od);
            for (int j = 0; j < dv; ++j) {
                o[(size_t)t * dv + j] = (float)od[j];
                if (!isfinite(o[(size_t)t * dv + j])) status = ORC_ENONFINITE;
            }
        }
        int st = orc_quantize_fit(bits, sfmt, rounds, dk, dv, S, w, block, x_out, tie_out, stie_out, delta);
        if (st == ORC_EINVAL) status = st;
        if (st == ORC_ENONFINITE && status == ORC_OK) status = st;
    }
    free(S);
    free(od);
    return status;
}

int orc_prefill_seq(int bits, int dk, int dv, int gate, uint8_t *block, int T, int chunk,
                    const double *q, const double *k, const double *v, const double *beta,
                    const double *alpha, const double *w, float *o, double *x_out,
                    uint8_t *tie_out, double delta)
{
    return orc_prefill_seq_s(bits, ORC_SCALE_F32, 0, dk, dv, gate, block, T, chunk, q, k, v, beta, alpha, w, o,
                             x_out, tie_out, NULL, delta);
}

/* ------------------------------------------------------------------------------------------ */
/* Chunk algebra in WY / UT form (fp64, scalar gate, no quantization)                         */
/*                                                                                            */
/* Used only to cross-check the chunked algebra that a parallel prefill implements against    */
/* the token-by-token recurrence. With u_t = beta_t (v_t - alpha_t S_{t-1}^T k_t) the update   */
/* reads S_t = alpha_t S_{t-1} + k_t u_t^T. Let g_t = sum_{s<=t} log alpha_s (t = 1..C within  */
/* the chunk) and Gamma_ts = exp(g_t - g_s). Unrolling gives, for the chunk's C tokens:        */
/*   A_ts = Gamma_ts k_t.k_s (s < t),  T = (I + diag(beta) A)^-1  (forward substitution)      */
/*   W    = T diag(beta e^g) K,   U~ = T diag(beta) V,   U = U~ - W S0                        */
/*   P_ts = Gamma_ts q_t.k_s (s <= t)                                                         */
/*   O    = diag(e^g) Q S0 + P U                                                              */
/*   S_C  = e^{g_C} S0 + K^T diag(e^{g_C - g}) U                                              */
/* Layouts: S0/S_end [dk][dv], q,k [C][dk], v [C][dv], beta/alpha [C], O [C][dv].              */
/* ------------------------------------------------------------------------------------------ */

int orc_chunk_wy(int dk, int dv, int C, const double *S0, const double *q, const double *k,
                 const double *v, const double *beta, const double *alpha, double *S_end,
                 double *O)
{
    if (dk < 1 || dv < 1 || C < 1) return ORC_EINVAL;
    double *g = (double *)malloc(sizeof(double) * C);
    double *A = (double *)calloc((size_t)C * C, sizeof(double));
    double *Tm = (double *)calloc((size_t)C * C, sizeof(double));
    double *Wm = (double *)calloc((size_t)C * dk, sizeof(double));
    double *U = (double *)calloc((size_t)C * dv, sizeof(double));
    double *P = (double *)calloc((size_t)C * C, sizeof(double));
    double run = 0.0;
    for (int t = 0; t < C; ++t) {
        run += log(alpha[t]);
        g[t] = run;
    }
    for (int t = 0; t < C; ++t)
        for (int s = 0; s < t; ++s) {
            double kk = 0.0;
            for (int i = 0; i < dk; ++i) kk += k[(size_t)t * dk + i] * k[(size_t)s * dk + i];
            A[(size_t)t * C + s] = exp(g[t] - g[s]) * kk;
        }
    /* T = (I + diag(beta) A)^-1, lower triangular with unit diagonal: solve column by column
     * (I + diag(beta) A) T[:,c] = e_c by forward substitution. */
    for (int c = 0; c < C; ++c) {
        for (int t = 0; t < C; ++t) {
            double rhs = (t == c) ? 1.0 : 0.0;
            for (int s = 0; s < t; ++s) rhs -= beta[t] * A[(size_t)t * C + s] * Tm[(size_t)s * C + c];
            Tm[(size_t)t * C + c] = rhs;
        }
    }
    /* W = T diag(beta e^g) K ; U~ = T diag(beta) V ; U = U~ - W S0 */
    for (int t = 0; t < C; ++t) {
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int s = 0; s < C; ++s)
                acc += Tm[(size_t)t * C + s] * beta[s] * exp(g[s]) * k[(size_t)s * dk + i];
            Wm[(size_t)t * dk + i] = acc;
        }
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int s = 0; s < C; ++s) acc += Tm[(size_t)t * C + s] * beta[s] * v[(size_t)s * dv + j];
            double ws = 0.0;
            for (int i = 0; i < dk; ++i) ws += Wm[(size_t)t * dk + i] * S0[(size_t)i * dv + j];
            U[(size_t)t * dv + j] = acc - ws;
        }
    }
    for (int t = 0; t < C; ++t)
        for (int s = 0; s <= t; ++s) {
            double qk = 0.0;
            for (int i = 0; i < dk; ++i) qk += q[(size_t)t * dk + i] * k[(size_t)s * dk + i];
            P[(size_t)t * C + s] = exp(g[t] - g[s]) * qk;
        }
    if (O) {
        for (int t = 0; t < C; ++t)
            for (int j = 0; j < dv; ++j) {
                double qs = 0.0;
                for (int i = 0; i < dk; ++i) qs += q[(size_t)t * dk + i] * S0[(size_t)i * dv + j];
                double pu = 0.0;
                for (int s = 0; s <= t; ++s) pu += P[(size_t)t * C + s] * U[(size_t)s * dv + j];
                O[(size_t)t * dv + j] = exp(g[t]) * qs + pu;
            }
    }
    if (S_end) {
        double gC = g[C - 1];
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double acc = exp(gC) * S0[(size_t)i * dv + j];
                for (int s = 0; s < C; ++s)
                    acc += k[(size_t)s * dk + i] * exp(gC - g[s]) * U[(size_t)s * dv + j];
                S_end[(size_t)i * dv + j] = acc;
            }
    }
    free(g);
    free(A);
    free(Tm);
    free(Wm);
    free(U);
    free(P);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Uniform baseline quantizer: one scale per head                                             */
/*                                                                                            */
/* [P5 直接量化为什么会翻车 / 数据说话] and [P1 實驗結果]: the pages compare the method with     */
/* uniform INT quantization of the state ("统一INT8"), the direct approach whose errors        */
/* accumulate. Reading: symmetric per-head (per-tensor) INT quantization with the method's     */
/* code range and rounding, fp32 scale:                                                        */
/*   s = max_ij |S_ij| / qmax,  s := 1 if it is 0,  s~ = fp32(s)                               */
/*   x_ij = S_ij / s~,  Q_ij = clamp(round_half_even(x_ij), -qmax, qmax)                       */
/* Block: the codes bitstream as for the method, zero padding to 16 bytes, s~ (fp32), zero    */
/* padding to 128 bytes.                                                                       */
/* ------------------------------------------------------------------------------------------ */

size_t orc_uniform_block_bytes(int bits, int dk, int dv)
{
    return round_up(orc_scale_offset(bits, dk, dv) + 4, 128);
}

int orc_quantize_uniform(int bits, int dk, int dv, const double *S, uint8_t *block, double *x_out,
                         uint8_t *tie_out, double delta)
{
    if (!(bits == 4 || bits == 6 || bits == 8) || dk < 1 || dv < 1) return ORC_EINVAL;
    size_t n = (size_t)dk * dv;
    int nonfinite = 0;
    double m = 0.0;
    for (size_t e = 0; e < n; ++e) {
        if (!isfinite(S[e])) nonfinite = 1;
        if (fabs(S[e]) > m) m = fabs(S[e]);
    }
    memset(block, 0, orc_uniform_block_bytes(bits, dk, dv));
    int qmax = orc_qmax(bits);
    double s = m / (double)qmax;
    if (s == 0.0) s = 1.0;
    float sf = (float)s;
    if (!isfinite(sf) || sf == 0.0f) nonfinite = 1;
    int32_t *u = (int32_t *)malloc(sizeof(int32_t) * n);
    for (size_t e = 0; e < n; ++e) {
        double x = S[e] / (double)sf;
        double qv = orc_round_half_even(x);
        if (qv > qmax) qv = qmax;
        if (qv < -qmax) qv = -qmax;
        if (!isfinite(x)) qv = 0.0;
        u[e] = (int32_t)qv + (1 << (bits - 1));
        if (x_out) x_out[e] = x;
        if (tie_out) tie_out[e] = isfinite(x) ? (tie_distance(x) <= delta) : 0;
    }
    orc_pack(bits, n, u, block);
    store_f32(block + orc_scale_offset(bits, dk, dv), sf);
    free(u);
    return nonfinite ? ORC_ENONFINITE : ORC_OK;
}

int orc_dequantize_uniform(int bits, int dk, int dv, const uint8_t *block, double *S)
{
    if (!(bits == 4 || bits == 6 || bits == 8) || dk < 1 || dv < 1) return ORC_EINVAL;
    size_t n = (size_t)dk * dv;
    int32_t *u = (int32_t *)malloc(sizeof(int32_t) * n);
    orc_unpack(bits, n, block, u);
    double s = (double)load_f32(block + orc_scale_offset(bits, dk, dv));
    for (size_t e = 0; e < n; ++e) S[e] = s * (double)(u[e] - (1 << (bits - 1)));
    free(u);
    return ORC_OK;
}

/* One decode step of a uniformly quantized head: dequantize -> update -> readout -> requantize. */
int orc_decode_step_uniform(int bits, int dk, int dv, int gate, uint8_t *block, const double *q,
                            const double *k, const double *v, double beta, const double *alpha,
                            float *o, double *x_out, uint8_t *tie_out, double delta)
{
    if (!(bits == 4 || bits == 6 || bits == 8) || dk < 1 || dv < 1) return ORC_EINVAL;
    if (gate != ORC_GATE_SCALAR && gate != ORC_GATE_CHANNEL && gate != ORC_GATE_CHANNEL_DECAY_FIRST)
        return ORC_EINVAL;
    size_t n = (size_t)dk * dv;
    double *S = (double *)malloc(sizeof(double) * n);
    double *od = (double *)malloc(sizeof(double) * dv);
    orc_dequantize_uniform(bits, dk, dv, block, S);
    orc_update(dk, dv, gate, S, q, k, v, beta, alpha, od);
    int nonfinite = 0;
    for (int j = 0; j < dv; ++j) {
        o[j] = (float)od[j];
        if (!isfinite(o[j])) nonfinite = 1;
    }
    int st = orc_quantize_uniform(bits, dk, dv, S, block, x_out, tie_out, delta);
    free(S);
    free(od);
    if (st != ORC_OK) return st;
    return nonfinite ? ORC_ENONFINITE : ORC_OK;
}
