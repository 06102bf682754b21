/*
 * qfp4_oracle.c -- plain single-threaded CPU oracle (TEST INFRASTRUCTURE ONLY;
 * see qfp4_oracle.h for who may call it and for the page citations).
 *
 * Written for a reader checking it against the pages: every step is scalar,
 * in the order the pages state it, with no blocking, fusion or reordering.
 * Build: gcc -O2 -std=c11 -ffp-contract=off (no -ffast-math).
 */
#include "qfp4_oracle.h"

#include <assert.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ========================================================================
 * E2M1 (FP4).  [LB] §FP4: 1 sign bit, 2 exponent bits, 1 mantissa bit; the
 * representable values are +-{0.5,1,1.5,2,3,4,6} and 0, range [-6,6].
 * Decoded here from the bit fields (exponent bias 1, subnormal when the
 * exponent field is 0); a test pins the 16 codes to the page's 15 values.
 * ====================================================================== */
float or_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, E = (code >> 1) & 3, m = code & 1;
    double mag = (E == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, E - 1);
    return (float)(s ? -mag : mag);
}

/* Round to the nearest grid value; a tie goes to the code whose mantissa bit
 * is 0 (the IEEE tie rule carried to E2M1, a reading: the page only says
 * "nearest grid point", [LB] §6).  Values beyond 6 take 6 (the nearest
 * finite value, range [-6,6]).  The sign bit is copied from v. */
uint8_t or_e2m1_rne(float v)
{
    assert(isfinite(v));
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(sign | 7);        /* range [-6, 6]      */
    int best = 0;
    double bd = a;                                   /* distance to 0; all
                                      distances below are exact in binary64 */
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - (double)or_e2m1_value((uint8_t)c));
        if (d < bd || (d == bd && (best & 1) && !(c & 1))) { best = c; bd = d; }
    }
    return (uint8_t)(sign | best);
}

/* Stochastic rounding ([QN] stochastic-rounding kernel; [TI] "stochastic
 * rounding ... unbiased gradients"): with lo <= |v| < hi adjacent grid
 * values, round up with probability p = (|v|-lo)/(hi-lo).  The uniform draw
 * is u = (r >> 8) * 2^-24 from one 32-bit random word; up iff u < p. */
uint8_t or_e2m1_sr(float v, uint32_t r)
{
    assert(isfinite(v));
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(sign | 7);
    int c = 0;
    while (c < 6 && (double)or_e2m1_value((uint8_t)(c + 1)) <= a) ++c;
    double lo = or_e2m1_value((uint8_t)c), hi = or_e2m1_value((uint8_t)(c + 1));
    double p = (a - lo) / (hi - lo);
    double u = ldexp((double)(r >> 8), -24);
    return (uint8_t)(sign | (u < p ? c + 1 : c));
}

/* ========================================================================
 * E4M3 (OCP FP8): bias 7, 3 mantissa bits, no infinities, 0x7F/0xFF NaN,
 * largest finite 448, subnormals m * 2^-9.  The pages name NVFP4 and MXFP8
 * ([QN] §QuTLASS, [TI] abstract, [46]) without giving the bits; this is the
 * public OCP definition.
 * ====================================================================== */
float or_e4m3_value(uint8_t b)
{
    int s = b >> 7, E = (b >> 3) & 15, m = b & 7;
    if (E == 15 && m == 7) return NAN;
    double mag = (E == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), E - 10);
    return (float)(s ? -mag : mag);
}

/* bracket |v| between consecutive non-negative finite E4M3 bytes lo, lo+1 */
static int e4m3_floor_byte(double a)
{
    int lo = 0, hi = 126;                            /* value(126) = 448 > a */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if ((double)or_e4m3_value((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    return lo;
}

/* nearest finite E4M3 value, ties to the even byte (mantissa LSB 0),
 * saturating to +-448 (satfinite); sign copied from v */
uint8_t or_e4m3_rne(float v)
{
    assert(isfinite(v));
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = e4m3_floor_byte(a), hi = lo + 1;
    double dl = a - (double)or_e4m3_value((uint8_t)lo);
    double dh = (double)or_e4m3_value((uint8_t)hi) - a;
    int pick = dl < dh ? lo : (dh < dl ? hi : ((lo & 1) == 0 ? lo : hi));
    return (uint8_t)(sign | pick);
}

/* the stochastic rule of or_e2m1_sr on the E4M3 grid, saturating at 448 */
uint8_t or_e4m3_sr(float v, uint32_t r)
{
    assert(isfinite(v));
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = e4m3_floor_byte(a);
    double vlo = or_e4m3_value((uint8_t)lo), vhi = or_e4m3_value((uint8_t)(lo + 1));
    double p = (a - vlo) / (vhi - vlo);
    double u = ldexp((double)(r >> 8), -24);
    return (uint8_t)(sign | (u < p ? lo + 1 : lo));
}

/* E4M3 rounded up: the least finite E4M3 value >= |v| (the truncation-free
 * rule of [TI] applied to the NVFP4 block scale, so that S >= amax_b / 6 and
 * no element of the block clips), saturating at 448; sign copied from v. */
uint8_t or_e4m3_up(float v)
{
    assert(isfinite(v));
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = e4m3_floor_byte(a);
    return (uint8_t)(sign | ((double)or_e4m3_value((uint8_t)lo) == a ? lo : lo + 1));
}

/* E8M0 ([LB] §3: an 8-bit exponent, scale 2^k only) */
double or_e8m0_value(uint8_t b)
{
    if (b == 255) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* Truncation-free power-of-two scale ([TI] "truncation-free scaling";
 * exponent 2^ceil(log2(amax/top))): the least integer k in [-127,127] with
 * top * 2^k >= amax, found by exact comparison.  top = 6 for E2M1 ([LB]
 * §FP4, S = |W|max/6 never clips), 448 for E4M3. amax = 0 gives -127. */
int or_scale_exp(float amax, double top)
{
    assert(isfinite(amax) && amax >= 0.0f);
    for (int k = -127; k <= 127; ++k)
        if (ldexp(top, k) >= (double)amax) return k;
    return 127;
}

/* The OCP MX rule for the shared exponent (the "2^k scale" of [LB] §3 with
 * its rounding direction taken from the OCP microscaling definition, as the
 * ablation next to [TI]'s truncation-free rule): k = floor(log2(amax)) -
 * emax, emax = 2 for E2M1 (largest value 6 = 1.5 * 2^2), i.e. the largest k
 * with 2^(k + emax) <= amax, clamped to [-127, 127].  amax / 2^k lies in
 * [4, 8), so values above 6 * 2^k are clipped to 6 (saturation).  amax = 0
 * gives -127. */
int or_scale_exp_floor(float amax, int emax)
{
    assert(isfinite(amax) && amax >= 0.0f);
    for (int k = 127; k >= -127; --k)
        if (ldexp(1.0, k + emax) <= (double)amax) return k;
    return -127;
}

/* ========================================================================
 * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC'11): 10 rounds of the 4x32 Philox S-box with
 * multipliers 0xD2511F53, 0xCD9E8D57 and Weyl key increments 0x9E3779B9,
 * 0xBB67AE85.
 * ====================================================================== */
static void mulhilo32(uint32_t a, uint32_t b, uint32_t *hi, uint32_t *lo)
{
    uint64_t p = (uint64_t)a * (uint64_t)b;
    *hi = (uint32_t)(p >> 32);
    *lo = (uint32_t)p;
}

void or_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint32_t hi0, lo0, hi1, lo1;
        mulhilo32(0xD2511F53u, c0, &hi0, &lo0);
        mulhilo32(0xCD9E8D57u, c2, &hi1, &lo1);
        uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Random word of element e (logical row-major index i*K+j): Philox keyed
 * on the seed, counter = e/4 (64 bits over the first two counter words),
 * output word e mod 4. */
uint32_t or_sr_word(uint64_t seed, uint64_t e)
{
    uint64_t c = e >> 2;
    uint32_t ctr[4] = {(uint32_t)c, (uint32_t)(c >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    or_philox4x32_10(ctr, key, out);
    return out[e & 3];
}

/* ========================================================================
 * Fast Walsh-Hadamard transform of one 128-element block ([QN] Hadamard
 * rotation; [LB] §7: H has +-1 entries divided by sqrt(n), O(n log n)).
 * Sylvester (natural) order, H[i][j] = (-1)^popcount(i&j) / sqrt(128).
 * Stages h = 1,2,4,...,64; each pair (i, i+h) with (i & h) == 0 becomes
 * (a+b, a-b) in binary32; then every entry is multiplied once by the
 * binary32 value nearest 2^-3.5 = 1/sqrt(128).
 * ====================================================================== */
void or_fwht128(float *x)
{
    for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; ++i)
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
    const float c = (float)(1.0 / sqrt(128.0));
    for (int i = 0; i < 128; ++i) x[i] = x[i] * c;
}

float or_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float load_elem(const void *x, int xdt, int64_t idx)
{
    if (xdt == OR_BF16) return or_bf16_to_f32(((const uint16_t *)x)[idx]);
    return ((const float *)x)[idx];
}

/* row i of X as binary32, rotated block by block when asked */
static void load_row(const void *x, int xdt, int64_t K, int64_t i, int rotate, float *row)
{
    for (int64_t j = 0; j < K; ++j) {
        row[j] = load_elem(x, xdt, i * K + j);
        assert(isfinite(row[j]));
    }
    if (rotate)
        for (int64_t b = 0; b < K; b += 128) or_fwht128(row + b);
}

static void put_nibble(uint8_t *buf, int64_t idx, uint8_t code)
{
    uint8_t *p = buf + (idx >> 1);
    if (idx & 1) *p = (uint8_t)((*p & 0x0F) | (code << 4));
    else         *p = (uint8_t)((*p & 0xF0) | (code & 0x0F));
}

static uint8_t fp4_round(float v, int rounding, uint64_t seed, uint64_t e)
{
    return rounding == OR_SR ? or_e2m1_sr(v, or_sr_word(seed, e)) : or_e2m1_rne(v);
}

/* ========================================================================
 * NVFP4 two-level scale.  The pages give the idea (a fine group scale under
 * one per-tensor FP scale, [LB] §3 VS-Quant; NVFP4 named in [QN], [46]);
 * the formula taken: per-tensor s_t = amax_t / (6*448) in binary32, and the
 * block scale byte enc = E4M3((amax_b / d) / s_t) with d = 6 (d = 4 for the
 * four-over-six candidate), rounded to nearest (default rule) or up (the
 * truncation-free rule), saturating at 448.  The effective block scale used
 * to divide is S = dec(enc) * s_t in binary32.
 * ====================================================================== */
static uint8_t nv_enc(float amax_b, float s_t, float d, int rule)
{
    float q = amax_b / d;
    float r = q / s_t;
    if (!(r < 448.0f)) return 0x7E;               /* 448 and beyond, incl. +inf */
    return rule == OR_RULE_E4M3_UP ? or_e4m3_up(r) : or_e4m3_rne(r);
}

static float nv_seff(uint8_t enc, float s_t)
{
    return or_e4m3_value(enc) * s_t;
}

/* E2M1 code of v = x / S; a quotient that overflowed binary32 (a tiny S)
 * saturates like any magnitude beyond 6. */
static uint8_t fp4_code(float v, int rounding, uint64_t seed, uint64_t e)
{
    if (isinf(v)) return (uint8_t)((signbit(v) ? 8 : 0) | 7);
    return fp4_round(v, rounding, seed, e);
}

/* quantize n values x[] (logical indices e[]) under effective scale S;
 * S == 0 (an all-zero or underflowed block) gives +0 codes. */
static void quant_block(const float *x, const uint64_t *e, int n, float S,
                        int rounding, uint64_t seed, uint8_t *codes)
{
    for (int t = 0; t < n; ++t) {
        if (S == 0.0f) { codes[t] = 0; continue; }
        float v = x[t] / S;
        codes[t] = fp4_code(v, rounding, seed, e[t]);
    }
}

/* Four-over-six ([46] Methodology 1-3): two candidate scales per block, the
 * standard one (amax/6) and a smaller-range one (amax/4); quantize with each
 * (round to nearest) and keep the one with the lower block squared error.
 * Readings: block = the NVFP4 16-element block (the MXFP4 32-element group
 * for the MXFP4 variant); error = sum over the block of (deq - x)^2 in
 * binary32 with deq = value(code) * S, summed as a fixed tree (pairs i,
 * i + n/2; then halves again down to 1); a tie keeps the standard scale. */
static float block_sse(const float *x, const uint8_t *codes, float S, int n)
{
    float e[32];
    for (int i = 0; i < n; ++i) {
        float deq = or_e2m1_value(codes[i]) * S;
        float d = deq - x[i];
        e[i] = d * d;
    }
    for (int h = n / 2; h >= 1; h >>= 1)
        for (int i = 0; i < h; ++i) e[i] = e[i] + e[i + h];
    return e[0];
}

static int nv_four6(const float *x16, float s_t, int rule, uint8_t *enc_out, uint8_t codes_out[16])
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x16[i]));
    uint64_t e[16] = {0};                         /* unused by RNE */
    uint8_t enc6 = nv_enc(amax, s_t, 6.0f, rule), enc4 = nv_enc(amax, s_t, 4.0f, rule);
    float S6 = nv_seff(enc6, s_t), S4 = nv_seff(enc4, s_t);
    uint8_t c6[16], c4[16];
    quant_block(x16, e, 16, S6, OR_RNE, 0, c6);
    quant_block(x16, e, 16, S4, OR_RNE, 0, c4);
    float sse6 = block_sse(x16, c6, S6, 16), sse4 = block_sse(x16, c4, S4, 16);
    int pick4 = sse4 < sse6;
    *enc_out = pick4 ? enc4 : enc6;
    memcpy(codes_out, pick4 ? c4 : c6, 16);
    return pick4;
}

int or_four6_pick(const float *x16, float s_t, uint8_t *enc_out, uint8_t codes_out[16])
{
    return nv_four6(x16, s_t, OR_RULE_DEFAULT, enc_out, codes_out);
}

/* MXFP4 group exponent under a scale rule: truncation-free ([TI]) by
 * default, the OCP floor rule as the ablation. */
static int mx_exp(float amax, int rule)
{
    return rule == OR_RULE_OCP_FLOOR ? or_scale_exp_floor(amax, 2) : or_scale_exp(amax, 6.0);
}

/* One MXFP4 group of 32: scale byte and codes.  With four6, the second
 * candidate is the least k4 with 4 * 2^k4 >= amax ([46]'s amax/4 scale
 * carried to power-of-two scales); the group keeps the candidate with the
 * lower block squared error (RNE), a tie keeps the rule's exponent.  An
 * all-zero group gives byte 0 and +0 codes. */
int or_mxfp4_group(const float *xg, const uint64_t *eg, int rounding, int four6, int rule,
                   uint64_t seed, uint8_t *sbyte, uint8_t cg[32])
{
    float amax = 0.0f;
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(xg[t]));
    if (amax == 0.0f) {
        *sbyte = 0;
        memset(cg, 0, 32);
        return 0;
    }
    int k = mx_exp(amax, rule), pick4 = 0;
    quant_block(xg, eg, 32, (float)ldexp(1.0, k), rounding, seed, cg);
    if (four6) {
        int k4 = or_scale_exp(amax, 4.0);
        uint8_t c4[32];
        quant_block(xg, eg, 32, (float)ldexp(1.0, k4), OR_RNE, 0, c4);
        float sse = block_sse(xg, cg, (float)ldexp(1.0, k), 32);
        float sse4 = block_sse(xg, c4, (float)ldexp(1.0, k4), 32);
        if (sse4 < sse) {
            k = k4;
            memcpy(cg, c4, 32);
            pick4 = 1;
        }
    }
    *sbyte = (uint8_t)(k + 127);
    return pick4;
}

/* ========================================================================
 * qfp4_quantize semantics.
 * ====================================================================== */
static int check_quantize_args(const void *x, int xdt, int64_t M, int64_t K, int fmt,
                               int rounding, int rotate, int block2d, int four6, int rule,
                               int64_t row0, const float *amax_in, const float *amax_out,
                               const uint8_t *codes, const uint8_t *scales,
                               const uint8_t *codesT, const uint8_t *scalesT,
                               const float *tscale)
{
    if (M < 0 || K < 0) return OR_ERR_SHAPE;
    if (fmt != OR_MXFP4 && fmt != OR_NVFP4) return OR_ERR_ARG;
    if (rounding != OR_RNE && rounding != OR_SR) return OR_ERR_ARG;
    if (xdt != OR_BF16 && xdt != OR_F32) return OR_ERR_ARG;
    if (rule < OR_RULE_DEFAULT || rule > OR_RULE_E4M3_UP || row0 < 0) return OR_ERR_ARG;
    if ((M * K > 0) && (!x || !codes || !scales)) return OR_ERR_ARG;
    if ((codesT == NULL) != (scalesT == NULL)) return OR_ERR_ARG;
    if (fmt == OR_NVFP4 && !tscale) return OR_ERR_ARG;
    int g = fmt == OR_MXFP4 ? 32 : 16;
    if (rule == OR_RULE_OCP_FLOOR && fmt != OR_MXFP4) return OR_ERR_UNSUPPORTED;
    if (rule == OR_RULE_E4M3_UP && fmt != OR_NVFP4) return OR_ERR_UNSUPPORTED;
    if ((amax_in || amax_out) && fmt != OR_NVFP4) return OR_ERR_UNSUPPORTED;
    if (four6 && (block2d || rounding != OR_RNE)) return OR_ERR_UNSUPPORTED;
    if (four6 && fmt == OR_MXFP4 && codesT) return OR_ERR_UNSUPPORTED;
    if (block2d && rotate) return OR_ERR_UNSUPPORTED;
    if (!block2d && rotate && codesT) return OR_ERR_UNSUPPORTED;
    if (row0 && (block2d || codesT)) return OR_ERR_UNSUPPORTED;
    if (K % g) return OR_ERR_SHAPE;
    if (rotate && K % 128) return OR_ERR_SHAPE;
    if (block2d && (M % g || K % g)) return OR_ERR_SHAPE;
    if (!block2d && codesT && M % g) return OR_ERR_SHAPE;
    return OR_OK;
}

/* per-tensor amax of the (rotated) input */
static float tensor_amax(const void *x, int xdt, int64_t M, int64_t K, int rotate, float *row)
{
    float amax_t = 0.0f;
    for (int64_t i = 0; i < M; ++i) {
        load_row(x, xdt, K, i, rotate, row);
        for (int64_t j = 0; j < K; ++j) amax_t = fmaxf(amax_t, fabsf(row[j]));
    }
    return amax_t;
}

float or_tensor_amax(const void *x, int xdt, int64_t M, int64_t K, int rotate)
{
    if (M <= 0 || K <= 0) return 0.0f;
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    if (!row) return NAN;
    float a = tensor_amax(x, xdt, M, K, rotate, row);
    free(row);
    return a;
}

/* 1D groups of g along K for one row (MXFP4 or NVFP4, optional 4/6); the
 * row's logical index is i (random words keyed on i*K + j), its outputs go
 * to local row il of codes / scales */
static void quantize_row_1d(const float *row, int64_t i, int64_t il, int64_t K, int fmt, int rounding,
                            int four6, int rule, uint64_t seed, float s_t,
                            uint8_t *codes, uint8_t *scales)
{
    int g = fmt == OR_MXFP4 ? 32 : 16;
    float xg[32];
    uint64_t eg[32];
    uint8_t cg[32];
    for (int64_t j0 = 0; j0 < K; j0 += g) {
        float amax = 0.0f;
        for (int t = 0; t < g; ++t) {
            xg[t] = row[j0 + t];
            eg[t] = (uint64_t)(i * K + j0 + t);
            amax = fmaxf(amax, fabsf(xg[t]));
        }
        uint8_t sbyte;
        if (fmt == OR_MXFP4) {
            or_mxfp4_group(xg, eg, rounding, four6, rule, seed, &sbyte, cg);
        } else if (four6) {
            nv_four6(xg, s_t, rule, &sbyte, cg);
        } else {
            sbyte = nv_enc(amax, s_t, 6.0f, rule);
            quant_block(xg, eg, g, nv_seff(sbyte, s_t), rounding, seed, cg);
        }
        scales[il * (K / g) + j0 / g] = sbyte;
        for (int t = 0; t < g; ++t) put_nibble(codes, il * K + j0 + t, cg[t]);
    }
}

int or_quantize_ex(const void *x, int xdt, int64_t M, int64_t K,
                   int fmt, int rounding, int rotate, int block2d, int four6, int rule,
                   uint64_t seed, int64_t row0, const float *amax_in,
                   uint8_t *codes, uint8_t *scales,
                   uint8_t *codesT, uint8_t *scalesT,
                   float *tscale, float *amax_out)
{
    int st = check_quantize_args(x, xdt, M, K, fmt, rounding, rotate, block2d, four6, rule, row0,
                                 amax_in, amax_out, codes, scales, codesT, scalesT, tscale);
    if (st != OR_OK) return st;
    if (M == 0 || K == 0) {
        if (fmt == OR_NVFP4) *tscale = amax_in ? *amax_in / 2688.0f : 0.0f;
        if (amax_out) *amax_out = 0.0f;
        return OR_OK;
    }
    int g = fmt == OR_MXFP4 ? 32 : 16;
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    if (!row) return OR_ERR_ARG;

    float s_t = 0.0f;
    if (fmt == OR_NVFP4) {
        /* the tensor scale from this tensor's own amax, or (delayed scaling,
         * [QN] open questions: an EMA / history of activation scales) from an
         * amax the caller supplies */
        if (!amax_in || amax_out) {
            float own = tensor_amax(x, xdt, M, K, rotate, row);
            if (amax_out) *amax_out = own;
            s_t = own / 2688.0f;                   /* 6 * 448 */
        }
        if (amax_in) s_t = *amax_in / 2688.0f;
        *tscale = s_t;
        if (s_t == 0.0f) {                /* all-zero (or underflowed) tensor scale */
            memset(codes, 0, (size_t)(M * K / 2));
            memset(scales, 0, (size_t)(M * (K / g)));
            if (codesT) {
                memset(codesT, 0, (size_t)(M * K / 2));
                memset(scalesT, 0, (size_t)(K * (M / g)));
            }
            free(row);
            return OR_OK;
        }
    }

    if (block2d) {
        /* [TI]: 2D blocks (the group size on both axes: 16x16 NVFP4, 32x32
         * MXFP4) so that X and X^T share one scale per block; codesT is the
         * transpose of codes. */
        int T = g;
        float *tile = (float *)malloc(sizeof(float) * 1024);
        uint64_t *et = (uint64_t *)malloc(sizeof(uint64_t) * 1024);
        uint8_t *ct = (uint8_t *)malloc(1024);
        for (int64_t bi = 0; bi < M; bi += T)
            for (int64_t bj = 0; bj < K; bj += T) {
                float amax = 0.0f;
                for (int r = 0; r < T; ++r)
                    for (int c = 0; c < T; ++c) {
                        int64_t e = (bi + r) * K + bj + c;
                        tile[r * T + c] = load_elem(x, xdt, e);
                        et[r * T + c] = (uint64_t)e;
                        amax = fmaxf(amax, fabsf(tile[r * T + c]));
                    }
                uint8_t enc;
                float S;
                if (fmt == OR_MXFP4) {
                    int k = amax == 0.0f ? -127 : mx_exp(amax, rule);
                    enc = amax == 0.0f ? 0 : (uint8_t)(k + 127);
                    S = amax == 0.0f ? 0.0f : (float)ldexp(1.0, k);
                } else {
                    enc = nv_enc(amax, s_t, 6.0f, rule);
                    S = nv_seff(enc, s_t);
                }
                quant_block(tile, et, T * T, S, rounding, seed, ct);
                for (int r = 0; r < T; ++r)
                    for (int c = 0; c < T; ++c) {
                        int64_t i = bi + r, j = bj + c;
                        put_nibble(codes, i * K + j, ct[r * T + c]);
                        if (codesT) put_nibble(codesT, j * M + i, ct[r * T + c]);
                    }
                for (int r = 0; r < T; ++r) scales[(bi + r) * (K / T) + bj / T] = enc;
                if (scalesT)
                    for (int c = 0; c < T; ++c) scalesT[(bj + c) * (M / T) + bi / T] = enc;
            }
        free(tile);
        free(et);
        free(ct);
        free(row);
        return OR_OK;
    }

    for (int64_t i = 0; i < M; ++i) {
        load_row(x, xdt, K, i, rotate, row);
        quantize_row_1d(row, row0 + i, i, K, fmt, rounding, four6, rule, seed, s_t, codes, scales);
    }

    if (codesT) {
        /* [TI]'s 1D baseline for X^T: an independent quantization of each
         * column with groups of g along M; random words keyed on X's index. */
        float xg[32];
        uint64_t eg[32];
        uint8_t cg[32];
        for (int64_t j = 0; j < K; ++j)
            for (int64_t i0 = 0; i0 < M; i0 += g) {
                float amax = 0.0f;
                for (int t = 0; t < g; ++t) {
                    xg[t] = load_elem(x, xdt, (i0 + t) * K + j);
                    eg[t] = (uint64_t)((i0 + t) * K + j);
                    amax = fmaxf(amax, fabsf(xg[t]));
                }
                uint8_t sbyte;
                if (fmt == OR_MXFP4) {
                    or_mxfp4_group(xg, eg, rounding, four6, rule, seed, &sbyte, cg);
                } else if (four6) {
                    nv_four6(xg, s_t, rule, &sbyte, cg);
                } else {
                    sbyte = nv_enc(amax, s_t, 6.0f, rule);
                    quant_block(xg, eg, g, nv_seff(sbyte, s_t), rounding, seed, cg);
                }
                scalesT[j * (M / g) + i0 / g] = sbyte;
                for (int t = 0; t < g; ++t) put_nibble(codesT, j * M + i0 + t, cg[t]);
            }
    }
    free(row);
    return OR_OK;
}

int or_quantize(const void *x, int xdt, int64_t M, int64_t K,
                int fmt, int rounding, int rotate, int block2d, int four6,
                uint64_t seed,
                uint8_t *codes, uint8_t *scales,
                uint8_t *codesT, uint8_t *scalesT,
                float *tscale)
{
    return or_quantize_ex(x, xdt, M, K, fmt, rounding, rotate, block2d, four6, OR_RULE_DEFAULT, seed, 0,
                          NULL, codes, scales, codesT, scalesT, tscale, NULL);
}

/* ========================================================================
 * MXFP8: E4M3 elements in groups of 32 under an E8M0 scale, truncation-free
 * k = least k with 448 * 2^k >= amax ([TI]: MXFP8 for the sensitive Q/K
 * projections; [QN]: FP8 backward).  codesT, when given, is the column-wise
 * quantization (groups of 32 along M), K x M codes.
 * ====================================================================== */
static void mxfp8_group(const float *xg, const uint64_t *eg, int rounding, uint64_t seed,
                        uint8_t *sbyte, uint8_t *cg)
{
    float amax = 0.0f;
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(xg[t]));
    if (amax == 0.0f) {
        *sbyte = 0;
        memset(cg, 0, 32);
        return;
    }
    int k = or_scale_exp(amax, 448.0);
    *sbyte = (uint8_t)(k + 127);
    float S = (float)ldexp(1.0, k);
    for (int t = 0; t < 32; ++t) {
        float v = xg[t] / S;
        cg[t] = rounding == OR_SR ? or_e4m3_sr(v, or_sr_word(seed, eg[t])) : or_e4m3_rne(v);
    }
}

int or_quantize_mxfp8(const void *x, int xdt, int64_t M, int64_t K,
                      int rounding, uint64_t seed,
                      uint8_t *codes, uint8_t *scales,
                      uint8_t *codesT, uint8_t *scalesT)
{
    if (M < 0 || K < 0) return OR_ERR_SHAPE;
    if (rounding != OR_RNE && rounding != OR_SR) return OR_ERR_ARG;
    if (xdt != OR_BF16 && xdt != OR_F32) return OR_ERR_ARG;
    if ((M * K > 0) && (!x || !codes || !scales)) return OR_ERR_ARG;
    if ((codesT == NULL) != (scalesT == NULL)) return OR_ERR_ARG;
    if (K % 32) return OR_ERR_SHAPE;
    if (codesT && M % 32) return OR_ERR_SHAPE;
    float xg[32];
    uint64_t eg[32];
    uint8_t cg[32], sb;
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j0 = 0; j0 < K; j0 += 32) {
            for (int t = 0; t < 32; ++t) {
                xg[t] = load_elem(x, xdt, i * K + j0 + t);
                eg[t] = (uint64_t)(i * K + j0 + t);
            }
            mxfp8_group(xg, eg, rounding, seed, &sb, cg);
            scales[i * (K / 32) + j0 / 32] = sb;
            memcpy(codes + i * K + j0, cg, 32);
        }
    if (codesT)
        for (int64_t j = 0; j < K; ++j)
            for (int64_t i0 = 0; i0 < M; i0 += 32) {
                for (int t = 0; t < 32; ++t) {
                    xg[t] = load_elem(x, xdt, (i0 + t) * K + j);
                    eg[t] = (uint64_t)((i0 + t) * K + j);
                }
                mxfp8_group(xg, eg, rounding, seed, &sb, cg);
                scalesT[j * (M / 32) + i0 / 32] = sb;
                memcpy(codesT + j * M + i0, cg, 32);
            }
    return OR_OK;
}

/* ========================================================================
 * FP32-scale modes of [LB] §1-§2: S = |W|max / 6 over the whole tensor, each
 * row (channel), or each group of 16 / 32 along K; v = x / S rounded to the
 * nearest E2M1 value.  scales: 1, M, or M*(K/g) binary32 values.
 * ====================================================================== */
int or_quantize_fp32scale(const void *x, int xdt, int64_t M, int64_t K, int gran,
                          uint8_t *codes, float *scales)
{
    if (M < 0 || K < 0) return OR_ERR_SHAPE;
    if (gran < OR_GRAN_TENSOR || gran > OR_GRAN_GROUP32) return OR_ERR_ARG;
    int64_t g = gran == OR_GRAN_TENSOR ? M * K : gran == OR_GRAN_ROW ? K
              : gran == OR_GRAN_GROUP16 ? 16 : 32;
    if (gran >= OR_GRAN_GROUP16 && K % g) return OR_ERR_SHAPE;
    if (K % 2) return OR_ERR_SHAPE;
    if (M * K == 0) return OR_OK;
    /* elements are visited in row-major order; group q covers [q*g, q*g+g) */
    for (int64_t q = 0; q * g < M * K; ++q) {
        float amax = 0.0f;
        for (int64_t e = q * g; e < (q + 1) * g; ++e) amax = fmaxf(amax, fabsf(load_elem(x, xdt, e)));
        float S = amax / 6.0f;
        scales[q] = S;
        for (int64_t e = q * g; e < (q + 1) * g; ++e)
            put_nibble(codes, e, S == 0.0f ? 0 : or_e2m1_rne(load_elem(x, xdt, e) / S));
    }
    return OR_OK;
}

/* ========================================================================
 * Dequantize: the exact value code * scale (* s_t) in binary64.
 * ====================================================================== */
static uint8_t get_nibble(const uint8_t *buf, int64_t idx)
{
    return (uint8_t)((buf[idx >> 1] >> ((idx & 1) * 4)) & 0x0F);
}

static double deq_elem(const uint8_t *codes, const uint8_t *scales, double s_t,
                       int64_t K, int fmt, int64_t i, int64_t j)
{
    if (fmt == OR_MXFP8)                             /* one E4M3 byte per element */
        return (double)or_e4m3_value(codes[i * K + j]) * or_e8m0_value(scales[i * (K / 32) + j / 32]);
    int g = fmt == OR_MXFP4 ? 32 : 16;
    double val = or_e2m1_value(get_nibble(codes, i * K + j));
    uint8_t sb = scales[i * (K / g) + j / g];
    if (fmt == OR_MXFP4) return val * or_e8m0_value(sb);
    return val * (double)or_e4m3_value(sb) * s_t;
}

int or_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tscale,
                  int64_t M, int64_t K, int fmt, double *out)
{
    if (M < 0 || K < 0) return OR_ERR_SHAPE;
    if (fmt != OR_MXFP4 && fmt != OR_NVFP4) return OR_ERR_ARG;
    int g = fmt == OR_MXFP4 ? 32 : 16;
    if (K % g) return OR_ERR_SHAPE;
    if (fmt == OR_NVFP4 && !tscale) return OR_ERR_ARG;
    double s_t = fmt == OR_NVFP4 ? (double)*tscale : 1.0;
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < K; ++j) out[i * K + j] = deq_elem(codes, scales, s_t, K, fmt, i, j);
    return OR_OK;
}

int or_dequantize_mxfp8(const uint8_t *codes, const uint8_t *scales,
                        int64_t M, int64_t K, double *out)
{
    if (M < 0 || K < 0 || K % 32) return OR_ERR_SHAPE;
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < K; ++j)
            out[i * K + j] = (double)or_e4m3_value(codes[i * K + j]) *
                             or_e8m0_value(scales[i * (K / 32) + j / 32]);
    return OR_OK;
}

float or_f64_to_f32(double v)
{
    return (float)v;                 /* IEEE conversion, round to nearest even */
}

/* round a binary64 value to the nearest bfloat16 (8 significant bits,
 * binary32 exponent range, subnormal quantum 2^-133), ties to even */
uint16_t or_f64_to_bf16(double v)
{
    assert(isfinite(v));
    double a = fabs(v), r;
    if (a == 0.0) {
        r = 0.0;
    } else {
        int e;
        frexp(a, &e);                                /* a = m * 2^e, m in [0.5,1) */
        int q = (e - 1 >= -126) ? (e - 8) : -133;    /* quantum of the result    */
        r = ldexp(nearbyint(ldexp(a, -q)), q);
    }
    float f = (float)(signbit(v) ? -r : r);          /* exact: r fits bfloat16 */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ========================================================================
 * GEMM reference ([QN] §QuTLASS: MXFP4/NVFP4 inputs, FP32 accumulate; the
 * FP8 backward of [QN]'s forward/backward split and [TI]'s MXFP8 operands):
 * Y[m][n] = sum_k deqA[m][k] * deqB[n][k], A M x K and B N x K (both
 * K-major), in binary64 over the dequantized operands.  For NVFP4 the sum
 * runs over code * dec(enc) and the tensor scales multiply the result;
 * MXFP8 operands are E4M3 bytes under E8M0 scales per 32.
 * ====================================================================== */
int or_gemm_sampled(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale,
                    const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale,
                    int64_t M, int64_t N, int64_t K, int fmt,
                    const int64_t *rows, const int64_t *cols, int64_t n_out,
                    double *out, double *absmag)
{
    if (M < 0 || N < 0 || K < 0) return OR_ERR_SHAPE;
    if (fmt != OR_MXFP4 && fmt != OR_NVFP4 && fmt != OR_MXFP8) return OR_ERR_ARG;
    int g = fmt == OR_NVFP4 ? 16 : 32;
    if (K % g) return OR_ERR_SHAPE;
    if (fmt == OR_NVFP4 && (!A_tscale || !B_tscale)) return OR_ERR_ARG;
    double tA = fmt == OR_NVFP4 ? (double)*A_tscale : 1.0;
    double tB = fmt == OR_NVFP4 ? (double)*B_tscale : 1.0;
    for (int64_t t = 0; t < n_out; ++t) {
        int64_t m = rows[t], n = cols[t];
        if (m < 0 || m >= M || n < 0 || n >= N) return OR_ERR_ARG;
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = deq_elem(A_codes, A_scales, 1.0, K, fmt, m, k);
            double b = deq_elem(B_codes, B_scales, 1.0, K, fmt, n, k);
            acc += a * b;
            mag += fabs(a) * fabs(b);
        }
        out[t] = acc * tA * tB;
        if (absmag) absmag[t] = mag * fabs(tA) * fabs(tB);
    }
    return OR_OK;
}

/* ========================================================================
 * KL-divergence clip calibration ([LB] §5, the TensorRT method the page
 * describes): for each candidate clip point T, P = the histogram of |x|
 * cut at T with everything beyond T counted in the last kept bin, and Q =
 * the kept histogram quantized to the quantizer's levels and spread back
 * over P's bins; the T with the least D_KL(P || Q) loses the least
 * information.  Readings (the page gives the idea, not the arithmetic):
 *   - histogram: `bins` bins over [0, amax] of the tensor; bin of |x| =
 *     min(bins - 1, trunc(fl(|x| * fl(bins / amax)))) in binary32;
 *   - candidates: i = first .. bins kept bins, T_i = fl(i * fl(amax / bins));
 *     first = levels (uniform) or 8 (E2M1);
 *   - levels: grid 0 = `levels` uniform levels, kept bin b in level
 *     floor(b / floor(i / levels)), the last level taking the remainder;
 *     grid 1 = the 8 E2M1 magnitudes {0,.5,1,1.5,2,3,4,6} scaled so that T
 *     maps to 6: bin b goes to the nearest magnitude of its centre,
 *     6 (b + 1/2) / i, ties to the even mantissa (decided exactly);
 *   - Q: each level's kept mass divided evenly among its bins where P != 0;
 *   - KL = sum over P > 0 of p log(p / q) with p, q normalised, binary64,
 *     bins in ascending order; a bin with P > 0 and Q = 0 makes the
 *     candidate's KL +infinity (rejected);
 *   - the least KL wins, the smallest i on a tie.
 * ====================================================================== */
int or_abs_histogram(const void *x, int xdt, int64_t n, int bins, float amax, uint64_t *hist)
{
    if (n < 0 || bins < 1 || !(amax >= 0.0f)) return OR_ERR_ARG;
    memset(hist, 0, sizeof(uint64_t) * (size_t)bins);
    if (amax == 0.0f) {                            /* all zeros: everything in bin 0 */
        hist[0] = (uint64_t)n;
        return OR_OK;
    }
    float inv = (float)bins / amax;
    for (int64_t e = 0; e < n; ++e) {
        float t = fabsf(load_elem(x, xdt, e)) * inv;
        int64_t b = (int64_t)t;                    /* truncation toward zero */
        if (b > bins - 1) b = bins - 1;
        hist[b] += 1;
    }
    return OR_OK;
}

/* E2M1 magnitude index (0..7) nearest to 6 (2b + 1) / (2i), ties to the even
 * mantissa: compared as integers against the midpoints m = 0.25, 0.75, 1.25,
 * 1.75, 2.5, 3.5, 5 (scaled by 8: 2, 6, 10, 14, 20, 28, 40): v < m iff
 * 24 (2b + 1) < 8 m i. */
int or_e2m1_level_of_bin(int64_t b, int64_t i)
{
    static const int64_t mid8[7] = {2, 6, 10, 14, 20, 28, 40};
    int64_t num = 24 * (2 * b + 1);                /* 8 * 6 (2b + 1) / 2, over i */
    int level = 0;
    for (int t = 0; t < 7; ++t) {
        int64_t rhs = mid8[t] * i;
        if (num > rhs) level = t + 1;
        else if (num == rhs) { level = ((t + 1) & 1) ? t : t + 1; break; }   /* tie: even code */
        else break;
    }
    return level;
}

static double kl_for_candidate(const uint64_t *hist, int bins, int i, int levels, int grid, int *level_of, double *qmass,
                               int64_t *nz)
{
    int L = grid ? 8 : levels;
    int per = grid ? 0 : i / levels;
    for (int l = 0; l < L; ++l) { qmass[l] = 0.0; nz[l] = 0; }
    uint64_t outliers = 0;
    for (int b = i; b < bins; ++b) outliers += hist[b];
    double total_p = 0.0;
    for (int b = 0; b < i; ++b) {
        int l = grid ? or_e2m1_level_of_bin(b, i) : (b / per < levels ? b / per : levels - 1);
        level_of[b] = l;
        qmass[l] += (double)hist[b];
        double pb = (double)hist[b] + (b == i - 1 ? (double)outliers : 0.0);
        if (pb != 0.0) nz[l] += 1;
        total_p += pb;
    }
    double total_q = 0.0;
    for (int l = 0; l < L; ++l) total_q += qmass[l];
    if (total_p == 0.0) return 0.0;
    if (total_q == 0.0) return INFINITY;
    double kl = 0.0;
    for (int b = 0; b < i; ++b) {
        double pb = (double)hist[b] + (b == i - 1 ? (double)outliers : 0.0);
        if (pb == 0.0) continue;
        int l = level_of[b];
        double qb = nz[l] ? qmass[l] / (double)nz[l] : 0.0;
        if (qb == 0.0) return INFINITY;
        double p = pb / total_p, q = qb / total_q;
        kl += p * log(p / q);
    }
    return kl;
}

int or_kl_calibrate(const uint64_t *hist, int bins, int levels, int grid, double *kl, int *best_i)
{
    if (bins < 8 || (grid != 0 && grid != 1)) return OR_ERR_ARG;
    if (!grid && (levels < 2 || levels > bins)) return OR_ERR_ARG;
    int first = grid ? 8 : levels;
    int *level_of = (int *)malloc(sizeof(int) * (size_t)bins);
    double qmass[4096 + 8];
    int64_t nz[4096 + 8];
    if (!level_of || (!grid && levels > 4096)) { free(level_of); return OR_ERR_ARG; }
    int best = bins;
    double best_kl = INFINITY;
    for (int i = first; i <= bins; ++i) {
        double d = kl_for_candidate(hist, bins, i, levels, grid, level_of, qmass, nz);
        if (kl) kl[i - first] = d;
        if (d < best_kl) { best_kl = d; best = i; }
    }
    free(level_of);
    *best_i = best;
    return OR_OK;
}

/* the clip point of candidate i: T = fl(i * fl(amax / bins)) */
float or_kl_threshold(float amax, int bins, int i)
{
    float w = amax / (float)bins;
    return (float)i * w;
}

