/*
 * qfp4_oracle.h -- plain, slow, single-threaded CPU oracle for FP4 microscaling
 * quantization and the block-scaled FP4 matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load or call this library.  The product
 * path (libqfp4, the CUDA kernels and their Python binding) never does; it
 * shares no code, header, table or constant with this file.
 *
 * Every routine follows a definition on the source pages, cited beside it:
 *   [QN]  "Quartet -- Native 4-bit training that actually trains"
 *         (GPU-MODE lecture 069 notes): Hadamard rotation identity
 *         y = xW = (xH)(H^T W); stochastic-rounding kernel; FP4/FP8 split.
 *   [LB]  "low-bit quantization" blog (caveduck, series #4):
 *         §FP4 (E2M1 grid +-{0,.5,1,1.5,2,3,4,6}, range [-6,6], S = |W|max/6),
 *         §1 (outlier table), §2 (per-channel / per-group(32) scales),
 *         §3 (E8M0 2^k group scale, effective bits), §7 (Hadamard rotation,
 *         H = +-1/sqrt(n), O(n log n)).
 *   [TI]  "Stable FP4 Training via Transposition-Invariant Block
 *         Quantization" (abstract): 2D blocks, truncation-free scaling,
 *         stochastic rounding, MXFP8 for Q/K.
 *   [46]  "Four Over Six: More Accurate NVFP4 Quantization with Adaptive
 *         Block Scaling" (summary, Methodology 1-3): two candidate scales per
 *         block, keep the one with lower error.
 * Where the pages are silent the oracle takes one fixed reading; each is
 * listed beside the function that applies it.
 *
 * Parity pins: every function here is pinned by tests (tests/test_oracle_*.py)
 * against closed forms, the pages' worked examples, brute force on tiny
 * inputs, published known-answer vectors (Philox) and invariants.
 *
 * Conventions: row-major M x K input; element e = i*K + j.  FP4 codes are
 * packed two per byte, element 2t in bits 0-3 and 2t+1 in bits 4-7.  Scales
 * are one byte each, row-major M x (K/g).  All arithmetic on floats is IEEE
 * binary32 or binary64 round-to-nearest, compiled with -ffp-contract=off.
 */
#ifndef QFP4_ORACLE_H
#define QFP4_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_MXFP4 = 0, OR_NVFP4 = 1, OR_MXFP8 = 2 };   /* group formats (MXFP8: GEMM reference only) */
enum { OR_RULE_DEFAULT = 0, OR_RULE_OCP_FLOOR = 1, OR_RULE_E4M3_UP = 2 };   /* scale rules */
enum { OR_RNE = 0, OR_SR = 1 };                /* rounding                 */
enum { OR_BF16 = 0, OR_F32 = 1 };              /* input / output dtypes    */
enum { OR_GRAN_TENSOR = 0, OR_GRAN_ROW = 1, OR_GRAN_GROUP16 = 2, OR_GRAN_GROUP32 = 3 };

/* status codes (mirrors the meaning of the product's, defined separately) */
enum { OR_OK = 0, OR_ERR_ARG = -1, OR_ERR_SHAPE = -2, OR_ERR_UNSUPPORTED = -3 };

/* ---- element formats -------------------------------------------------- */
float   or_e2m1_value(uint8_t code);              /* 4-bit code -> value     */
uint8_t or_e2m1_rne(float v);                     /* nearest, ties to even   */
uint8_t or_e2m1_sr(float v, uint32_t r);          /* stochastic, word r      */
float   or_e4m3_value(uint8_t b);                 /* OCP E4M3 byte -> value  */
uint8_t or_e4m3_rne(float v);                     /* nearest, satfinite      */
uint8_t or_e4m3_sr(float v, uint32_t r);          /* stochastic, satfinite   */
double  or_e8m0_value(uint8_t b);                 /* 2^(b-127)               */
int     or_scale_exp(float amax, double top);     /* least k: top*2^k>=amax  */
int     or_scale_exp_floor(float amax, int emax); /* OCP: floor(log2 amax)-emax */
uint8_t or_e4m3_up(float v);                      /* least E4M3 >= |v|, sat.  */

/* ---- building blocks -------------------------------------------------- */
void     or_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
uint32_t or_sr_word(uint64_t seed, uint64_t e);   /* random word of element e */
void     or_fwht128(float *x);                    /* in place, normalised    */
float    or_bf16_to_f32(uint16_t h);

/* ---- quantize (qfp4_quantize semantics) -------------------------------- */
int or_quantize(const void *x, int xdt, int64_t M, int64_t K,
                int fmt, int rounding, int rotate, int block2d, int four6,
                uint64_t seed,
                uint8_t *codes, uint8_t *scales,
                uint8_t *codesT, uint8_t *scalesT,
                float *tscale);

/* The same with the scale-rule variants and a given tensor amax:
 *   rule      OR_RULE_DEFAULT (MXFP4 truncation-free E8M0, NVFP4 E4M3 nearest),
 *             OR_RULE_OCP_FLOOR (MXFP4: k = floor(log2 amax) - 2, may clip),
 *             OR_RULE_E4M3_UP (NVFP4: block scale byte rounded up, no clipping);
 *   four6     NVFP4 16-blocks, or MXFP4 32-groups (candidate 4 * 2^k4 >= amax);
 *   block2d   16x16 NVFP4 or 32x32 MXFP4 tiles;
 *   row0      logical index of x's first row (random words keyed on
 *             (row0 + i) * K + j), so row slices can be quantized apart (1D);
 *   amax_in   NVFP4: NULL = the tensor's own amax; else s_t = *amax_in / 2688;
 *   amax_out  NVFP4: NULL, or receives the tensor's own (rotated) amax. */
int or_quantize_ex(const void *x, int xdt, int64_t M, int64_t K,
                   int fmt, int rounding, int rotate, int block2d, int four6, int rule,
                   uint64_t seed, int64_t row0, const float *amax_in,
                   uint8_t *codes, uint8_t *scales,
                   uint8_t *codesT, uint8_t *scalesT,
                   float *tscale, float *amax_out);

/* max |x| over the tensor after the optional rotation (NVFP4's amax_t) */
float or_tensor_amax(const void *x, int xdt, int64_t M, int64_t K, int rotate);

/* four-over-six decision for one 16-block (returns 1 if the amax/4 candidate
 * is chosen); exposed for brute-force pins. */
int or_four6_pick(const float *x16, float s_t, uint8_t *enc_out, uint8_t codes_out[16]);

/* one MXFP4 group of 32 values x (logical indices e): scale byte and codes
 * under `rule`, with the four-over-six choice when four6 (returns 1 when the
 * 4 * 2^k4 candidate is kept); exposed for brute-force pins. */
int or_mxfp4_group(const float *x, const uint64_t *e, int rounding, int four6, int rule,
                   uint64_t seed, uint8_t *sbyte, uint8_t codes[32]);

/* ---- MXFP8 E4M3 quantize ------------------------------------------------ */
int or_quantize_mxfp8(const void *x, int xdt, int64_t M, int64_t K,
                      int rounding, uint64_t seed,
                      uint8_t *codes, uint8_t *scales,
                      uint8_t *codesT, uint8_t *scalesT);

/* ---- FP32-scale modes (per tensor / row / group), RNE ---------------------- */
int or_quantize_fp32scale(const void *x, int xdt, int64_t M, int64_t K, int gran,
                          uint8_t *codes, float *scales);

/* ---- dequantize: exact value in binary64 ------------------------------- */
int or_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tscale,
                  int64_t M, int64_t K, int fmt, double *out);
int or_dequantize_mxfp8(const uint8_t *codes, const uint8_t *scales,
                        int64_t M, int64_t K, double *out);
/* binary64 -> output dtype, one rounding (nearest even). */
uint16_t or_f64_to_bf16(double v);
float    or_f64_to_f32(double v);

/* ---- block-scaled GEMM reference: Y = deq(A) * deq(B)^T in binary64 ---- */
/* Y for the (m,n) pairs listed in rows[]/cols[] (count n_out); also returns
 * the per-element magnitude sum  sum_k |deqA||deqB|  in absmag (may be NULL). */
int or_gemm_sampled(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale,
                    const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale,
                    int64_t M, int64_t N, int64_t K, int fmt,
                    const int64_t *rows, const int64_t *cols, int64_t n_out,
                    double *out, double *absmag);

/* ---- KL-divergence clip calibration ([LB] §5) ------------------------- */
/* histogram of |x| over [0, amax] in `bins` bins (see the .c for the bin rule) */
int or_abs_histogram(const void *x, int xdt, int64_t n, int bins, float amax, uint64_t *hist);
/* E2M1 magnitude index nearest to bin b's centre when i kept bins map to [0, 6] */
int or_e2m1_level_of_bin(int64_t b, int64_t i);
/* KL for every candidate i = first .. bins (kl[i - first], may be NULL) and
 * the winning i; grid 0: `levels` uniform levels (first = levels), grid 1:
 * the E2M1 magnitudes (first = 8). */
int or_kl_calibrate(const uint64_t *hist, int bins, int levels, int grid, double *kl, int *best_i);
float or_kl_threshold(float amax, int bins, int i);

#ifdef __cplusplus
}
#endif
#endif
