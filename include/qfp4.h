/*
 * qfp4.h -- C ABI of libqfp4: FP4 microscaling quantization of training
 * tensors and the block-scaled FP4 matmul that consumes them, on NVIDIA
 * B200 (sm_100a).
 *
 * Sources (the method; citations name the page and its section):
 *   [QN] "Quartet -- Native 4-bit training that actually trains" (GPU-MODE
 *        lecture 069 notes): Hadamard rotation y = xW = (xH)(H^T W); QuTLASS
 *        fused rotation, online quantization, stochastic-rounding kernel,
 *        MXFP4/NVFP4 GEMM with FP32 accumulate, FP4 forward / FP8 backward.
 *   [LB] "low-bit quantization" blog (caveduck, series #4): §FP4 (E2M1 grid
 *        +-{0,.5,1,1.5,2,3,4,6}, S = |W|max/6), §2 (group scales, MXFP4 = FP4
 *        elements + one shared scale per 32), §3 (E8M0 2^k scale, effective
 *        bits 4.25), §7 (Hadamard rotation, +-1/sqrt(n), O(n log n)).
 *   [TI] "Stable FP4 Training via Transposition-Invariant Block
 *        Quantization" (abstract): 2D blocks shared by X and X^T,
 *        truncation-free scaling, stochastic rounding, MXFP8 for Q/K.
 *   [46] "Four Over Six: More Accurate NVFP4 Quantization with Adaptive
 *        Block Scaling" (summary, Methodology 1-3): per block, the better of
 *        two candidate scales.
 *
 * General conventions
 *   - Every pointer argument is DEVICE memory owned by the caller, unless a
 *     parameter says otherwise.  The library allocates no device memory.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream).  The
 *     returned status covers argument validation and kernel launch; it is
 *     decided before anything is launched, so an error return leaves every
 *     output untouched.
 *   - Matrices are row-major.  X is M x K; element (i, j) has the logical
 *     index e = i*K + j.
 *   - FP4 (E2M1) codes: two per byte, element 2t in bits 0-3 and element
 *     2t+1 in bits 4-7; bit 3 of a code is the sign.  A row of K elements
 *     takes K/2 bytes.
 *   - Scale bytes: one per group, row-major M x (K/g).  MXFP4 (g = 32): an
 *     E8M0 byte, the scale is 2^(byte-127).  NVFP4 (g = 16): an OCP E4M3
 *     byte, the scale is e4m3(byte) * s_t with s_t the per-tensor scale.
 *   - All buffers need 16-byte aligned base pointers.
 *   - Size limits (QFP4_ERR_SHAPE beyond them): the quantize, dequantize
 *     and calibration calls take at most 2^38 elements (M*K, or n), a
 *     512 GB bf16 tensor; the GEMM and linear calls take M, N, K below
 *     2^30.  Within them every byte count fits int64.
 */
#ifndef QFP4_H
#define QFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qfp4_stream_t;   /* == cudaStream_t */

typedef enum {
    QFP4_MXFP4 = 0,             /* E2M1 elements, E8M0 scale per 32                          */
    QFP4_NVFP4 = 1,             /* E2M1 elements, E4M3 scale per 16, fp32 tensor scale       */
    QFP4_MXFP8 = 2              /* E4M3 elements (one byte each), E8M0 scale per 32, as
                                   qfp4_quantize_mxfp8 writes them: GEMM operands only       */
} qfp4_fmt;
typedef enum { QFP4_RNE = 0, QFP4_SR = 1 } qfp4_round;
typedef enum { QFP4_BF16 = 0, QFP4_F32 = 1 } qfp4_dtype;
typedef enum {
    QFP4_GRAN_TENSOR = 0, QFP4_GRAN_ROW = 1, QFP4_GRAN_GROUP16 = 2, QFP4_GRAN_GROUP32 = 3
} qfp4_gran;
/* Scale rules of qfp4_quantize_ex (see there). */
typedef enum {
    QFP4_SCALE_DEFAULT = 0,     /* MXFP4: truncation-free E8M0; NVFP4: E4M3 block scale to nearest */
    QFP4_SCALE_OCP_FLOOR = 1,   /* MXFP4 only: E8M0 k = floor(log2 amax) - 2 (the OCP rule; may clip) */
    QFP4_SCALE_E4M3_UP = 2      /* NVFP4 only: E4M3 block scale rounded up (no element clips) */
} qfp4_scale_rule;

enum {
    QFP4_OK = 0,
    QFP4_ERR_ARG = -1,          /* NULL where a buffer is required, bad enum, short workspace */
    QFP4_ERR_SHAPE = -2,        /* dimensions violate the call's divisibility or size rules   */
    QFP4_ERR_UNSUPPORTED = -3,  /* option combination not defined by the method              */
    QFP4_ERR_ALIGN = -4,        /* a pointer is not 16-byte aligned                           */
    QFP4_ERR_CUDA = -5,         /* a CUDA launch or driver call failed                        */
    QFP4_ERR_TIMEOUT = -6       /* a bounded device-side wait gave up (see qfp4_last_device_error) */
};

/* ------------------------------------------------------------------------
 * qfp4_quantize -- quantize X to FP4 with per-group scales.
 *
 * Per row block ([QN] Hadamard rotation and QuTLASS online quantization;
 * [LB] §FP4, §2, §3, §7; [TI]; [46]):
 *   (1) rotate != 0: each contiguous 128-element block along K is replaced
 *       by its normalised Walsh-Hadamard transform (Sylvester order, stages
 *       h = 1..64 of (a+b, a-b) in binary32, then one multiply by the
 *       binary32 value of 1/sqrt(128)).  Needs K % 128 == 0.
 *   (2) scales.  MXFP4: groups of 32 along K; the E8M0 exponent k is the
 *       least integer with 6 * 2^k >= amax (truncation-free; k clamped to
 *       [-127, 127]; an all-zero group gets byte 0 and +0 codes).  NVFP4:
 *       s_t = amax_t / (6*448) in binary32 over the whole (rotated) tensor;
 *       per 16-block enc = E4M3_RNE_satfinite((amax_b / 6) / s_t) and the
 *       effective scale S = e4m3(enc) * s_t (binary32).
 *   (3) four6 != 0 (RNE, 1D only; MXFP4: see qfp4_quantize_ex): a second candidate scale from
 *       amax_b / 4; each block keeps the candidate whose binary32 squared
 *       error sum(deq - x)^2 (summed as pairs i,i+8; +4; +2; +1) is lower,
 *       ties keeping amax/6.
 *   (4) v = x / S in binary32, then round to E2M1: rounding = QFP4_RNE,
 *       nearest grid value with ties to the even mantissa and saturation to
 *       +-6; rounding = QFP4_SR, stochastic: with lo <= |v| < hi adjacent
 *       grid values, up iff u < (|v|-lo)/(hi-lo), u = (w >> 8) * 2^-24 where
 *       w is word (e mod 4) of Philox4x32-10 keyed (seed low 32, seed high
 *       32) at counter (e/4 low 32, e/4 high 32, 0, 0).  The code's sign
 *       bit is the sign of v.
 *   (5) block2d != 0 (no rotation, no four6): T x T tiles share one scale
 *       (amax over the tile), so X and X^T use the same scales; T = 16 for
 *       NVFP4, 32 for MXFP4.  scales[i][j/T] and scalesT[j][i/T] both hold
 *       tile (i/T, j/T); codesT (K x M/2) is exactly the transpose of codes.
 *       Needs M % T == 0 and K % T == 0.
 *   In 1D mode a non-NULL codesT/scalesT asks for an independent
 *   quantization of every column (groups of g along M; K x M/2 codes,
 *   K x M/g scales), the baseline [TI] contrasts with 2D blocks; needs
 *   M % g == 0 and rotate == 0.
 *
 * Arguments
 *   x            M x K input, bf16 (xdt = QFP4_BF16) or binary32 (QFP4_F32).
 *   codes        out, M*K/2 bytes.       scales   out, M*(K/g) bytes.
 *   codesT       out or NULL, K*M/2.     scalesT  out or NULL, K*(M/g).
 *   tscale       NVFP4: out, one float, the decode tensor scale s_t.
 *                MXFP4: ignored (may be NULL).
 *   workspace    NVFP4: device scratch of at least
 *                qfp4_quantize_workspace_bytes() bytes (holds the partial
 *                tensor maxima; contents on entry do not matter).  MXFP4:
 *                may be NULL.
 * Errors: QFP4_ERR_SHAPE for K % g != 0, K % 128 != 0 with rotate, M or K
 *   not a multiple of the tile with block2d, M % g != 0 with a 1D codesT;
 *   QFP4_ERR_UNSUPPORTED for four6 with SR or block2d (or MXFP4 with a 1D
 *   codesT), block2d with rotate, rotate with a 1D codesT.
 * ---------------------------------------------------------------------- */
size_t qfp4_quantize_workspace_bytes(int64_t M, int64_t K, qfp4_fmt fmt, int rotate, int block2d);

int qfp4_quantize(const void *x, qfp4_dtype xdt, int64_t M, int64_t K,
                  qfp4_fmt fmt, qfp4_round rounding, int rotate, int block2d, int four6,
                  uint64_t seed,
                  uint8_t *codes, uint8_t *scales,
                  uint8_t *codesT, uint8_t *scalesT,
                  float *tscale,
                  void *workspace, size_t workspace_bytes,
                  qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_quantize_ex -- qfp4_quantize with the scale-rule variants, the 2D and
 * four-over-six options on MXFP4, and a caller-supplied tensor amax.
 * qfp4_quantize(...) is qfp4_quantize_ex(..., QFP4_SCALE_DEFAULT, seed,
 * NULL, NULL, ...).
 *   rule   QFP4_SCALE_DEFAULT, or the ablations the pages imply ([LB] §3:
 *          what a power-of-two scale costs; [TI]: truncation-free scaling):
 *          QFP4_SCALE_OCP_FLOOR (MXFP4): k = floor(log2 amax) - 2, the
 *            largest k with 2^(k+2) <= amax, so amax / 2^k is in [4, 8) and
 *            magnitudes above 6 * 2^k saturate to 6;
 *          QFP4_SCALE_E4M3_UP (NVFP4): enc = the least E4M3 value >=
 *            (amax_b / d) / s_t (saturating at 448), so S >= amax_b / d.
 *   four6  NVFP4 as in qfp4_quantize; MXFP4 (RNE, 1D rows only): the
 *          second candidate exponent is the least k4 with 4 * 2^k4 >= amax,
 *          kept only when the group's binary32 squared error (summed as
 *          pairs i, i+16; +8; +4; +2; +1) is strictly lower ([46]).  Under
 *          the default rule it never is (the 2^(k+1) grid is a subset below
 *          amax); under the OCP floor rule it trades clipping for range.
 *   block2d  NVFP4 16 x 16 tiles, or MXFP4 32 x 32 tiles (one E8M0 scale per
 *          tile, the scale rule applied to the tile amax); needs M and K
 *          multiples of the tile size.
 *   amax_in  NVFP4: NULL (the call measures the tensor's amax: an extra read
 *          of X), or a DEVICE pointer to a finite amax_t >= 0 from elsewhere
 *          -- a previous step's, a moving average of several ([QN] open
 *          questions: EMA / delayed activation scales), or a calibrated clip
 *          (qfp4_kl_calibrate).  s_t = fl(*amax_in / 2688); the quantize
 *          then reads X once, and blocks whose values exceed the implied
 *          range saturate (E4M3 byte 0x7E, codes +-6).  MXFP4: must be NULL.
 *   amax_out NVFP4: NULL, or a DEVICE float that receives this tensor's own
 *          amax (after rotation), e.g. for the next step's amax_in.
 *          MXFP4: must be NULL.
 *   workspace NVFP4: needed (qfp4_quantize_workspace_bytes) unless amax_in
 *          is given and amax_out is NULL.
 * Errors: as qfp4_quantize, plus QFP4_ERR_ARG for an unknown rule,
 *   QFP4_ERR_UNSUPPORTED for a rule of the other format, amax_in / amax_out
 *   with MXFP4, MXFP4 four6 with a 1D codesT.
 * ---------------------------------------------------------------------- */
int qfp4_quantize_ex(const void *x, qfp4_dtype xdt, int64_t M, int64_t K,
                     qfp4_fmt fmt, qfp4_round rounding, int rotate, int block2d, int four6,
                     qfp4_scale_rule rule, uint64_t seed,
                     const float *amax_in, float *amax_out,
                     uint8_t *codes, uint8_t *scales,
                     uint8_t *codesT, uint8_t *scalesT,
                     float *tscale,
                     void *workspace, size_t workspace_bytes,
                     qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_quantize_mxfp8 -- MXFP8 variant ([TI]: MXFP8 for the sensitive Q/K
 * projections; [QN]: FP8 backward): E4M3 elements in groups of 32 along K
 * under an E8M0 scale with k the least integer such that 448 * 2^k >= amax.
 * Elements: E4M3 round-to-nearest-even saturating to +-448, or the
 * stochastic rule of qfp4_quantize on the E4M3 grid (same Philox words).
 * codes M*K bytes, scales M*(K/32); codesT/scalesT (K*M and K*(M/32), or
 * NULL) hold the column-wise quantization (groups of 32 along M).
 * Needs K % 32 == 0 (and M % 32 == 0 with codesT).
 * ---------------------------------------------------------------------- */
int qfp4_quantize_mxfp8(const void *x, qfp4_dtype xdt, int64_t M, int64_t K,
                        qfp4_round rounding, uint64_t seed,
                        uint8_t *codes, uint8_t *scales,
                        uint8_t *codesT, uint8_t *scalesT,
                        qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_quantize_fp32scale -- the per-tensor / per-row / per-group FP32
 * scale modes of [LB] §1-§2: S = amax / 6 in binary32 over the tensor, each
 * row, or each group of 16 or 32 along K; v = x / S rounded to the nearest
 * E2M1 value (ties to even, saturating); S == 0 gives +0 codes.
 * scales: 1, M, M*K/16 or M*K/32 binary32 values.  Needs K % 16 == 0
 * (K % 32 == 0 for QFP4_GRAN_GROUP32).  workspace: qfp4_quantize_workspace_bytes
 * (M, K, QFP4_NVFP4, 0, 0) bytes for QFP4_GRAN_TENSOR, else may be NULL.
 * ---------------------------------------------------------------------- */
int qfp4_quantize_fp32scale(const void *x, qfp4_dtype xdt, int64_t M, int64_t K,
                            qfp4_gran gran, uint8_t *codes, float *scales,
                            void *workspace, size_t workspace_bytes,
                            qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_dequantize -- out[i][j] = value(code) * scale (* s_t for NVFP4),
 * formed exactly and rounded once to out_dt (nearest even).  tscale:
 * NVFP4 device pointer to s_t, MXFP4 ignored.  Needs K % g == 0.  A scale
 * byte that encodes NaN (E8M0 0xFF; E4M3 0x7F, 0xFF -- the quantize calls
 * never write one) gives NaN outputs for its group.
 * ---------------------------------------------------------------------- */
int qfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tscale,
                    int64_t M, int64_t K, qfp4_fmt fmt, qfp4_dtype out_dt, void *out,
                    qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_gemm_blockscaled -- Y = deq(A) * deq(B)^T ([QN] §QuTLASS: MXFP4 /
 * NVFP4 operands, FP32 accumulation; [LB] §FP4: Blackwell FP4 tensor
 * cores; [QN] forward/backward split and [TI]: MXFP8 operands for the FP8
 * backward and the Q/K projections).  A is M x K and B is N x K, both
 * K-major (codes + scales exactly as qfp4_quantize writes them, or for
 * fmt = QFP4_MXFP8 as qfp4_quantize_mxfp8 writes them); for NVFP4 the
 * tensor scales multiply the accumulated sum: Y = acc * (s_tA * s_tB)
 * (A_tscale, B_tscale device pointers; ignored for MXFP4 and MXFP8).  out:
 * M x N row-major, binary32 or bf16 (round to nearest even).  Runs on
 * 5th-generation tensor cores (tcgen05 block-scaled MMA: kind::mxf4,
 * kind::mxf4nvf4 or kind::mxf8f6f4; fp32 accumulators in tensor memory).
 * workspace: device scratch of at least qfp4_gemm_workspace_bytes(M, N, K,
 *   fmt) bytes; it receives the scales rearranged for the tensor cores
 *   (contents on entry do not matter, the call overwrites them).
 * Needs K % 32 == 0 (a K tail short of the 256-element tile is zero-filled),
 * N % 4 == 0 (binary32 out) or N % 8 == 0 (bf16 out), M, N, K < 2^30.
 * ---------------------------------------------------------------------- */
size_t qfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);

int qfp4_gemm_blockscaled(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale,
                          const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale,
                          int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
                          qfp4_dtype out_dt, void *out,
                          void *workspace, size_t workspace_bytes,
                          qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_gemm_blockscaled_noalloc -- qfp4_gemm_blockscaled for callers that
 * cannot allocate device memory (an op or plugin hook that forbids
 * allocation while enqueuing, an allocation-free real-time loop, a library
 * handed only its inputs and outputs).  No counterpart on the source pages:
 * it is a packaging of the same GEMM.  Same arguments, semantics and
 * results as qfp4_gemm_blockscaled, minus the workspace: the rearranged
 * scales go to a 16 MiB scratch array built into the library, which every
 * GPU that loads the library's kernels holds until the process exits.
 * The first call on a device looks up the array's device address (with
 * that device current); make it before any stream capture.  All calls share
 * the array (nothing in it needs to start at zero); calls whose work
 * overlaps on the GPU race on it.  Returns QFP4_ERR_SHAPE when the shape's
 * rearranged scales, qfp4_gemm_workspace_bytes(M, N, K, fmt), exceed
 * 16 MiB.  Allocates nothing (no cudaMalloc / cudaFree, no allocating
 * library call).
 * ---------------------------------------------------------------------- */
int qfp4_gemm_blockscaled_noalloc(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale,
                                  const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale,
                                  int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
                                  qfp4_dtype out_dt, void *out, qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_gemm_fused_rq -- the same GEMM with A given in bf16: A is rotated
 * (rotate != 0, along K in 128 blocks) and quantized (fmt, RNE, four6 as in
 * qfp4_quantize) inside the call, then multiplied by the pre-quantized B
 * ([QN] §QuTLASS: fused rotation and online quantization before the GEMM;
 * B is expected to be rotated the same way offline, so that
 * (xH)(WH)^T = xW^T).  A is quantized once (not once per output tile) into
 * the workspace by the 1D quantize kernel, then consumed by the tensor-core
 * kernel; the launches follow each other as dependent launches.  NVFP4
 * first measures A's tensor amax (an extra read of A; see
 * qfp4_gemm_fused_rq_ex to supply it).
 * workspace: at least qfp4_gemm_fused_rq_workspace_bytes(M, N, K, fmt)
 * bytes of device scratch.  Same shape rules as qfp4_gemm_blockscaled,
 * plus K % 128 == 0 with rotate.
 * ---------------------------------------------------------------------- */
size_t qfp4_gemm_fused_rq_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);

int qfp4_gemm_fused_rq(const void *A_bf16, int64_t M, int64_t K, int rotate, int four6, qfp4_fmt fmt,
                       const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale, int64_t N,
                       void *workspace, size_t workspace_bytes,
                       qfp4_dtype out_dt, void *out, qfp4_stream_t stream);

/* qfp4_gemm_fused_rq with NVFP4's tensor amax of A supplied and / or
 * reported, as in qfp4_quantize_ex: A_amax_in (device float, or NULL) gives
 * s_t = fl(*A_amax_in / 2688) and removes the extra read of A; A_amax_out
 * (device float, or NULL) receives A's own amax after rotation.  MXFP4: both
 * must be NULL (QFP4_ERR_UNSUPPORTED). */
int qfp4_gemm_fused_rq_ex(const void *A_bf16, int64_t M, int64_t K, int rotate, int four6, qfp4_fmt fmt,
                          const float *A_amax_in, float *A_amax_out,
                          const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale, int64_t N,
                          void *workspace, size_t workspace_bytes,
                          qfp4_dtype out_dt, void *out, qfp4_stream_t stream);

/* Where qfp4_gemm_fused_rq leaves A's quantized operand in its workspace
 * once the call's work is done: codes (M*K/2 bytes, as qfp4_quantize writes
 * them) at byte *codes_off, row-major scales (M*(K/g) bytes) at
 * *scales_off, and for NVFP4 the tensor scale (one float) at *tscale_off;
 * each offset is a multiple of 256.  The three out-pointers are host
 * memory.  Returns QFP4_ERR_ARG for a bad fmt or a NULL out-pointer,
 * QFP4_ERR_SHAPE for a negative dimension. */
int qfp4_gemm_fused_rq_workspace_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, size_t *codes_off,
                                        size_t *scales_off, size_t *tscale_off);

/* ------------------------------------------------------------------------
 * qfp4_linear_forward -- the forward of a Quartet-style linear layer,
 * Y = X W^T computed as Q(X H) Q(W H)^T ([QN] Hadamard rotation: y = xW^T =
 * (xH)(WH)^T with H orthogonal, so the rotation cancels; FP4 forward).
 *   X  M x K bf16 activations, W  N x K bf16 weights (out x in features),
 *      both row-major device memory, rotated along K in 128-blocks and
 *      quantized (fmt = QFP4_MXFP4 or QFP4_NVFP4, RNE, four6 for NVFP4) as
 *      qfp4_quantize does; Y  M x N, out_dt binary32 or bf16.
 *   workspace: qfp4_linear_forward_workspace_bytes(M, N, K, fmt) bytes of
 *      device scratch (the quantized operands and the GEMM's scale chunks).
 * Needs K % 128 == 0, N % 4 (binary32 out) or N % 8 (bf16 out).  Errors as
 * qfp4_quantize and qfp4_gemm_blockscaled.
 * ---------------------------------------------------------------------- */
size_t qfp4_linear_forward_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);

int qfp4_linear_forward(const void *X, const void *W, int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, int four6,
                        qfp4_dtype out_dt, void *Y, void *workspace, size_t workspace_bytes, qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_linear_backward -- the backward of the same layer from the output
 * gradient G: dX = G W (M x K) and dW = G^T X (N x K), with the gradient
 * stochastically rounded (Philox keyed on seed and G's element index) and
 * each operand quantized once for both of its uses ([QN] forward/backward
 * split: FP4 or FP8 backward; [TI] transposition-invariant 2D blocks, MXFP8
 * operands):
 *   fmt = QFP4_NVFP4: G, W and X in 2D 16 x 16 NVFP4 blocks (G by SR, W and X
 *     by RNE), each pass emitting the operand and its transpose;
 *   fmt = QFP4_MXFP8: G as MXFP8 rows (groups along N) and columns (along M)
 *     by SR, W and X as MXFP8 columns by RNE.
 *   dX = GEMM(A = G, B = W^T) and dW = GEMM(A = G^T, B = X^T) on the
 *   block-scaled tensor cores.
 *   G  M x N, X  M x K, W  N x K bf16; dX  M x K and dW  N x K out_dt; either
 *   output may be NULL to skip it (X or W is then not read).
 *   workspace: qfp4_linear_backward_workspace_bytes(M, N, K, fmt) bytes.
 * Needs M % 32 == 0, N % 32 == 0, K % 16 (NVFP4) or K % 32 (MXFP8) == 0.
 * ---------------------------------------------------------------------- */
size_t qfp4_linear_backward_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);

int qfp4_linear_backward(const void *G, const void *X, const void *W, int64_t M, int64_t N, int64_t K,
                         qfp4_fmt fmt, uint64_t seed, qfp4_dtype out_dt, void *dX, void *dW,
                         void *workspace, size_t workspace_bytes, qfp4_stream_t stream);

/* ------------------------------------------------------------------------
 * qfp4_kl_calibrate -- KL-divergence clip point of an activation tensor
 * ([LB] §5, the TensorRT method): for each candidate clip T, P = the
 * histogram of |x| cut at T with the tail counted in the last kept bin, Q =
 * the kept histogram quantized to the levels and spread back over P's
 * nonzero bins; the T with the least D_KL(P || Q) is the clip point.
 *   x         n elements (bf16 or binary32), device memory.
 *   bins      histogram bins over [0, amax] (8 .. 8192); bin of |x| =
 *             min(bins-1, trunc(fl(|x| * fl(bins / amax)))).
 *   grid      0: `levels` uniform levels (2 .. bins; a bin b of the i kept
 *             ones is in level floor(b / floor(i / levels)), the last level
 *             taking the remainder), candidates i = levels .. bins;
 *             1: the E2M1 magnitudes scaled so T maps to 6 (a bin goes to the
 *             magnitude nearest its centre, ties to the even code; `levels`
 *             is ignored), candidates i = 8 .. bins.
 *   KL in binary64 (p, q normalised; a bin with P > 0 and Q = 0 rejects the
 *   candidate); the least KL wins, the smallest i on a tie; all rejected
 *   keeps every bin.  T = fl(i * fl(amax / bins)).
 *   clip_out       device float, receives T (for example as the amax_in of
 *                  qfp4_quantize_ex, or S = T / 6 for a per-tensor scale).
 *   best_bins_out  device int (or NULL): the winning i.
 *   kl_out         device double[bins - first + 1] (or NULL): every KL.
 *   hist_out       device uint64[bins] (or NULL): the histogram.
 *   workspace      qfp4_kl_calibrate_workspace_bytes(bins, levels, grid).
 * Errors: QFP4_ERR_ARG for bins, levels or grid out of range, a NULL x
 * (n > 0) or clip_out, a short workspace; QFP4_ERR_SHAPE for n < 0 or
 * n > 2^38; QFP4_ERR_ALIGN for a pointer off 16 bytes.
 * ---------------------------------------------------------------------- */
size_t qfp4_kl_calibrate_workspace_bytes(int bins, int levels, int grid);

int qfp4_kl_calibrate(const void *x, qfp4_dtype xdt, int64_t n, int bins, int levels, int grid,
                      float *clip_out, int *best_bins_out, double *kl_out, uint64_t *hist_out,
                      void *workspace, size_t workspace_bytes, qfp4_stream_t stream);

/* Human-readable text of a status code (static storage). */
const char *qfp4_status_string(int status);

/* Sticky device-side error word of the current device: 0 when clean, else
 * the code of the first device-side failure since the last read (cleared by
 * the read); -1 if the device could not be read.  Synchronizes the current
 * device.  Codes: */
enum {
    QFP4_DEV_ERR_TIMEOUT = 1    /* a bounded wait inside a kernel gave up (the kernel returned early) */
};
int qfp4_last_device_error(void);

/* Diagnostics: launch a one-thread kernel whose only action is a bounded
 * wait on a barrier that nothing completes, giving up after limit_us
 * microseconds (1 .. 10^6).  Nothing else is in flight, so it exercises the
 * give-up path every other kernel's waits share: afterwards
 * qfp4_last_device_error() returns QFP4_DEV_ERR_TIMEOUT and the context
 * stays usable.  No counterpart on the source pages (a library self-test). */
int qfp4_selftest_wait_timeout(int64_t limit_us, qfp4_stream_t stream);

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
int qfp4_version(void);

/* Diagnostics: number of kernels this process has launched through the
 * library so far (host-side counter, all devices). */
uint64_t qfp4_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* QFP4_H */
