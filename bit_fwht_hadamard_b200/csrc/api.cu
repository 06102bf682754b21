// api.cu -- the extern "C" entry points of libqfp4: argument validation
// (all of it before any launch) and dispatch to the kernels.
#include "qfp4_common.cuh"
#include "quantize1d.cuh"

namespace qfp4 {
int dequantize(const uint8_t *codes, const uint8_t *scales, const float *tscale, int64_t n, qfp4_fmt fmt,
               qfp4_dtype out_dt, void *out, cudaStream_t stream);
int quantize_fp32scale(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_gran gran, uint8_t *codes,
                       float *scales, float *partials, cudaStream_t stream);
int quantize_columns(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_fmt fmt, qfp4_round rounding,
                     int four6, uint64_t seed, uint8_t *codesT, uint8_t *scalesT, const float *partials,
                     int n_partials, cudaStream_t stream, const QuantOpts &opt);
int quantize2d(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_fmt fmt, qfp4_round rounding,
               uint64_t seed, uint8_t *codes, uint8_t *scales, uint8_t *codesT, uint8_t *scalesT, float *tscale,
               float *partials, cudaStream_t stream, const QuantOpts &opt);
int tscale_from_amax(const float *amax_in, float *tscale, cudaStream_t stream);
int quantize_mxfp8(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_round rounding, uint64_t seed,
                   uint8_t *codes, uint8_t *scales, uint8_t *codesT, uint8_t *scalesT, cudaStream_t stream);
int gemm_blockscaled(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale, const uint8_t *B_codes,
                     const uint8_t *B_scales, const float *B_tscale, int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
                     qfp4_dtype out_dt, void *out, void *workspace, cudaStream_t stream);
size_t gemm_workspace(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);
int gemm_fused_rq(const void *A_bf16, int64_t M, int64_t K, int rotate, int four6, qfp4_fmt fmt,
                  const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale, int64_t N, void *workspace,
                  qfp4_dtype out_dt, void *out, cudaStream_t stream, const float *amax_in, float *amax_out);
size_t gemm_fused_rq_workspace(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);
void gemm_fused_rq_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, size_t *codes, size_t *scales,
                          size_t *tscale);
}  // namespace qfp4

using namespace qfp4;

static bool ok_align(const void *p) { return p == nullptr || aligned16(p); }

// At most 2^38 elements in an M x K operand (a 512 GB bf16 tensor, above one
// GPU's memory): every byte count fits int64, and the 1D pass's tensor map
// (rows of 64 elements) stays within its 2^32-row limit.
constexpr int64_t kMaxElems = int64_t(1) << 38;
static bool size_ok(int64_t M, int64_t K) { return M <= kMaxElems && K <= kMaxElems && (M == 0 || K <= kMaxElems / M); }

extern "C" size_t qfp4_quantize_workspace_bytes(int64_t M, int64_t K, qfp4_fmt fmt, int rotate, int block2d)
{
    (void)M; (void)K; (void)rotate; (void)block2d;
    return fmt == QFP4_NVFP4 ? sizeof(float) * kMaxPartials : 0;
}

extern "C" int qfp4_quantize_ex(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_fmt fmt,
                                qfp4_round rounding, int rotate, int block2d, int four6, qfp4_scale_rule rule,
                                uint64_t seed, const float *amax_in, float *amax_out, uint8_t *codes,
                                uint8_t *scales, uint8_t *codesT, uint8_t *scalesT, float *tscale, void *workspace,
                                size_t workspace_bytes, qfp4_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (M < 0 || K < 0 || !size_ok(M, K)) return QFP4_ERR_SHAPE;
    if (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4) return QFP4_ERR_ARG;
    if (rounding != QFP4_RNE && rounding != QFP4_SR) return QFP4_ERR_ARG;
    if (xdt != QFP4_BF16 && xdt != QFP4_F32) return QFP4_ERR_ARG;
    if (rule != QFP4_SCALE_DEFAULT && rule != QFP4_SCALE_OCP_FLOOR && rule != QFP4_SCALE_E4M3_UP) return QFP4_ERR_ARG;
    const int64_t n = M * K;
    if (n > 0 && (!x || !codes || !scales)) return QFP4_ERR_ARG;
    if ((codesT == nullptr) != (scalesT == nullptr)) return QFP4_ERR_ARG;
    if (fmt == QFP4_NVFP4 && !tscale) return QFP4_ERR_ARG;
    const int g = fmt == QFP4_MXFP4 ? 32 : 16;
    if (rule == QFP4_SCALE_OCP_FLOOR && fmt != QFP4_MXFP4) return QFP4_ERR_UNSUPPORTED;
    if (rule == QFP4_SCALE_E4M3_UP && fmt != QFP4_NVFP4) return QFP4_ERR_UNSUPPORTED;
    if ((amax_in || amax_out) && fmt != QFP4_NVFP4) return QFP4_ERR_UNSUPPORTED;
    if (four6 && (block2d || rounding != QFP4_RNE)) return QFP4_ERR_UNSUPPORTED;
    if (four6 && fmt == QFP4_MXFP4 && codesT) return QFP4_ERR_UNSUPPORTED;
    if (block2d && rotate) return QFP4_ERR_UNSUPPORTED;
    if (!block2d && rotate && codesT) return QFP4_ERR_UNSUPPORTED;
    if (K % g) return QFP4_ERR_SHAPE;
    if (rotate && K % 128) return QFP4_ERR_SHAPE;
    if (block2d && (M % g || K % g)) return QFP4_ERR_SHAPE;
    if (!block2d && codesT && M % g) return QFP4_ERR_SHAPE;
    if (!ok_align(x) || !ok_align(codes) || !ok_align(scales) || !ok_align(codesT) || !ok_align(scalesT))
        return QFP4_ERR_ALIGN;
    const bool needs_ws = fmt == QFP4_NVFP4 && (!amax_in || amax_out);
    if (needs_ws && (!workspace || workspace_bytes < sizeof(float) * kMaxPartials)) return QFP4_ERR_ARG;
    if (needs_ws && !ok_align(workspace)) return QFP4_ERR_ALIGN;
    float *partials = static_cast<float *>(workspace);
    QuantOpts opt;
    opt.rule = rule;
    opt.amax_in = amax_in;
    opt.amax_out = amax_out;

    if (n == 0) {
        if (fmt == QFP4_NVFP4) {
            if (amax_in) {
                const int st = tscale_from_amax(amax_in, tscale, stream);   // s_t = fl(amax / 2688)
                if (st != QFP4_OK) return st;
            } else if (cudaMemsetAsync(tscale, 0, sizeof(float), stream) != cudaSuccess) {
                return QFP4_ERR_CUDA;
            }
            if (amax_out && cudaMemsetAsync(amax_out, 0, sizeof(float), stream) != cudaSuccess) return QFP4_ERR_CUDA;
        }
        return QFP4_OK;
    }
    if (block2d)
        return quantize2d(x, xdt, M, K, fmt, rounding, seed, codes, scales, codesT, scalesT, tscale, partials, stream,
                          opt);
    int n_parts = 0;
    int st = quantize1d(x, xdt, n, fmt, rounding, rotate, four6, seed, codes, scales, tscale, partials, &n_parts,
                        stream, opt);
    if (st != QFP4_OK || !codesT) return st;
    // The NVFP4 amax pass above left its partial maxima in the workspace:
    // the column-wise quantization reuses them for the same s_t.
    return quantize_columns(x, xdt, M, K, fmt, rounding, four6, seed, codesT, scalesT, partials, n_parts, stream, opt);
}

extern "C" int qfp4_quantize(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_fmt fmt, qfp4_round rounding,
                             int rotate, int block2d, int four6, uint64_t seed, uint8_t *codes, uint8_t *scales,
                             uint8_t *codesT, uint8_t *scalesT, float *tscale, void *workspace,
                             size_t workspace_bytes, qfp4_stream_t stream)
{
    return qfp4_quantize_ex(x, xdt, M, K, fmt, rounding, rotate, block2d, four6, QFP4_SCALE_DEFAULT, seed, nullptr,
                            nullptr, codes, scales, codesT, scalesT, tscale, workspace, workspace_bytes, stream);
}

extern "C" int qfp4_quantize_mxfp8(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_round rounding,
                                   uint64_t seed, uint8_t *codes, uint8_t *scales, uint8_t *codesT, uint8_t *scalesT,
                                   qfp4_stream_t stream)
{
    if (M < 0 || K < 0 || !size_ok(M, K)) return QFP4_ERR_SHAPE;
    if (rounding != QFP4_RNE && rounding != QFP4_SR) return QFP4_ERR_ARG;
    if (xdt != QFP4_BF16 && xdt != QFP4_F32) return QFP4_ERR_ARG;
    if (M * K > 0 && (!x || !codes || !scales)) return QFP4_ERR_ARG;
    if ((codesT == nullptr) != (scalesT == nullptr)) return QFP4_ERR_ARG;
    if (K % 32) return QFP4_ERR_SHAPE;
    if (codesT && M % 32) return QFP4_ERR_SHAPE;
    if (!ok_align(x) || !ok_align(codes) || !ok_align(scales) || !ok_align(codesT) || !ok_align(scalesT))
        return QFP4_ERR_ALIGN;
    if (M * K == 0) return QFP4_OK;
    return quantize_mxfp8(x, xdt, M, K, rounding, seed, codes, scales, codesT, scalesT,
                          reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int qfp4_quantize_fp32scale(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_gran gran,
                                       uint8_t *codes, float *scales, void *workspace, size_t workspace_bytes,
                                       qfp4_stream_t stream)
{
    if (M < 0 || K < 0 || !size_ok(M, K)) return QFP4_ERR_SHAPE;
    if (xdt != QFP4_BF16 && xdt != QFP4_F32) return QFP4_ERR_ARG;
    if (gran < QFP4_GRAN_TENSOR || gran > QFP4_GRAN_GROUP32) return QFP4_ERR_ARG;
    if (M * K > 0 && (!x || !codes || !scales)) return QFP4_ERR_ARG;
    if (K % 16) return QFP4_ERR_SHAPE;
    if (gran == QFP4_GRAN_GROUP32 && K % 32) return QFP4_ERR_SHAPE;
    if (!ok_align(x) || !ok_align(codes) || !ok_align(scales)) return QFP4_ERR_ALIGN;
    if (gran == QFP4_GRAN_TENSOR && (!workspace || workspace_bytes < sizeof(float) * kMaxPartials))
        return QFP4_ERR_ARG;
    return quantize_fp32scale(x, xdt, M, K, gran, codes, scales, static_cast<float *>(workspace),
                              reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int qfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tscale, int64_t M, int64_t K,
                               qfp4_fmt fmt, qfp4_dtype out_dt, void *out, qfp4_stream_t stream)
{
    if (M < 0 || K < 0 || !size_ok(M, K)) return QFP4_ERR_SHAPE;
    if (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4) return QFP4_ERR_ARG;
    if (out_dt != QFP4_BF16 && out_dt != QFP4_F32) return QFP4_ERR_ARG;
    if (M * K > 0 && (!codes || !scales || !out)) return QFP4_ERR_ARG;
    if (fmt == QFP4_NVFP4 && !tscale) return QFP4_ERR_ARG;
    if (K % (fmt == QFP4_MXFP4 ? 32 : 16)) return QFP4_ERR_SHAPE;
    if (!ok_align(codes) || !ok_align(scales) || !ok_align(out)) return QFP4_ERR_ALIGN;
    return dequantize(codes, scales, tscale, M * K, fmt, out_dt, out, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t qfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    return gemm_workspace(M, N, K, fmt);
}

// shape rules shared by both GEMM entry points
static int gemm_shape_check(int64_t M, int64_t N, int64_t K, qfp4_dtype out_dt)
{
    if (M < 0 || N < 0 || K < 0) return QFP4_ERR_SHAPE;
    if (K % 32) return QFP4_ERR_SHAPE;
    if (N % (out_dt == QFP4_F32 ? 4 : 8)) return QFP4_ERR_SHAPE;
    if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return QFP4_ERR_SHAPE;
    return QFP4_OK;
}

extern "C" int qfp4_gemm_blockscaled(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale,
                                     const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale,
                                     int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, qfp4_dtype out_dt, void *out,
                                     void *workspace, size_t workspace_bytes, qfp4_stream_t stream)
{
    if (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4 && fmt != QFP4_MXFP8) return QFP4_ERR_ARG;
    if (out_dt != QFP4_BF16 && out_dt != QFP4_F32) return QFP4_ERR_ARG;
    int st = gemm_shape_check(M, N, K, out_dt);
    if (st != QFP4_OK) return st;
    if (M * N > 0 && (!A_codes || !A_scales || !B_codes || !B_scales || !out)) return QFP4_ERR_ARG;
    if (fmt == QFP4_NVFP4 && M * N > 0 && (!A_tscale || !B_tscale)) return QFP4_ERR_ARG;
    if (!ok_align(A_codes) || !ok_align(A_scales) || !ok_align(B_codes) || !ok_align(B_scales) || !ok_align(out) ||
        !ok_align(workspace))
        return QFP4_ERR_ALIGN;
    if (M * N == 0) return QFP4_OK;
    if (K == 0) return cudaMemsetAsync(out, 0, M * N * (out_dt == QFP4_F32 ? 4 : 2),
                                       reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? QFP4_OK : QFP4_ERR_CUDA;
    if (!workspace || workspace_bytes < gemm_workspace(M, N, K, fmt)) return QFP4_ERR_ARG;
    return gemm_blockscaled(A_codes, A_scales, A_tscale, B_codes, B_scales, B_tscale, M, N, K, fmt, out_dt, out,
                            workspace, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t qfp4_gemm_fused_rq_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    return gemm_fused_rq_workspace(M, N, K, fmt);
}

extern "C" int qfp4_gemm_fused_rq_workspace_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, size_t *codes_off,
                                                   size_t *scales_off, size_t *tscale_off)
{
    if (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4) return QFP4_ERR_ARG;
    if (!codes_off || !scales_off || !tscale_off) return QFP4_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return QFP4_ERR_SHAPE;
    gemm_fused_rq_layout(M, N, K, fmt, codes_off, scales_off, tscale_off);
    return QFP4_OK;
}

extern "C" int qfp4_gemm_fused_rq_ex(const void *A_bf16, int64_t M, int64_t K, int rotate, int four6, qfp4_fmt fmt,
                                     const float *A_amax_in, float *A_amax_out, const uint8_t *B_codes,
                                     const uint8_t *B_scales, const float *B_tscale, int64_t N, void *workspace,
                                     size_t workspace_bytes, qfp4_dtype out_dt, void *out, qfp4_stream_t stream)
{
    if (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4) return QFP4_ERR_ARG;
    if (out_dt != QFP4_BF16 && out_dt != QFP4_F32) return QFP4_ERR_ARG;
    int st = gemm_shape_check(M, N, K, out_dt);
    if (st != QFP4_OK) return st;
    if (M * N > 0 && (!A_bf16 || !B_codes || !B_scales || !out)) return QFP4_ERR_ARG;
    if (fmt == QFP4_NVFP4 && M * N > 0 && !B_tscale) return QFP4_ERR_ARG;
    if (four6 && fmt != QFP4_NVFP4) return QFP4_ERR_UNSUPPORTED;
    if ((A_amax_in || A_amax_out) && fmt != QFP4_NVFP4) return QFP4_ERR_UNSUPPORTED;
    if (rotate && K % 128) return QFP4_ERR_SHAPE;
    if (!ok_align(A_bf16) || !ok_align(B_codes) || !ok_align(B_scales) || !ok_align(out) || !ok_align(workspace))
        return QFP4_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (M * N == 0 || K == 0) {
        if (A_amax_out && cudaMemsetAsync(A_amax_out, 0, sizeof(float), s) != cudaSuccess) return QFP4_ERR_CUDA;
        if (M * N == 0) return QFP4_OK;
        return cudaMemsetAsync(out, 0, M * N * (out_dt == QFP4_F32 ? 4 : 2), s) == cudaSuccess ? QFP4_OK
                                                                                               : QFP4_ERR_CUDA;
    }
    if (!workspace || workspace_bytes < gemm_fused_rq_workspace(M, N, K, fmt)) return QFP4_ERR_ARG;
    return gemm_fused_rq(A_bf16, M, K, rotate, four6, fmt, B_codes, B_scales, B_tscale, N, workspace, out_dt, out, s,
                         A_amax_in, A_amax_out);
}

extern "C" int qfp4_gemm_fused_rq(const void *A_bf16, int64_t M, int64_t K, int rotate, int four6, qfp4_fmt fmt,
                                  const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale, int64_t N,
                                  void *workspace, size_t workspace_bytes, qfp4_dtype out_dt, void *out,
                                  qfp4_stream_t stream)
{
    return qfp4_gemm_fused_rq_ex(A_bf16, M, K, rotate, four6, fmt, nullptr, nullptr, B_codes, B_scales, B_tscale, N,
                                 workspace, workspace_bytes, out_dt, out, stream);
}
