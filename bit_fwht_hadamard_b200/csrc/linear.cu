// linear.cu -- the Quartet-style linear layer on the library's kernels:
// the forward Y = X W^T as an FP4 GEMM of operands rotated and quantized
// along K, and the backward dX = G W and dW = G^T X on operands quantized
// once with their transposes (2D 16 x 16 NVFP4 blocks) or as MXFP8 rows and
// columns.
//
// Method: [QN] Hadamard rotation (y = xW^T = (xH)(WH)^T), forward/backward
// precision split (FP4 forward, FP4 or FP8 backward), QuTLASS (MXFP4 /
// NVFP4 GEMMs, stochastic rounding for the gradients); [TI] (one 2D-block
// quantization serves X and X^T; MXFP8 operands).  Every step runs in the
// kernels of quantize1d.cu, quantize2d.cu and gemm.cu; this file only lays
// out the workspace and orders the launches on the caller's stream.
#include "qfp4_common.cuh"
#include "quantize1d.cuh"

namespace qfp4 {

int quantize2d(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_fmt fmt, qfp4_round rounding,
               uint64_t seed, uint8_t *codes, uint8_t *scales, uint8_t *codesT, uint8_t *scalesT, float *tscale,
               float *partials, cudaStream_t stream, const QuantOpts &opt);
int quantize_mxfp8(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_round rounding, uint64_t seed,
                   uint8_t *codes, uint8_t *scales, uint8_t *codesT, uint8_t *scalesT, cudaStream_t stream);
int quantize_mxfp8_columns(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_round rounding, uint64_t seed,
                           uint8_t *codesT, uint8_t *scalesT, cudaStream_t stream);
int gemm_blockscaled(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale, const uint8_t *B_codes,
                     const uint8_t *B_scales, const float *B_tscale, int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
                     qfp4_dtype out_dt, void *out, void *workspace, cudaStream_t stream);
size_t gemm_workspace(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);

// Bump allocator over the caller's workspace (256-byte aligned pieces).
struct Carve {
    uint8_t *base;
    size_t off = 0;
    template <typename T>
    T *take(size_t bytes)
    {
        T *p = reinterpret_cast<T *>(base ? base + off : nullptr);
        off += (bytes + 255) & ~size_t(255);
        return p;
    }
};

// One quantized operand: codes, scales, and (FP4 2D) the transposed pair.
struct Operand {
    uint8_t *codes, *scales, *codesT, *scalesT;
    float *tscale;
};

// ------------------------------------------------------------------ forward
// X (M x K) and W (N x K) bf16, each rotated along K and quantized (fmt,
// RNE, four6), then Y = Q(XH) Q(WH)^T.
static size_t linear_fwd_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, uint8_t *ws, Operand *X, Operand *W,
                                float **partials, uint8_t **gemm_ws)
{
    const int g = fmt == QFP4_MXFP4 ? 32 : 16;
    Carve c{ws};
    Operand x{}, w{};
    x.codes = c.take<uint8_t>(M * K / 2);
    x.scales = c.take<uint8_t>(M * (K / g));
    x.tscale = c.take<float>(sizeof(float));
    w.codes = c.take<uint8_t>(N * K / 2);
    w.scales = c.take<uint8_t>(N * (K / g));
    w.tscale = c.take<float>(sizeof(float));
    float *part = c.take<float>(sizeof(float) * kMaxPartials);
    uint8_t *gw = c.take<uint8_t>(gemm_workspace(M, N, K, fmt));
    if (X) *X = x;
    if (W) *W = w;
    if (partials) *partials = part;
    if (gemm_ws) *gemm_ws = gw;
    return c.off;
}

static int linear_fwd_check(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, int four6, qfp4_dtype out_dt)
{
    if (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4) return QFP4_ERR_ARG;
    if (out_dt != QFP4_BF16 && out_dt != QFP4_F32) return QFP4_ERR_ARG;
    if (four6 && fmt != QFP4_NVFP4) return QFP4_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K < 0) return QFP4_ERR_SHAPE;
    if (K % 128) return QFP4_ERR_SHAPE;                     // rotation blocks along K
    if (N % (out_dt == QFP4_F32 ? 4 : 8)) return QFP4_ERR_SHAPE;
    if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return QFP4_ERR_SHAPE;
    return QFP4_OK;
}

// ------------------------------------------------------------------ backward
// G (M x N), X (M x K), W (N x K) bf16.  NVFP4: 2D 16 x 16 blocks, G with
// Philox SR, X and W with RNE, each giving its transpose from the same pass.
// MXFP8: G rows + columns with SR, W and X columns with RNE.
//   dX = G W:   A = G   (M x N, groups along N), B = W^T (K x N)
//   dW = G^T X: A = G^T (N x M, groups along M), B = X^T (K x M)
static size_t linear_bwd_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, uint8_t *ws, Operand *G, Operand *W,
                                Operand *X, float **partials, uint8_t **gemm_ws)
{
    Carve c{ws};
    Operand gq{}, wq{}, xq{};
    if (fmt == QFP4_NVFP4) {
        gq.codes = c.take<uint8_t>(M * N / 2);
        gq.scales = c.take<uint8_t>(M * (N / 16));
        gq.codesT = c.take<uint8_t>(N * M / 2);
        gq.scalesT = c.take<uint8_t>(N * (M / 16));
        gq.tscale = c.take<float>(sizeof(float));
        wq.codes = c.take<uint8_t>(N * K / 2);
        wq.scales = c.take<uint8_t>(N * (K / 16));
        wq.codesT = c.take<uint8_t>(K * N / 2);
        wq.scalesT = c.take<uint8_t>(K * (N / 16));
        wq.tscale = c.take<float>(sizeof(float));
        xq.codes = c.take<uint8_t>(M * K / 2);
        xq.scales = c.take<uint8_t>(M * (K / 16));
        xq.codesT = c.take<uint8_t>(K * M / 2);
        xq.scalesT = c.take<uint8_t>(K * (M / 16));
        xq.tscale = c.take<float>(sizeof(float));
    } else {
        gq.codes = c.take<uint8_t>(M * N);
        gq.scales = c.take<uint8_t>(M * (N / 32));
        gq.codesT = c.take<uint8_t>(N * M);
        gq.scalesT = c.take<uint8_t>(N * (M / 32));
        wq.codesT = c.take<uint8_t>(K * N);
        wq.scalesT = c.take<uint8_t>(K * (N / 32));
        xq.codesT = c.take<uint8_t>(K * M);
        xq.scalesT = c.take<uint8_t>(K * (M / 32));
    }
    float *part = c.take<float>(sizeof(float) * kMaxPartials);
    const size_t gws = imax(gemm_workspace(M, K, N, fmt), gemm_workspace(N, K, M, fmt));
    uint8_t *gw = c.take<uint8_t>(gws);
    if (G) *G = gq;
    if (W) *W = wq;
    if (X) *X = xq;
    if (partials) *partials = part;
    if (gemm_ws) *gemm_ws = gw;
    return c.off;
}

static int linear_bwd_check(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, qfp4_dtype out_dt)
{
    if (fmt != QFP4_NVFP4 && fmt != QFP4_MXFP8) return QFP4_ERR_ARG;
    if (out_dt != QFP4_BF16 && out_dt != QFP4_F32) return QFP4_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return QFP4_ERR_SHAPE;
    // inner dimensions of the two GEMMs (N and M) in whole 32-groups; K in
    // whole 2D tiles (16) or groups (32), and a multiple of the output store width
    if (M % 32 || N % 32) return QFP4_ERR_SHAPE;
    if (K % (fmt == QFP4_NVFP4 ? 16 : 32)) return QFP4_ERR_SHAPE;
    if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return QFP4_ERR_SHAPE;
    return QFP4_OK;
}

}  // namespace qfp4

using namespace qfp4;

extern "C" size_t qfp4_linear_forward_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    if (M <= 0 || N <= 0 || K <= 0 || (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4)) return 0;
    return linear_fwd_layout(M, N, K, fmt, nullptr, nullptr, nullptr, nullptr, nullptr);
}

extern "C" int qfp4_linear_forward(const void *X, const void *W, int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
                                   int four6, qfp4_dtype out_dt, void *Y, void *workspace, size_t workspace_bytes,
                                   qfp4_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const int st = linear_fwd_check(M, N, K, fmt, four6, out_dt);
    if (st != QFP4_OK) return st;
    if (M * N > 0 && (!X || !W || !Y)) return QFP4_ERR_ARG;
    if (!aligned16(X) || !aligned16(W) || !aligned16(Y) || !aligned16(workspace)) return QFP4_ERR_ALIGN;
    if (M * N == 0) return QFP4_OK;
    if (K == 0)
        return cudaMemsetAsync(Y, 0, M * N * (out_dt == QFP4_F32 ? 4 : 2), stream) == cudaSuccess ? QFP4_OK
                                                                                                   : QFP4_ERR_CUDA;
    if (!workspace || workspace_bytes < qfp4_linear_forward_workspace_bytes(M, N, K, fmt)) return QFP4_ERR_ARG;
    Operand xq, wq;
    float *partials;
    uint8_t *gws;
    linear_fwd_layout(M, N, K, fmt, static_cast<uint8_t *>(workspace), &xq, &wq, &partials, &gws);
    int s = quantize1d(X, QFP4_BF16, M * K, fmt, QFP4_RNE, 1, four6, 0, xq.codes, xq.scales, xq.tscale, partials,
                       nullptr, stream);
    if (s != QFP4_OK) return s;
    s = quantize1d(W, QFP4_BF16, N * K, fmt, QFP4_RNE, 1, four6, 0, wq.codes, wq.scales, wq.tscale, partials, nullptr,
                   stream);
    if (s != QFP4_OK) return s;
    return gemm_blockscaled(xq.codes, xq.scales, xq.tscale, wq.codes, wq.scales, wq.tscale, M, N, K, fmt, out_dt, Y,
                            gws, stream);
}

extern "C" size_t qfp4_linear_backward_workspace_bytes(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    if (M <= 0 || N <= 0 || K <= 0 || (fmt != QFP4_NVFP4 && fmt != QFP4_MXFP8)) return 0;
    return linear_bwd_layout(M, N, K, fmt, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
}

extern "C" int qfp4_linear_backward(const void *G, const void *X, const void *W, int64_t M, int64_t N, int64_t K,
                                    qfp4_fmt fmt, uint64_t seed, qfp4_dtype out_dt, void *dX, void *dW,
                                    void *workspace, size_t workspace_bytes, qfp4_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const int st = linear_bwd_check(M, N, K, fmt, out_dt);
    if (st != QFP4_OK) return st;
    if (!dX && !dW) return QFP4_ERR_ARG;
    const int64_t work = M * N * K;
    if (work > 0 && (!G || (dX && !W) || (dW && !X))) return QFP4_ERR_ARG;
    if (!aligned16(G) || !aligned16(X) || !aligned16(W) || !aligned16(dX) || !aligned16(dW) ||
        !aligned16(workspace))
        return QFP4_ERR_ALIGN;
    const size_t osz = out_dt == QFP4_F32 ? 4 : 2;
    if (work == 0) {
        // an empty inner dimension gives zero gradients; an empty output is nothing to do
        if (dX && M * K > 0 && cudaMemsetAsync(dX, 0, M * K * osz, stream) != cudaSuccess) return QFP4_ERR_CUDA;
        if (dW && N * K > 0 && cudaMemsetAsync(dW, 0, N * K * osz, stream) != cudaSuccess) return QFP4_ERR_CUDA;
        return QFP4_OK;
    }
    if (!workspace || workspace_bytes < qfp4_linear_backward_workspace_bytes(M, N, K, fmt)) return QFP4_ERR_ARG;
    Operand gq, wq, xq;
    float *partials;
    uint8_t *gws;
    linear_bwd_layout(M, N, K, fmt, static_cast<uint8_t *>(workspace), &gq, &wq, &xq, &partials, &gws);
    int s;
    if (fmt == QFP4_NVFP4) {
        s = quantize2d(G, QFP4_BF16, M, N, QFP4_NVFP4, QFP4_SR, seed, gq.codes, gq.scales, gq.codesT, gq.scalesT,
                       gq.tscale, partials, stream, QuantOpts{});
        if (s != QFP4_OK) return s;
        if (dX) {
            s = quantize2d(W, QFP4_BF16, N, K, QFP4_NVFP4, QFP4_RNE, 0, wq.codes, wq.scales, wq.codesT, wq.scalesT,
                           wq.tscale, partials, stream, QuantOpts{});
            if (s != QFP4_OK) return s;
        }
        if (dW) {
            s = quantize2d(X, QFP4_BF16, M, K, QFP4_NVFP4, QFP4_RNE, 0, xq.codes, xq.scales, xq.codesT, xq.scalesT,
                           xq.tscale, partials, stream, QuantOpts{});
            if (s != QFP4_OK) return s;
        }
    } else {
        s = quantize_mxfp8(G, QFP4_BF16, M, N, QFP4_SR, seed, gq.codes, gq.scales, dW ? gq.codesT : nullptr,
                           dW ? gq.scalesT : nullptr, stream);
        if (s != QFP4_OK) return s;
        if (dX) {
            s = quantize_mxfp8_columns(W, QFP4_BF16, N, K, QFP4_RNE, 0, wq.codesT, wq.scalesT, stream);
            if (s != QFP4_OK) return s;
        }
        if (dW) {
            s = quantize_mxfp8_columns(X, QFP4_BF16, M, K, QFP4_RNE, 0, xq.codesT, xq.scalesT, stream);
            if (s != QFP4_OK) return s;
        }
    }
    if (dX) {
        s = gemm_blockscaled(gq.codes, gq.scales, gq.tscale, wq.codesT, wq.scalesT, wq.tscale, M, K, N, fmt, out_dt,
                             dX, gws, stream);
        if (s != QFP4_OK) return s;
    }
    if (dW)
        s = gemm_blockscaled(gq.codesT, gq.scalesT, gq.tscale, xq.codesT, xq.scalesT, xq.tscale, N, K, M, fmt, out_dt,
                             dW, gws, stream);
    return s;
}
