// dequant_fp32scale.cu -- dequantize (exact value, one rounding to the
// output type) and the FP32-scale quantize modes of the low-bit blog (§1-§2:
// S = |W|max / 6 per tensor, per row, or per group of 16 / 32).
#include "qfp4_common.cuh"

namespace qfp4 {

// binary64 -> bfloat16, round to nearest even: 8 significant bits with the
// binary32 exponent range (subnormal quantum 2^-133).
__device__ __forceinline__ uint16_t f64_to_bf16_rn(double v)
{
    const double a = fabs(v);
    uint32_t u = 0;
    if (a != 0.0) {
        const int e = ilogb(a);
        const int qe = max(e - 7, -133);
        const double r = ldexp(rint(ldexp(a, -qe)), qe);    // exact scalings, one rounding
        u = __float_as_uint(static_cast<float>(r));         // r fits bfloat16, so binary32
    }
    return static_cast<uint16_t>((u >> 16) | (signbit(v) ? 0x8000u : 0u));
}

__device__ __forceinline__ double e2m1_value_f64(uint32_t c)
{
    const uint32_t E = (c >> 1) & 3u, m = c & 1u;
    const double mag = (E == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, static_cast<int>(E) - 1);
    return (c & 8u) ? -mag : mag;
}

// One thread: 16 consecutive elements (one NVFP4 block, half an MXFP4 group).
template <int FMT, int OUT>
__global__ void __launch_bounds__(256) k_dequant(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                                                 const float *__restrict__ tscale, int64_t n, void *out)
{
    const int64_t chunks = n / 16;
    const double st = FMT == QFP4_NVFP4 ? static_cast<double>(*tscale) : 1.0;
    for (int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; c < chunks;
         c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t e0 = c * 16;
        const uint2 w = *reinterpret_cast<const uint2 *>(codes + e0 / 2);
        const uint32_t sb = scales[FMT == QFP4_MXFP4 ? e0 / 32 : e0 / 16];
        const double sc = FMT == QFP4_MXFP4 ? ldexp(1.0, static_cast<int>(sb) - 127)
                                            : static_cast<double>(e4m3_value(sb)) * st;
        double d[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t code = ((i < 8 ? w.x : w.y) >> (4 * (i & 7))) & 15u;
            d[i] = e2m1_value_f64(code) * sc;                 // exact: <= 31 significant bits
        }
        if (OUT == QFP4_F32) {
            float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + e0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o[q] = make_float4(__double2float_rn(d[4 * q]), __double2float_rn(d[4 * q + 1]),
                                   __double2float_rn(d[4 * q + 2]), __double2float_rn(d[4 * q + 3]));
        } else {
            uint32_t h[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                h[q] = static_cast<uint32_t>(f64_to_bf16_rn(d[2 * q])) |
                       (static_cast<uint32_t>(f64_to_bf16_rn(d[2 * q + 1])) << 16);
            uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + e0);
            o[0] = make_uint4(h[0], h[1], h[2], h[3]);
            o[1] = make_uint4(h[4], h[5], h[6], h[7]);
        }
    }
}

int dequantize(const uint8_t *codes, const uint8_t *scales, const float *tscale, int64_t n, qfp4_fmt fmt,
               qfp4_dtype out_dt, void *out, cudaStream_t stream)
{
    if (n == 0) return QFP4_OK;
    const int64_t chunks = n / 16;
    const int grid = static_cast<int>(imin<int64_t>((chunks + 255) / 256, 8 * num_sms()));
    if (fmt == QFP4_MXFP4) {
        if (out_dt == QFP4_F32) k_dequant<QFP4_MXFP4, QFP4_F32><<<grid, 256, 0, stream>>>(codes, scales, tscale, n, out);
        else k_dequant<QFP4_MXFP4, QFP4_BF16><<<grid, 256, 0, stream>>>(codes, scales, tscale, n, out);
    } else {
        if (out_dt == QFP4_F32) k_dequant<QFP4_NVFP4, QFP4_F32><<<grid, 256, 0, stream>>>(codes, scales, tscale, n, out);
        else k_dequant<QFP4_NVFP4, QFP4_BF16><<<grid, 256, 0, stream>>>(codes, scales, tscale, n, out);
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

// ---------------------------------------------------------------- FP32-scale modes
template <typename T>
__device__ __forceinline__ float ld_elem(const T *x, int64_t i)
{
    if (sizeof(T) == 4) return reinterpret_cast<const float *>(x)[i];
    return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t *>(x)[i]) << 16);
}

__device__ __forceinline__ float block_max_any(float m, float *red)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        m = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) red[0] = m;
    }
    __syncthreads();
    return red[0];
}

// 16 elements [e0, e0+16) under scale S -> 2 code words.
template <typename T>
__device__ __forceinline__ void fp32s_chunk(const T *x, int64_t e0, float S, uint8_t *codes)
{
    uint32_t w[2] = {0u, 0u};
    if (S != 0.0f) {
        float q[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(ld_elem(x, e0 + i), S);
        w[0] = e2m1x8_rne(q);
        w[1] = e2m1x8_rne(q + 8);
    }
    *reinterpret_cast<uint2 *>(codes + e0 / 2) = make_uint2(w[0], w[1]);
}

template <typename T>
__global__ void __launch_bounds__(256) k_absmax_partials(const T *x, int64_t n, float *partials)
{
    __shared__ float red[32];
    float m = 0.0f;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        m = fmaxf(m, fabsf(ld_elem(x, i)));
    m = block_max_any(m, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

template <typename T>
__global__ void __launch_bounds__(256) k_fp32s_tensor(const T *x, int64_t n, const float *partials, int n_parts,
                                                      uint8_t *codes, float *scales)
{
    __shared__ float red[32];
    float m = 0.0f;
    for (int i = threadIdx.x; i < n_parts; i += blockDim.x) m = fmaxf(m, partials[i]);
    m = block_max_any(m, red);
    const float S = __fdiv_rn(m, 6.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) scales[0] = S;
    for (int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; c < n / 16;
         c += static_cast<int64_t>(gridDim.x) * blockDim.x)
        fp32s_chunk(x, c * 16, S, codes);
}

template <typename T>
__global__ void __launch_bounds__(256) k_fp32s_row(const T *x, int64_t K, uint8_t *codes, float *scales)
{
    __shared__ float red[32];
    const int64_t i = blockIdx.x;
    float m = 0.0f;
    for (int64_t j = threadIdx.x; j < K; j += blockDim.x) m = fmaxf(m, fabsf(ld_elem(x, i * K + j)));
    m = block_max_any(m, red);
    const float S = __fdiv_rn(m, 6.0f);
    if (threadIdx.x == 0) scales[i] = S;
    for (int64_t c = threadIdx.x; c < K / 16; c += blockDim.x) fp32s_chunk(x, i * K + c * 16, S, codes);
}

template <typename T, int G>
__global__ void __launch_bounds__(256) k_fp32s_group(const T *x, int64_t n, uint8_t *codes, float *scales)
{
    const int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (q >= n / G) return;
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < G; ++i) m = fmaxf(m, fabsf(ld_elem(x, q * G + i)));
    const float S = __fdiv_rn(m, 6.0f);
    scales[q] = S;
#pragma unroll
    for (int c = 0; c < G / 16; ++c) fp32s_chunk(x, q * G + 16 * c, S, codes);
}

template <typename T>
static int fp32scale_t(const T *x, int64_t M, int64_t K, qfp4_gran gran, uint8_t *codes, float *scales,
                       float *partials, cudaStream_t stream)
{
    const int64_t n = M * K;
    if (n == 0) return QFP4_OK;
    switch (gran) {
    case QFP4_GRAN_TENSOR: {
        const int grid = static_cast<int>(imin<int64_t>((n + 255) / 256, num_sms()));
        k_absmax_partials<T><<<grid, 256, 0, stream>>>(x, n, partials);
        QFP4_LAUNCH_CHECK();
        const int g2 = static_cast<int>(imin<int64_t>((n / 16 + 255) / 256, 4 * num_sms()));
        k_fp32s_tensor<T><<<g2, 256, 0, stream>>>(x, n, partials, grid, codes, scales);
        break;
    }
    case QFP4_GRAN_ROW:
        k_fp32s_row<T><<<static_cast<unsigned>(M), 256, 0, stream>>>(x, K, codes, scales);
        break;
    case QFP4_GRAN_GROUP16:
        k_fp32s_group<T, 16><<<static_cast<unsigned>((n / 16 + 255) / 256), 256, 0, stream>>>(x, n, codes, scales);
        break;
    default:
        k_fp32s_group<T, 32><<<static_cast<unsigned>((n / 32 + 255) / 256), 256, 0, stream>>>(x, n, codes, scales);
        break;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

int quantize_fp32scale(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_gran gran, uint8_t *codes,
                       float *scales, float *partials, cudaStream_t stream)
{
    if (xdt == QFP4_F32)
        return fp32scale_t(static_cast<const float *>(x), M, K, gran, codes, scales, partials, stream);
    return fp32scale_t(static_cast<const uint16_t *>(x), M, K, gran, codes, scales, partials, stream);
}

}  // namespace qfp4
