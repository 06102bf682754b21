// dequant_fp32scale.cu -- dequantize (exact value, one rounding to the
// output type) and the FP32-scale quantize modes of the low-bit blog (§1-§2:
// S = |W|max / 6 per tensor, per row, or per group of 16 / 32).
#include "qfp4_common.cuh"

namespace qfp4 {

// 2^(b - 128) for a byte b, as binary32 (2^-128 and 2^-127 are subnormal).
__device__ __forceinline__ float exp2_b128(uint32_t b)
{
    return __uint_as_float(b >= 2u ? (b - 1u) << 23 : 0x00200000u << b);
}

// E2M1 codes of four elements (16 bits, element t in bits 4t .. 4t + 3) as
// two bfloat16 pairs (exact: bfloat16 holds every E2M1 value).  The high and
// low bytes of the eight magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 (bf16 0x0000,
// 0x3F00, 0x3F80, 0x3FC0, 0x4000, 0x4040, 0x4080, 0x40C0) are two byte-permute
// tables indexed by the 3-bit magnitudes, two more permutes interleave them,
// and the sign bits go to bits 15 and 31.
__device__ __forceinline__ void e2m1x4_to_bf16x2(uint32_t w16, uint32_t &p01, uint32_t &p23)
{
    const uint32_t sel = w16 & 0x7777u;
    const uint32_t hi = __byte_perm(0x3F3F3F00u, 0x40404040u, sel);
    const uint32_t lo = __byte_perm(0xC0800000u, 0xC0804000u, sel);
    p01 = __byte_perm(lo, hi, 0x5140u) | ((w16 << 12) & 0x8000u) | ((w16 << 24) & 0x80000000u);
    p23 = __byte_perm(lo, hi, 0x7362u) | ((w16 << 4) & 0x8000u) | ((w16 << 16) & 0x80000000u);
}

// Four consecutive elements e0 .. e0 + 3 from their two code bytes w16 and
// their scale byte sb.  Every output is the exact value g * scale (* s_t)
// rounded once:
// - MXFP4: g * 2^(b-127) = (2 g) * 2^(b-128) has at most two significant bits
//   and an exponent >= -129, so it is exact in binary32 and in bfloat16.
// - NVFP4: m = g * dec(enc) is exact (at most 6 significant bits, inside the
//   normal range), and fl(m * s_t) is the one rounding (binary32 out); for
//   bfloat16 out the product is formed exactly in binary64 and converted
//   once (cvt.rn.bf16.f64: one rounding, which the tests check on products
//   placed on and next to bfloat16 midpoints).
// A scale byte that encodes NaN (E8M0 0xFF, E4M3 0x7F / 0xFF) gives NaN.
template <int FMT, int OUT>
__device__ __forceinline__ void dequant_quad(uint32_t w16, uint32_t sb, float st, int64_t e0, void *out)
{
    uint32_t p01, p23;
    e2m1x4_to_bf16x2(w16, p01, p23);
    const uint64_t g[2] = {f2pack(__uint_as_float(p01 << 16), __uint_as_float(p01 & 0xFFFF0000u)),
                           f2pack(__uint_as_float(p23 << 16), __uint_as_float(p23 & 0xFFFF0000u))};
    uint64_t v[2], m[2];
    const double st64 = st;
    if (FMT == QFP4_MXFP4) {
        const float h = sb == 255u ? __uint_as_float(0x7FC00000u) : exp2_b128(sb);   // E8M0 0xFF: NaN
        const uint64_t two = f2pack(2.0f, 2.0f), h2 = f2pack(h, h);
#pragma unroll
        for (int j = 0; j < 2; ++j) v[j] = f2mul(f2mul(g[j], two), h2);
    } else {
        const float d = (sb & 0x7Fu) == 0x7Fu ? __uint_as_float(0x7FC00000u) : e4m3_value(sb);   // E4M3 NaN
        const uint64_t d2 = f2pack(d, d), st2 = f2pack(st, st);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            m[j] = f2mul(g[j], d2);
            v[j] = f2mul(m[j], st2);
        }
    }
    if (OUT == QFP4_F32) {
        float a, b, c, d;
        f2unpack(v[0], a, b);
        f2unpack(v[1], c, d);
        *reinterpret_cast<float4 *>(static_cast<float *>(out) + e0) = make_float4(a, b, c, d);
    } else {
        uint32_t h[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float p[2], mm[2];
            f2unpack(v[j], p[0], p[1]);
            uint32_t b16[2];
            if (FMT == QFP4_MXFP4) {
                b16[0] = __float_as_uint(p[0]) >> 16;          // exact in bfloat16
                b16[1] = __float_as_uint(p[1]) >> 16;
            } else {
                // m * s_t is exact in binary64 (at most 6 + 24 significant
                // bits); one conversion rounds it to bfloat16
                f2unpack(m[j], mm[0], mm[1]);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    uint16_t r16;
                    asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r16) : "d"(static_cast<double>(mm[t]) * st64));
                    b16[t] = mm[t] != mm[t] ? 0x7FC0u : r16;
                }
            }
            h[j] = b16[0] | (b16[1] << 16);
        }
        *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(out) + e0) = make_uint2(h[0], h[1]);
    }
}

// Four consecutive elements a thread (a warp covers 128 elements: 64
// contiguous code bytes in, 512 (binary32) or 256 (bf16) contiguous bytes
// out), four such quads a thread per loop iteration with all their loads
// issued first.  n % 16 == 0 (checked on the host).
template <int FMT, int OUT>
__global__ void __launch_bounds__(256) k_dequant(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                                                  const float *__restrict__ tscale, int64_t n, void *out)
{
    constexpr int U = 4;
    const int64_t quads = n / 4;
    const float st = FMT == QFP4_NVFP4 ? *tscale : 1.0f;
    const int64_t nth = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const uint16_t *c16 = reinterpret_cast<const uint16_t *>(codes);
    for (int64_t base = 0; base < quads; base += U * nth) {
        uint32_t w[U], sb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t qd = base + t0 + u * nth;
            w[u] = qd < quads ? c16[qd] : 0u;
            sb[u] = qd < quads ? scales[FMT == QFP4_MXFP4 ? qd / 8 : qd / 4] : 0u;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t qd = base + t0 + u * nth;
            if (qd < quads) dequant_quad<FMT, OUT>(w[u], sb[u], st, 4 * qd, out);
        }
    }
}

int dequantize(const uint8_t *codes, const uint8_t *scales, const float *tscale, int64_t n, qfp4_fmt fmt,
               qfp4_dtype out_dt, void *out, cudaStream_t stream)
{
    if (n == 0) return QFP4_OK;
    const int64_t quads = n / 4;
    const int grid = static_cast<int>(imin<int64_t>((quads + 1023) / 1024, 8 * num_sms()));
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
