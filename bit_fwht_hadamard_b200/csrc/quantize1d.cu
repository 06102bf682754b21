// quantize1d.cu -- 1D FP4 microscaling quantize (MXFP4 / NVFP4), optional
// 128-point Walsh-Hadamard rotation, RNE or Philox stochastic rounding,
// optional four-over-six; the NVFP4 tensor-amax pass; and the row-wise MXFP8
// quantize, which shares the same kernel.
//
// Method ([QN] Hadamard rotation + QuTLASS online quantization; [LB] §FP4,
// §2, §3, §7; [46] Methodology): per 128 block along K an optional
// normalised FWHT, per group of g a scale (E8M0 truncation-free for MXFP4,
// E4M3 under the tensor scale for NVFP4), v = x / S, round onto E2M1.
//
// Layout: the input is a flat stream of n = M*K elements (groups never cross
// rows because K % g == 0, and rotation blocks never cross rows because
// K % 128 == 0).  Main (bf16) kernel: one persistent CTA per SM, 20 warps
// (16 with four-over-six), each warp with its own 2-stage ring of 4 KiB
// tiles (32 rows of 64 bf16) brought in by TMA with 128-byte swizzle; an SM
// takes a contiguous range of tiles and its warps interleave over it.  A
// thread owns one 64-element row as 32 packed binary32 pairs; the
// rotation's stages h = 2..32 run as f32x2 operations inside the thread and
// h = 64 pairs it with the neighbouring lane.  The direct kernel serves
// binary32 inputs and the ragged tail (n % 64) of bf16 inputs.
#include "qfp4_common.cuh"
#include "quantize1d.cuh"

namespace qfp4 {


// E2M1 code -> binary32 value (exact), from the bit fields.
__device__ __forceinline__ float e2m1_value(uint32_t c)
{
    const uint32_t E = (c >> 1) & 3u, m = c & 1u;
    const float mag = (E == 0) ? (m ? 0.5f : 0.0f) : __uint_as_float(((E + 126u) << 23) | (m << 22));
    return (c & 8u) ? -mag : mag;
}

// Walsh-Hadamard transform of a 128 block held as 64 values in each of two
// lanes (lane^1 partner; the even lane holds elements 0..63).  Stages
// h = 1..32 are local, h = 64 crosses the pair, then the 1/sqrt(128) scale.
__device__ __forceinline__ void fwht128_pair(float (&v)[64], bool upper)
{
#pragma unroll
    for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const float o = __shfl_xor_sync(0xFFFFFFFFu, v[i], 1);
        v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
    const float c = inv_sqrt128();
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __fmul_rn(v[i], c);
}

// Result of one unit: 64 nibbles (8 words) and up to 4 scale bytes.
struct UnitOut {
    uint32_t codes[8];
    uint32_t scales;        // byte g = scale of group g within the unit
};

// ---------------------------------------------------------------- NVFP4 without a division per element
// fl(a / b) (b > 0) from y = fl(1/b), correctly rounded, and two FMA
// corrections: q0 = fl(a y) is within 1.5 ulp of a / b; q1 = fl(q0 + r0 y),
// r0 = fl(a - b q0), is within one ulp (faithful); and with q1 faithful the
// remainder r1 = a - b q1 is exact and q2 = fl(q1 + r1 y) is fl(a / b)
// (P. Markstein, IBM J. Res. Dev. 34(1), 1990: a reciprocal within half an
// ulp plus a faithful quotient give the correctly rounded one).  This needs
// normal intermediate values; quotients below the normal range only decide
// a zero code, whose sign is taken from a.  nb = -b.
__device__ __forceinline__ float div_rn_by(float a, float y, float nb)
{
    float q = __fmul_rn(a, y);
    q = __fmaf_rn(__fmaf_rn(q, nb, a), y, q);
    return __fmaf_rn(__fmaf_rn(q, nb, a), y, q);
}

// The same on packed pairs; the sign of each a is put on its quotient.
__device__ __forceinline__ uint64_t div_rn_by2(uint64_t a, uint64_t y2, uint64_t nb2)
{
    uint64_t q = f2mul(a, y2);
    q = f2fma(f2fma(q, nb2, a), y2, q);
    q = f2fma(f2fma(q, nb2, a), y2, q);
    return q | (a & 0x8000000080000000ull);
}

// fl(x_i / S) for 16 values held as 8 packed pairs, S > 0, amax = max |x_i|.
// Outside S in [2^-125, 2^125] (1/S not normal), and when a quotient could
// overflow (a block scale saturated under a caller-supplied tensor amax far
// below the block's values), the IEEE division, whose infinities saturate
// like any magnitude beyond 6.
__device__ __forceinline__ void nv_quot16_pairs(const uint64_t *pp, float S, float amax, uint64_t *q)
{
    if (S >= 0x1p-125f && S <= 0x1p125f && amax <= S * 0x1p100f) {
        const float y = __frcp_rn(S);
        const uint64_t y2 = f2pack(y, y), nS2 = f2pack(-S, -S);
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = div_rn_by2(pp[j], y2, nS2);
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float a, b;
            f2unpack(pp[j], a, b);
            q[j] = f2pack(__fdiv_rn(a, S), __fdiv_rn(b, S));
        }
    }
}

// E2M1 round-to-nearest-even codes of fl(x_i / S): two words of nibbles.
__device__ __forceinline__ void nv_codes16_pairs(const uint64_t *pp, float S, float amax, uint32_t *w2)
{
    uint64_t q[8];
    nv_quot16_pairs(pp, S, amax, q);
    w2[0] = e2m1x8_rne_pairs(q[0], q[1], q[2], q[3]);
    w2[1] = e2m1x8_rne_pairs(q[4], q[5], q[6], q[7]);
}

// Quantize 16 values (8 packed pairs) under effective scale S (RNE): codes
// (2 words), and when `sse` is given the binary32 squared error of the
// dequantized values, sum(fl(fl(fl(g_i S) - x_i)^2)) as a fixed tree
// (i + 8 into i, then i + 4, i + 2, i + 1).
__device__ __forceinline__ void nv_block_rne_pairs(const uint64_t *pp, float S, float amax, uint32_t *w2, float *sse)
{
    if (S == 0.0f) w2[0] = w2[1] = 0u;
    else nv_codes16_pairs(pp, S, amax, w2);
    if (sse) {
        // Scalar IEEE operations: the multiply feeding the subtraction must
        // stay two roundings.  The packed f32x2 multiply, subtract and tree
        // gave different sums on B200 (153 of 16.8 M codes of the full-size
        // four-over-six test changed, with either E2M1 decode), and the sums
        // decide the selection.
        uint64_t g[8];
        e2m1x8_values(w2[0], g);
        e2m1x8_values(w2[1], g + 4);
        float e[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float g0, g1, x0, x1;
            f2unpack(g[j], g0, g1);
            f2unpack(pp[j], x0, x1);
            const float d0 = __fsub_rn(__fmul_rn(g0, S), x0), d1 = __fsub_rn(__fmul_rn(g1, S), x1);
            e[2 * j] = __fmul_rn(d0, d0);
            e[2 * j + 1] = __fmul_rn(d1, d1);
        }
#pragma unroll
        for (int h = 8; h >= 1; h >>= 1)
#pragma unroll
            for (int i = 0; i < h; ++i) e[i] = __fadd_rn(e[i], e[i + h]);
        *sse = e[0];
    }
}

// The same for 16 unpacked values.
__device__ __forceinline__ void nv_block_rne(const float *x, float S, float amax, uint32_t *w2, float *sse)
{
    uint64_t pp[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) pp[j] = f2pack(x[2 * j], x[2 * j + 1]);
    nv_block_rne_pairs(pp, S, amax, w2, sse);
}

// NVFP4 block scale bytes enc = E4M3_RNE(fl(fl(amax / d) / s_t)), d = 6 or 4,
// with the quotients from div_rn_by: fl(amax / 6) by y = fl(1/6), fl(amax / 4)
// is exact, and fl(t / s_t) by fl(1/s_t), worked out once per thread.  The
// fast path needs amax / d and 1/s_t normal; otherwise IEEE divisions.
// rule: QFP4_SCALE_DEFAULT (E4M3 nearest) or QFP4_SCALE_E4M3_UP (the least
// E4M3 value not below the quotient, so no element of the block clips).
// A quotient of 448 or more (also +inf, from a caller-supplied tensor amax
// far below the block's values) takes the largest byte, 0x7E.
struct NvScale {
    float s_t, y_t;
    bool fast;
    int rule;
};

__device__ __forceinline__ NvScale nv_scale_setup(float s_t, int rule = QFP4_SCALE_DEFAULT)
{
    NvScale z;
    z.s_t = s_t;
    z.fast = s_t >= 0x1p-120f && s_t <= 0x1p120f;
    z.y_t = z.fast ? __frcp_rn(s_t) : 0.0f;
    z.rule = rule;
    return z;
}

template <bool D6>
__device__ __forceinline__ uint32_t nv_scale_byte(float amax, const NvScale &z)
{
    float r;
    if (z.fast && amax >= 0x1p-120f) {
        const float t = D6 ? div_rn_by(amax, __uint_as_float(0x3E2AAAABu), -6.0f)   // fl(1/6)
                           : __fmul_rn(amax, 0.25f);
        r = div_rn_by(t, z.y_t, -z.s_t);
    } else {
        r = __fdiv_rn(__fdiv_rn(amax, D6 ? 6.0f : 4.0f), z.s_t);
    }
    if (!(r < 448.0f)) return 0x7Eu;              // saturated; a NaN from an overflowed chain too
    const uint32_t enc = e4m3_rne(r);
    return z.rule == QFP4_SCALE_E4M3_UP ? e4m3_up_byte(r, enc) : enc;
}

// Stochastic rounding of 16 (NVFP4) or 32 (MXFP4) values v (already divided
// by the scale) whose first element has logical index e (e % 4 == 0).
// Each value goes to its signed E2M1 grid value in binary32; eight of those
// then take one packed hardware conversion (exact: they are grid values).
template <int G>
__device__ __forceinline__ void sr_group(const float *v, uint64_t e, uint64_t seed, uint32_t *words)
{
#pragma unroll
    for (int w = 0; w < G / 8; ++w) {
        float r[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 rw = sr_words4(seed, (e >> 2) + 2 * w + h);
            r[4 * h + 0] = e2m1_sr_grid(v[8 * w + 4 * h + 0], rw.x);
            r[4 * h + 1] = e2m1_sr_grid(v[8 * w + 4 * h + 1], rw.y);
            r[4 * h + 2] = e2m1_sr_grid(v[8 * w + 4 * h + 2], rw.z);
            r[4 * h + 3] = e2m1_sr_grid(v[8 * w + 4 * h + 3], rw.w);
        }
        words[w] = e2m1x8_rne(r);
    }
}

// sr_group on values held as G / 2 packed pairs (e2m1_sr_grid2).
template <int G>
__device__ __forceinline__ void sr_group_pairs(const uint64_t *pp, uint64_t e, uint64_t seed, uint32_t *words)
{
#pragma unroll
    for (int w = 0; w < G / 8; ++w) {
        float r[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 rw = sr_words4(seed, (e >> 2) + 2 * w + h);
            f2unpack(e2m1_sr_grid2(pp[4 * w + 2 * h], rw.x, rw.y), r[4 * h + 0], r[4 * h + 1]);
            f2unpack(e2m1_sr_grid2(pp[4 * w + 2 * h + 1], rw.z, rw.w), r[4 * h + 2], r[4 * h + 3]);
        }
        words[w] = e2m1x8_rne(r);
    }
}

// binary32 squared error of 32 values x under codes w (4 words) and scale
// 2^k: sum(fl(fl(fl(g_i 2^k) - x_i)^2)) as a fixed tree (i + 16 into i, then
// + 8, + 4, + 2, + 1); g_i 2^k is exact.  The code values come from the E2M1
// bit fields (e2m1_value), not from the hardware nibble-pair conversion: on
// B200 that conversion, fed words just produced by cvt.rn.satfinite.e2m1x2
// in the same function, returned zeros for bytes 2-3 of the word.
__device__ __forceinline__ float mx_sse32(const float *x, const uint32_t *w, int k)
{
    const float sc = exp2i(k);
    float e[32];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float d = __fsub_rn(__fmul_rn(e2m1_value((w[t] >> (4 * u)) & 0xFu), sc), x[8 * t + u]);
            e[8 * t + u] = __fmul_rn(d, d);
        }
    }
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1)
#pragma unroll
        for (int i = 0; i < h; ++i) e[i] = __fadd_rn(e[i], e[i + h]);
    return e[0];
}

// Four-over-six on an MXFP4 group of 32 (RNE): the second candidate is the
// least k4 with 4 * 2^k4 >= amax; it replaces the rule's exponent k (codes w)
// only when its squared error is strictly lower.  Returns the kept exponent.
__device__ __forceinline__ int mx_four6(const float *x, float amax, int k, uint32_t *w)
{
    const int k4 = scale_exp(amax, 0u, 2);
    if (k4 == k) return k;
    const float m4 = exp2i(-k4);
    uint32_t w4[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float q8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) q8[u] = __fmul_rn(x[8 * t + u], m4);
        w4[t] = e2m1x8_rne(q8);
    }
    if (!(mx_sse32(x, w4, k4) < mx_sse32(x, w, k))) return k;
#pragma unroll
    for (int t = 0; t < 4; ++t) w[t] = w4[t];
    return k4;
}

template <int FMT, bool SR, bool FOUR6>
__device__ __forceinline__ void quant_unit(const float (&v)[64], uint64_t e0, const NvScale &nz, uint64_t seed,
                                           UnitOut &o)
{
    o.scales = 0u;
    if (FMT == QFP4_MXFP4) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[32 * g + i]));
            uint32_t *w = o.codes + 4 * g;
            if (amax == 0.0f) {                      // all-zero group: byte 0, +0 codes
                w[0] = w[1] = w[2] = w[3] = 0u;
                continue;
            }
            int k = mx_scale_exp(amax, nz.rule);
            const float mul = exp2i(-k);             // x * 2^-k == x / 2^k exactly
            float q[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) q[i] = __fmul_rn(v[32 * g + i], mul);
            if (SR) {
                sr_group<32>(q, e0 + 32 * g, seed, w);
            } else {
#pragma unroll
                for (int t = 0; t < 4; ++t) w[t] = e2m1x8_rne(q + 8 * t);
            }
            if (FOUR6) k = mx_four6(v + 32 * g, amax, k, w);
            o.scales |= static_cast<uint32_t>(k + 127) << (8 * g);
        }
    } else {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float *x = v + 16 * b;
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
            uint32_t *w = o.codes + 2 * b;
            uint32_t enc = 0u;
            float S = 0.0f;
            if (nz.s_t != 0.0f) {
                enc = nv_scale_byte<true>(amax, nz);
                S = __fmul_rn(e4m3_value(enc), nz.s_t);
            }
            if (FOUR6) {
                uint32_t w6[2], w4[2];
                float sse6, sse4;
                uint32_t enc4 = 0u;
                float S4 = 0.0f;
                if (nz.s_t != 0.0f) {
                    enc4 = nv_scale_byte<false>(amax, nz);
                    S4 = __fmul_rn(e4m3_value(enc4), nz.s_t);
                }
                nv_block_rne(x, S, amax, w6, &sse6);
                nv_block_rne(x, S4, amax, w4, &sse4);
                const bool pick4 = sse4 < sse6;
                w[0] = pick4 ? w4[0] : w6[0];
                w[1] = pick4 ? w4[1] : w6[1];
                enc = pick4 ? enc4 : enc;
            } else if (SR) {
                if (S == 0.0f) {
                    w[0] = w[1] = 0u;
                } else {
                    uint64_t pp[8], qq[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) pp[j] = f2pack(x[2 * j], x[2 * j + 1]);
                    nv_quot16_pairs(pp, S, amax, qq);
                    float q[16];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f2unpack(qq[j], q[2 * j], q[2 * j + 1]);
                    sr_group<16>(q, e0 + 16 * b, seed, w);
                }
            } else {
                nv_block_rne(x, S, amax, w, nullptr);
            }
            o.scales |= enc << (8 * b);
        }
    }
}

__device__ __forceinline__ float block_max(float m, float *red)
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

// s_t = amax_t / (6 * 448), amax_t the max of the partial maxima.
__device__ __forceinline__ float tensor_scale_from(const float *partials, int n_partials, float *red)
{
    float m = 0.0f;
    for (int i = threadIdx.x; i < n_partials; i += blockDim.x) m = fmaxf(m, partials[i]);
    m = block_max(m, red);
    return __fdiv_rn(m, 2688.0f);
}

// s_t of a quantize pass: from the caller's tensor amax when given (uniform
// over the grid), else from the partial maxima of the amax pass.
__device__ __forceinline__ float tensor_scale(const QuantParams &p, float *red)
{
    if (p.amax_in) return __fdiv_rn(*p.amax_in, 2688.0f);
    return tensor_scale_from(p.partials, p.n_partials, red);
}

template <int G>
__device__ __forceinline__ void store_unit(const UnitOut &o, const QuantParams &p, uint64_t e0, int64_t n_valid)
{
    // n_valid: elements of this unit inside the launch range (a multiple of G)
    uint8_t *cdst = p.codes + (e0 >> 1);
    uint8_t *sdst = p.scales + e0 / G;
    if (n_valid >= 64) {
        uint4 *c4 = reinterpret_cast<uint4 *>(cdst);
        c4[0] = make_uint4(o.codes[0], o.codes[1], o.codes[2], o.codes[3]);
        c4[1] = make_uint4(o.codes[4], o.codes[5], o.codes[6], o.codes[7]);
        if (G == 32) *reinterpret_cast<uint16_t *>(sdst) = static_cast<uint16_t>(o.scales);
        else *reinterpret_cast<uint32_t *>(sdst) = o.scales;
    } else {
#pragma unroll
        for (int gi = 0; gi < 64 / G; ++gi) {
            if (gi * G < n_valid) {
#pragma unroll
                for (int w = 0; w < G / 8; ++w)
                    reinterpret_cast<uint32_t *>(cdst)[gi * (G / 8) + w] = o.codes[gi * (G / 8) + w];
                sdst[gi] = static_cast<uint8_t>(o.scales >> (8 * gi));
            }
        }
    }
}

// ---------------------------------------------------------------- packed units (TMA kernel)
// A unit is UP packed binary32 pairs (pair k = elements 2k, 2k+1): UP = 64
// holds a whole 128-element rotation block, UP = 32 holds half of one and
// exchanges the h = 64 stage with its partner lane (lane ^ 1, the even lane
// holding the lower half).  Stage h = 1 runs inside each pair; stages
// h = 2 .. 2*UP between pairs k and k + h/2 as f32x2 add / sub; then, when
// NORM, one f32x2 multiply by 1/sqrt(128) (callers that fold the
// normalisation into their scale multiply pass NORM = false).
template <int UP, bool NORM>
__device__ __forceinline__ void fwht_packed(uint64_t (&p)[UP], bool upper)
{
#pragma unroll
    for (int k = 0; k < UP; ++k) {
        float a, b;
        f2unpack(p[k], a, b);
        p[k] = f2pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < UP; hp <<= 1) {
#pragma unroll
        for (int k = 0; k < UP; ++k) {
            if ((k & hp) == 0) {
                const uint64_t a = p[k], b = p[k + hp];
                p[k] = f2add(a, b);
                p[k + hp] = f2sub(a, b);
            }
        }
    }
    if (UP == 32) {
        // h = 64 across the lane pair: lower gets other + mine, upper gets
        // other - mine, both as one rounding of other + (+-1) * mine
        const float sg = upper ? -1.0f : 1.0f;
        const uint64_t sg2 = f2pack(sg, sg);
#pragma unroll
        for (int k = 0; k < UP; ++k) {
            const uint32_t lo = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(p[k]), 1);
            const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(p[k] >> 32), 1);
            p[k] = f2fma(p[k], sg2, (static_cast<uint64_t>(hi) << 32) | lo);
        }
    }
    if (NORM) {
        const uint64_t c2 = f2pack(inv_sqrt128(), inv_sqrt128());
#pragma unroll
        for (int k = 0; k < UP; ++k) p[k] = f2mul(p[k], c2);
    }
}

// in-place reduction of m[0 .. N) to m[0] with three-input maxima
// (compile-time sizes, so m stays in registers)
template <int N>
__device__ __forceinline__ void max3_reduce(float *m)
{
    if constexpr (N > 1) {
        constexpr int T = (N + 2) / 3;
#pragma unroll
        for (int j = 0; j < T; ++j) {
            const float a = m[3 * j];
            const float b = 3 * j + 1 < N ? m[3 * j + 1] : a;
            const float c = 3 * j + 2 < N ? m[3 * j + 2] : a;
            m[j] = fmax3(a, b, c);
        }
        max3_reduce<T>(m);
    }
}

// max |x| over N packed pairs
template <int N>
__device__ __forceinline__ float absmax_pairs(const uint64_t *p)
{
    float m[N];
#pragma unroll
    for (int j = 0; j < N; ++j) {
        float a, b;
        f2unpack(p[j], a, b);
        m[j] = fmaxf(fabsf(a), fabsf(b));
    }
    max3_reduce<N>(m);
    return m[0];
}

template <int UP>
struct UnitP {
    uint32_t codes[UP / 4];     // 2*UP nibbles
    uint32_t scales[2];         // up to 8 scale bytes
};

// RAW: the rotation left out its 1/sqrt(128) (fwht_packed<UP, false>); only
// the MXFP4 round-to-nearest path takes raw values.  With c = 1/sqrt(128) the
// normalised group maximum is fl(amax_raw * c) (rounding is monotone), and
// fl(x * (c * 2^-k)) equals fl(fl(x * c) * 2^-k) whenever the latter is a
// normal number; when it is subnormal both encode to a zero of x's sign.
// c * 2^-k itself is normal for k <= 120; larger k (groups near the top of
// the binary32 range) take the two multiplies.
template <int UP, int FMT, bool SR, bool FOUR6, bool RAW = false>
__device__ __forceinline__ void quant_unit_packed(uint64_t (&p)[UP], uint64_t e0, const NvScale &nz, uint64_t seed,
                                                  UnitP<UP> &o)
{
    static_assert(!RAW || (FMT == QFP4_MXFP4 && !SR && !FOUR6), "raw values only on the plain MXFP4 round-to-nearest path");
    o.scales[0] = o.scales[1] = 0u;
    if (FMT == QFP4_MXFP4) {
#pragma unroll
        for (int g = 0; g < UP / 16; ++g) {
            uint64_t *pg = p + 16 * g;
            uint32_t *w = o.codes + 4 * g;
            const float amax = RAW ? __fmul_rn(absmax_pairs<16>(pg), inv_sqrt128()) : absmax_pairs<16>(pg);
            if (amax == 0.0f) {                      // all-zero group: byte 0, +0 codes
                w[0] = w[1] = w[2] = w[3] = 0u;
                continue;
            }
            int k = mx_scale_exp(amax, nz.rule);
            if (RAW && k > 120) {
                const uint64_t c2 = f2pack(inv_sqrt128(), inv_sqrt128());
#pragma unroll
                for (int j = 0; j < 16; ++j) pg[j] = f2mul(pg[j], c2);
            }
            const float mk = (RAW && k <= 120) ? __fmul_rn(inv_sqrt128(), exp2i(-k)) : exp2i(-k);
            const uint64_t m2 = f2pack(mk, mk);      // x * 2^-k == x / 2^k exactly
            float xs[FOUR6 ? 32 : 1];                 // the group's values, for four-over-six
            if (FOUR6) {
#pragma unroll
                for (int j = 0; j < 16; ++j) f2unpack(pg[j], xs[2 * j], xs[2 * j + 1]);
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) pg[j] = f2mul(pg[j], m2);
            if (SR) {
                sr_group_pairs<32>(pg, e0 + 32 * g, seed, w);
            } else {
#pragma unroll
                for (int t = 0; t < 4; ++t) w[t] = e2m1x8_rne_pairs(pg[4 * t], pg[4 * t + 1], pg[4 * t + 2], pg[4 * t + 3]);
            }
            if (FOUR6) k = mx_four6(xs, amax, k, w);
            o.scales[0] |= static_cast<uint32_t>(k + 127) << (8 * g);
        }
    } else {
#pragma unroll
        for (int b = 0; b < UP / 8; ++b) {
            float x[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) f2unpack(p[8 * b + j], x[2 * j], x[2 * j + 1]);
            const float amax = absmax_pairs<8>(p + 8 * b);
            uint32_t *w = o.codes + 2 * b;
            uint32_t enc = 0u;
            float S = 0.0f;
            if (nz.s_t != 0.0f) {
                enc = nv_scale_byte<true>(amax, nz);
                S = __fmul_rn(e4m3_value(enc), nz.s_t);
            }
            if (FOUR6) {
                uint32_t w6[2], w4[2], enc4 = 0u;
                float sse6, sse4, S4 = 0.0f;
                if (nz.s_t != 0.0f) {
                    enc4 = nv_scale_byte<false>(amax, nz);
                    S4 = __fmul_rn(e4m3_value(enc4), nz.s_t);
                }
                nv_block_rne_pairs(p + 8 * b, S, amax, w6, &sse6);
                nv_block_rne_pairs(p + 8 * b, S4, amax, w4, &sse4);
                const bool pick4 = sse4 < sse6;
                w[0] = pick4 ? w4[0] : w6[0];
                w[1] = pick4 ? w4[1] : w6[1];
                enc = pick4 ? enc4 : enc;
            } else if (SR) {
                if (S == 0.0f) {
                    w[0] = w[1] = 0u;
                } else {
                    uint64_t qq[8];
                    nv_quot16_pairs(p + 8 * b, S, amax, qq);
                    sr_group_pairs<16>(qq, e0 + 16 * b, seed, w);
                }
            } else {
                nv_block_rne_pairs(p + 8 * b, S, amax, w, nullptr);
            }
            o.scales[b >> 2] |= enc << (8 * (b & 3));
        }
    }
}

template <int UP, int G>
__device__ __forceinline__ void store_unit_packed(const UnitP<UP> &o, const QuantParams &p, uint64_t e0,
                                                  int64_t n_valid)
{
    // n_valid: 2*UP, or 64 when the launch range ends half way through a 128-element unit
    uint4 *c4 = reinterpret_cast<uint4 *>(p.codes + (e0 >> 1));
    uint8_t *sdst = p.scales + e0 / G;
    const bool full = n_valid >= 2 * UP;
#pragma unroll
    for (int c = 0; c < UP / 16; ++c)
        if (full || c < 2) c4[c] = make_uint4(o.codes[4 * c], o.codes[4 * c + 1], o.codes[4 * c + 2], o.codes[4 * c + 3]);
    constexpr int nsb = 2 * UP / G;                   // scale bytes of a full unit: 2, 4 or 8
    const int nb = full ? nsb : 64 / G;
    if (nb == 8) *reinterpret_cast<uint2 *>(sdst) = make_uint2(o.scales[0], o.scales[1]);
    else if (nb == 4) *reinterpret_cast<uint32_t *>(sdst) = o.scales[0];
    else *reinterpret_cast<uint16_t *>(sdst) = static_cast<uint16_t>(o.scales[0]);
}

// MXFP8 of UP packed pairs (2*UP values, groups of 32): E8M0 scale with
// 448 * 2^k >= amax (least k), elements fl(v * 2^-k) to E4M3 by
// round-to-nearest-even or by the stochastic rule on the E4M3 grid (one
// Philox call per 4 elements, counter = index / 4).  An all-zero group gives
// scale byte 0 and zero codes.  2*UP code bytes in UP/2 words.
template <int UP, bool SR>
__device__ __forceinline__ void mxfp8_unit_packed(uint64_t (&p)[UP], uint64_t e0, uint64_t seed, uint32_t *codes,
                                                  uint32_t &scales)
{
    scales = 0u;
#pragma unroll
    for (int g = 0; g < UP / 16; ++g) {
        uint64_t *pg = p + 16 * g;
        uint32_t *w = codes + 8 * g;
        const float amax = absmax_pairs<16>(pg);
        if (amax == 0.0f) {
#pragma unroll
            for (int t = 0; t < 8; ++t) w[t] = 0u;
            continue;
        }
        const int k = scale_exp(amax, 0x600000u, 8);
        scales |= static_cast<uint32_t>(k + 127) << (8 * g);
        const float mk = exp2i(-k);
        const uint64_t m2 = f2pack(mk, mk);
#pragma unroll
        for (int j = 0; j < 16; ++j) pg[j] = f2mul(pg[j], m2);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float a, b, c, d;
            f2unpack(pg[2 * t], a, b);
            f2unpack(pg[2 * t + 1], c, d);
            if (SR) {
                const uint4 rw = sr_words4(seed, ((e0 + 32 * g) >> 2) + t);
                w[t] = e4m3_sr2(a, b, rw.x, rw.y) | (e4m3_sr2(c, d, rw.z, rw.w) << 16);
            } else {
                w[t] = e4m3x2_rne(a, b) | (e4m3x2_rne(c, d) << 16);
            }
        }
    }
}

// 2*UP MXFP8 code bytes and UP/16 scale bytes of a unit starting at element
// e0 (n_valid: 2*UP, or 64 when the launch range ends half way through).
template <int UP>
__device__ __forceinline__ void mxfp8_store_unit(const uint32_t *codes, uint32_t scales, const QuantParams &p,
                                                 uint64_t e0, int64_t n_valid)
{
    uint4 *c4 = reinterpret_cast<uint4 *>(p.codes + e0);
    const int nc = n_valid >= 2 * UP ? UP / 8 : 4;         // 16-byte chunks
#pragma unroll
    for (int c = 0; c < UP / 8; ++c)
        if (c < nc) c4[c] = make_uint4(codes[4 * c], codes[4 * c + 1], codes[4 * c + 2], codes[4 * c + 3]);
    uint8_t *sdst = p.scales + e0 / 32;
    if (n_valid >= 2 * UP && UP == 32) *reinterpret_cast<uint16_t *>(sdst) = static_cast<uint16_t>(scales);
    else
#pragma unroll
        for (int g = 0; g < UP / 16; ++g)
            if (32 * g < n_valid) sdst[g] = static_cast<uint8_t>(scales >> (8 * g));
}

// ---------------------------------------------------------------- TMA kernel
// WARPS warps per CTA (one CTA per SM), each with a STAGES-deep ring of tiles
// of 32 * (UP / 32) ... = UP rows of 64 bf16 (one unit of UP pairs per lane).
template <int MODE, int FMT, bool ROT, bool SR, bool FOUR6, int WARPS, int STAGES, int UP>
__global__ void __launch_bounds__(32 * WARPS, 1) k_quant1d_tma(const __grid_constant__ CUtensorMap tm, QuantParams p)
{
    constexpr int ROWS_PER_LANE = UP / 32;             // 64-element rows per unit
    constexpr int TILE_ROWS = 32 * ROWS_PER_LANE;
    constexpr int STAGE_BYTES = TILE_ROWS * 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[WARPS][STAGES];
    __shared__ float red[32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = p.n / 64;
    const int64_t ntiles = (rows + TILE_ROWS - 1) / TILE_ROWS;
    // contiguous tile range of this CTA, balanced to one tile
    const int64_t t_begin = ntiles * blockIdx.x / gridDim.x, t_end = ntiles * (blockIdx.x + 1) / gridDim.x;
    constexpr int G = FMT == QFP4_NVFP4 ? 16 : 32;

    uint64_t *bars = full[warp];
    uint8_t *ring = smem + warp * (STAGES * STAGE_BYTES);
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        if (warp == 0) prefetch_tensormap(&tm);
    }
    __syncwarp();
    pdl_wait();
    pdl_trigger();
    float s_t = 0.0f;
    if (MODE == MODE_QUANT && FMT == QFP4_NVFP4) {
        s_t = tensor_scale(p, red);
        if (p.write_tscale && blockIdx.x == 0 && threadIdx.x == 0) *p.tscale_out = s_t;
    }
    const NvScale nz = nv_scale_setup(s_t, p.rule);
    // a quantize pass under a caller-supplied amax can still report this
    // tensor's own amax: partial maxima of the (rotated) values it reads
    const bool own_max = MODE == MODE_AMAX || p.partials_out != nullptr;

    auto issue = [&](int64_t t, int s) {
        mbar_arrive_expect_tx(&bars[s], STAGE_BYTES);
        tma_load_2d(ring + s * STAGE_BYTES, &tm, &bars[s], 0, static_cast<int>(t * TILE_ROWS));
    };
    if (lane == 0)
        for (int s = 0; s < STAGES; ++s) {
            const int64_t t = t_begin + warp + static_cast<int64_t>(s) * WARPS;
            if (t < t_end) issue(t, s);
        }

    float tmax = 0.0f;
    int it = 0;
    bool gave_up = false;
    for (int64_t t = t_begin + warp; t < t_end; t += WARPS, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        const bool ok = mbar_wait(&bars[s], ph);
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            gave_up = true;
            break;
        }

        // this lane's unit: rows ROWS_PER_LANE*lane + h of the tile (128-byte swizzle)
        const uint8_t *st = ring + s * STAGE_BYTES;
        uint64_t v[UP];
#pragma unroll
        for (int h = 0; h < ROWS_PER_LANE; ++h) {
            const int r = ROWS_PER_LANE * lane + h;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w = *reinterpret_cast<const uint4 *>(st + r * 128 + ((c ^ (r & 7)) << 4));
                v[32 * h + 4 * c + 0] = bf16x2_to_f2(w.x);
                v[32 * h + 4 * c + 1] = bf16x2_to_f2(w.y);
                v[32 * h + 4 * c + 2] = bf16x2_to_f2(w.z);
                v[32 * h + 4 * c + 3] = bf16x2_to_f2(w.w);
            }
        }
        // The refill below is an async-proxy write to the stage these
        // generic-proxy reads come from: without the proxy fence in every
        // lane the two are unordered, and late reads (the last row chunks,
        // which a short computation needs last) could see the next tile.
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
            const int64_t tn = t + static_cast<int64_t>(STAGES) * WARPS;
            if (tn < t_end) issue(tn, s);
        }

        const int64_t row0 = t * TILE_ROWS + ROWS_PER_LANE * lane;   // first 64-element row of the unit
        const int64_t n_valid = imin<int64_t>(2 * UP, (rows - row0) * 64);
        constexpr bool RAW = ROT && MODE == MODE_QUANT && FMT == QFP4_MXFP4 && !SR && !FOUR6;
        if (ROT) fwht_packed<UP, !RAW>(v, (lane & 1) != 0);
        if (MODE == MODE_AMAX || (FMT == QFP4_NVFP4 && own_max))
            tmax = fmaxf(tmax, absmax_pairs<UP>(v));   // rows past the end were zero-filled by TMA
        if (MODE == MODE_QUANT && n_valid > 0) {
            const uint64_t e0 = p.e_base + static_cast<uint64_t>(row0) * 64u;
            if constexpr (FMT == FMT_MXFP8) {
                uint32_t cw[UP / 2], sc;
                mxfp8_unit_packed<UP, SR>(v, e0, p.seed, cw, sc);
                mxfp8_store_unit<UP>(cw, sc, p, e0, n_valid);
            } else {
                UnitP<UP> o;
                quant_unit_packed<UP, FMT, SR, FOUR6, RAW>(v, e0, nz, p.seed, o);
                store_unit_packed<UP, G>(o, p, e0, n_valid);
            }
        }
    }
    if (gave_up && lane == 0) settle_ns(kSettleNs);   // loads of this warp's ring may still be landing
    if (MODE == MODE_AMAX || (FMT == QFP4_NVFP4 && own_max)) {
        tmax = block_max(tmax, red);
        if (threadIdx.x == 0) p.partials_out[blockIdx.x] = tmax;
    }
}

// Production configuration of the TMA kernel.
// 20 warps (<= 96 registers a thread) except four-over-six, which needs the
// registers of 16 warps
__host__ __device__ constexpr int qt_warps(bool four6) { return four6 ? 16 : 20; }
constexpr int QT_STAGES = 2, QT_UP = 32;
constexpr int QT_TILE_ROWS = QT_UP;
__host__ __device__ constexpr int qt_smem_bytes(bool four6) { return qt_warps(four6) * QT_STAGES * QT_UP * 128 + 1024; }

// ---------------------------------------------------------------- direct kernel
// Loads straight from global memory (bf16 or binary32), one unit per thread;
// serves binary32 inputs and the ragged tail (n % 64) of bf16 inputs.
template <int MODE, int FMT, bool ROT, bool SR, bool FOUR6, typename T>
__global__ void __launch_bounds__(128) k_quant1d_direct(const T *__restrict__ x, QuantParams p)
{
    __shared__ float red[32];
    pdl_wait();
    pdl_trigger();
    constexpr int G = FMT == QFP4_MXFP4 ? 32 : 16;
    float s_t = 0.0f;
    if (MODE == MODE_QUANT && FMT == QFP4_NVFP4) {
        s_t = tensor_scale(p, red);
        if (p.write_tscale && blockIdx.x == 0 && threadIdx.x == 0) *p.tscale_out = s_t;
    }
    const NvScale nz = nv_scale_setup(s_t, p.rule);
    const bool own_max = MODE == MODE_AMAX || p.partials_out != nullptr;
    const int64_t units = (p.n + 63) / 64;
    float tmax = 0.0f;
    for (int64_t u0 = static_cast<int64_t>(blockIdx.x) * blockDim.x; u0 < units;
         u0 += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t u = u0 + threadIdx.x;
        const int64_t off = u * 64;
        const int64_t n_valid = u < units ? imin<int64_t>(64, p.n - off) : 0;
        float v[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) v[i] = 0.0f;
        if (n_valid > 0) {
            // whole 16-byte vectors where they lie inside the range, single
            // elements for a last partial vector (the amax pass of an
            // arbitrary-length input reaches one; the quantize passes, whose
            // lengths are multiples of the group, do not)
            if (sizeof(T) == 4) {
                const float4 *src = reinterpret_cast<const float4 *>(x + off);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    if (4 * c + 4 <= n_valid) {
                        const float4 f = src[c];
                        v[4 * c] = f.x;
                        v[4 * c + 1] = f.y;
                        v[4 * c + 2] = f.z;
                        v[4 * c + 3] = f.w;
                    } else if (4 * c < n_valid) {
                        for (int t = 0; t < 4; ++t)
                            if (4 * c + t < n_valid) v[4 * c + t] = reinterpret_cast<const float *>(x + off)[4 * c + t];
                    }
                }
            } else {
                const uint4 *src = reinterpret_cast<const uint4 *>(x + off);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (8 * c + 8 <= n_valid) {
                        const uint4 w = src[c];
                        v[8 * c] = bf16lo(w.x);
                        v[8 * c + 1] = bf16hi(w.x);
                        v[8 * c + 2] = bf16lo(w.y);
                        v[8 * c + 3] = bf16hi(w.y);
                        v[8 * c + 4] = bf16lo(w.z);
                        v[8 * c + 5] = bf16hi(w.z);
                        v[8 * c + 6] = bf16lo(w.w);
                        v[8 * c + 7] = bf16hi(w.w);
                    } else if (8 * c < n_valid) {
                        const uint16_t *h = reinterpret_cast<const uint16_t *>(x + off);
                        for (int t = 0; t < 8; ++t)
                            if (8 * c + t < n_valid)
                                v[8 * c + t] = __uint_as_float(static_cast<uint32_t>(h[8 * c + t]) << 16);
                    }
                }
            }
        }
        if (ROT) fwht128_pair(v, (threadIdx.x & 1) != 0);   // n % 128 == 0: pairs are whole
        if (MODE == MODE_AMAX || (FMT == QFP4_NVFP4 && own_max)) {
#pragma unroll
            for (int i = 0; i < 64; ++i) tmax = fmaxf(tmax, fabsf(v[i]));
        }
        if (MODE == MODE_QUANT && n_valid > 0) {
            const uint64_t e0 = p.e_base + static_cast<uint64_t>(off);
            UnitOut o;
            quant_unit<FMT, SR, FOUR6>(v, e0, nz, p.seed, o);
            store_unit<G>(o, p, e0, n_valid);
        }
    }
    if (MODE == MODE_AMAX || (FMT == QFP4_NVFP4 && own_max)) {
        tmax = block_max(tmax, red);
        if (threadIdx.x == 0) p.partials_out[blockIdx.x] = tmax;
    }
}

// ---------------------------------------------------------------- host launchers
template <int MODE, int FMT, bool ROT, bool SR, bool FOUR6>
static int launch_tma(const CUtensorMap &tm, const QuantParams &p, int grid, cudaStream_t stream)
{
    constexpr int W = qt_warps(FOUR6), SMEM = qt_smem_bytes(FOUR6);
    auto kern = k_quant1d_tma<MODE, FMT, ROT, SR, FOUR6, W, QT_STAGES, QT_UP>;
    if (ensure_dyn_smem<k_quant1d_tma<MODE, FMT, ROT, SR, FOUR6, W, QT_STAGES, QT_UP>>(SMEM) != QFP4_OK)
        return QFP4_ERR_CUDA;
    if (launch_pdl(kern, dim3(grid), dim3(32 * W), SMEM, stream, tm, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

template <int MODE, int FMT, bool ROT, bool SR, bool FOUR6, typename T>
static int launch_direct(const T *x, const QuantParams &p, int grid, cudaStream_t stream)
{
    if (launch_pdl(k_quant1d_direct<MODE, FMT, ROT, SR, FOUR6, T>, dim3(grid), dim3(128), 0, stream, x, p) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

// One pass (amax or quantize) over x[0, n): the bf16 64-aligned body through
// the TMA kernel, the rest through the direct kernel.  Partial maxima are
// written to partials_out[0 ..) (amax pass); returns the number written.
template <int MODE, int FMT, bool ROT, bool SR, bool FOUR6>
static int run_pass(const void *x, qfp4_dtype xdt, int64_t n, QuantParams p, cudaStream_t stream, int *n_parts)
{
    const int nsm = num_sms();
    int parts = 0;
    int64_t body = 0;
    const bool was_write = p.write_tscale;
    if (xdt == QFP4_BF16) {
        body = (n / 64) * 64;
        if (body > 0) {
            CUtensorMap tm;
            const uint64_t dims[2] = {64, static_cast<uint64_t>(body / 64)};
            const uint64_t strides[1] = {128};
            const uint32_t box[2] = {64, QT_TILE_ROWS};
            int st = encode_tensor_map(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides,
                                       box, CU_TENSOR_MAP_SWIZZLE_128B);
            if (st != QFP4_OK) return st;
            const int64_t ntiles = (body / 64 + QT_TILE_ROWS - 1) / QT_TILE_ROWS;
            const int grid = static_cast<int>(imin<int64_t>((ntiles + qt_warps(FOUR6) - 1) / qt_warps(FOUR6), nsm));
            QuantParams q = p;
            q.n = body;
            q.partials_out = p.partials_out;
            st = launch_tma<MODE, FMT, ROT, SR, FOUR6>(tm, q, grid, stream);
            if (st != QFP4_OK) return st;
            parts += grid;
            p.write_tscale = false;
        }
    }
    const int64_t rest = n - body;
    if (rest > 0) {
        QuantParams q = p;
        q.n = rest;
        q.e_base = p.e_base + body;
        q.write_tscale = body > 0 ? false : was_write;
        q.partials_out = p.partials_out ? p.partials_out + parts : nullptr;
        const int64_t units = (rest + 63) / 64;
        const int grid = static_cast<int>(imin<int64_t>((units + 127) / 128, 4 * nsm));
        int st;
        if (xdt == QFP4_BF16)
            st = launch_direct<MODE, FMT, ROT, SR, FOUR6>(static_cast<const uint16_t *>(x) + body, q, grid, stream);
        else
            st = launch_direct<MODE, FMT, ROT, SR, FOUR6>(static_cast<const float *>(x), q, grid, stream);
        if (st != QFP4_OK) return st;
        parts += grid;
    }
    if (n_parts) *n_parts = parts;
    return QFP4_OK;
}

// MXFP8 row-wise codes and E8M0 scales of x[0, n) (bf16, n % 64 == 0) through
// the TMA kernel.
int mxfp8_rows(const void *x, int64_t n, bool sr, uint64_t seed, uint8_t *codes, uint8_t *scales, cudaStream_t stream)
{
    if (n <= 0) return QFP4_OK;
    CUtensorMap tm;
    const uint64_t dims[2] = {64, static_cast<uint64_t>(n / 64)};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, QT_TILE_ROWS};
    int st = encode_tensor_map(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != QFP4_OK) return st;
    QuantParams q{};
    q.n = n;
    q.e_base = 0;
    q.codes = codes;
    q.scales = scales;
    q.seed = seed;
    const int64_t ntiles = (n / 64 + QT_TILE_ROWS - 1) / QT_TILE_ROWS;
    const int grid = static_cast<int>(imin<int64_t>((ntiles + qt_warps(false) - 1) / qt_warps(false), num_sms()));
    return sr ? launch_tma<MODE_QUANT, FMT_MXFP8, false, true, false>(tm, q, grid, stream)
              : launch_tma<MODE_QUANT, FMT_MXFP8, false, false, false>(tm, q, grid, stream);
}

// Partial maxima of |x| over a flat range (the NVFP4 tensor-amax pass, no rotation).
int amax_partials(const void *x, qfp4_dtype xdt, int64_t n, float *partials, int *n_parts, cudaStream_t stream)
{
    QuantParams p{};
    p.n = n;
    p.partials_out = partials;
    return run_pass<MODE_AMAX, QFP4_NVFP4, false, false, false>(x, xdt, n, p, stream, n_parts);
}

// amax_out = max of n partial maxima (one block)
__global__ void __launch_bounds__(256) k_partials_max(const float *partials, int n, float *amax_out)
{
    __shared__ float red[32];
    pdl_wait();
    pdl_trigger();
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partials[i]);
    m = block_max(m, red);
    if (threadIdx.x == 0) *amax_out = m;
}

int partials_max(const float *partials, int n, float *amax_out, cudaStream_t stream)
{
    if (launch_pdl(k_partials_max, dim3(1), dim3(256), 0, stream, partials, n, amax_out) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

__global__ void k_tscale_from_amax(const float *amax_in, float *tscale)
{
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) *tscale = __fdiv_rn(*amax_in, 2688.0f);
}

int tscale_from_amax(const float *amax_in, float *tscale, cudaStream_t stream)
{
    if (launch_pdl(k_tscale_from_amax, dim3(1), dim3(32), 0, stream, amax_in, tscale) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

// NVFP4: with no caller amax, an amax pass (partial maxima into `partials`)
// then the quantize pass; with a caller amax, the quantize pass alone, which
// also writes its own partial maxima when the tensor's amax is asked for.
template <int FMT, bool ROT, bool SR, bool FOUR6>
static int quantize1d_t(const void *x, qfp4_dtype xdt, int64_t n, uint64_t seed, uint8_t *codes, uint8_t *scales,
                        float *tscale, float *partials, int *n_parts_out, const QuantOpts &opt,
                        cudaStream_t stream)
{
    QuantParams p{};
    p.n = n;
    p.e_base = 0;
    p.codes = codes;
    p.scales = scales;
    p.seed = seed;
    p.tscale_out = tscale;
    p.write_tscale = true;
    p.rule = opt.rule;
    int n_parts = 0;
    if (FMT == QFP4_NVFP4 && !opt.amax_in) {
        p.partials_out = partials;
        int st = run_pass<MODE_AMAX, FMT, ROT, false, false>(x, xdt, n, p, stream, &n_parts);
        if (st != QFP4_OK) return st;
        p.partials_out = nullptr;
        p.partials = partials;
        p.n_partials = n_parts;
    }
    if (FMT == QFP4_NVFP4 && opt.amax_in) {
        p.amax_in = opt.amax_in;
        p.partials_out = opt.amax_out ? partials : nullptr;
    }
    int quant_parts = 0;
    int st = run_pass<MODE_QUANT, FMT, ROT, SR, FOUR6>(x, xdt, n, p, stream, &quant_parts);
    if (st != QFP4_OK) return st;
    if (opt.amax_in && opt.amax_out) n_parts = quant_parts;
    if (n_parts_out) *n_parts_out = n_parts;
    if (FMT == QFP4_NVFP4 && opt.amax_out) return partials_max(partials, n_parts, opt.amax_out, stream);
    return QFP4_OK;
}

int quantize1d(const void *x, qfp4_dtype xdt, int64_t n, qfp4_fmt fmt, qfp4_round rounding, int rotate, int four6,
               uint64_t seed, uint8_t *codes, uint8_t *scales, float *tscale, float *partials, int *n_parts_out,
               cudaStream_t stream, const QuantOpts &opt)
{
    const bool sr = rounding == QFP4_SR;
#define QFP4_Q1(F, R, S, F6) \
    quantize1d_t<F, R, S, F6>(x, xdt, n, seed, codes, scales, tscale, partials, n_parts_out, opt, stream)
    if (fmt == QFP4_MXFP4) {
        if (four6) return rotate ? QFP4_Q1(QFP4_MXFP4, true, false, true) : QFP4_Q1(QFP4_MXFP4, false, false, true);
        if (rotate) return sr ? QFP4_Q1(QFP4_MXFP4, true, true, false) : QFP4_Q1(QFP4_MXFP4, true, false, false);
        return sr ? QFP4_Q1(QFP4_MXFP4, false, true, false) : QFP4_Q1(QFP4_MXFP4, false, false, false);
    }
    if (four6) return rotate ? QFP4_Q1(QFP4_NVFP4, true, false, true) : QFP4_Q1(QFP4_NVFP4, false, false, true);
    if (rotate) return sr ? QFP4_Q1(QFP4_NVFP4, true, true, false) : QFP4_Q1(QFP4_NVFP4, true, false, false);
    return sr ? QFP4_Q1(QFP4_NVFP4, false, true, false) : QFP4_Q1(QFP4_NVFP4, false, false, false);
#undef QFP4_Q1
}

}  // namespace qfp4
