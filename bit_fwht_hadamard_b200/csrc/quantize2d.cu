// quantize2d.cu -- 2D transposition-invariant NVFP4 blocks (X and X^T from
// one pass), the 1D column-wise quantization of X^T, and the MXFP8 (E4M3)
// variant with its column-wise output.
//
// Method: [TI] (2D blocks give X and X^T one shared scale set; stochastic
// rounding; MXFP8 for the sensitive projections), [46] (four-over-six on the
// column groups of the 1D baseline), [LB] §2-§3 (group scales, E8M0).
//
// 2D kernel (`k_quant2d`): a warp task is 64 rows x 32 columns, four 16-row
// bands of two adjacent 16x16 tiles; lane (h, r) loads row r of tile h in
// each band (16 bf16 = 32 B, so every 32-byte sector a warp touches is fully
// used).  The tile amax is a 16-lane shuffle reduction; each lane quantizes
// its row (RNE or Philox SR keyed on X's element index) and stores its 8
// code bytes; then a 4-stage nibble transpose across the 16 lanes (byte
// permutes, one shuffle a stage) gives each lane one column of the tile --
// the codes of X^T, bit-identical by construction because every element was
// rounded once -- and the four bands make 32 contiguous bytes of an X^T row.
// `k_quant2d_mx` is the MXFP4 form on 32x32 tiles (a scale-rule variant).
//
// Column-wise outputs (1D X^T baseline, MXFP8 columns) from bf16 input:
// round to nearest in `k_cols4` (32 rows x 128 columns a warp, 4 adjacent
// columns a lane, 256-byte row loads per warp instruction), stochastic
// rounding in `k_cols_sr` (32 rows x 64 columns a warp, a lane pair sharing
// 4 columns and each Philox call); binary32 inputs use `k_quant_cols` /
// `k_mxfp8` on 32 x 32 tiles with one column a lane.  Either way a column
// group of 32 (or two of 16) sits in one lane's registers.  The row-wise
// MXFP8 output of a bf16 input comes from the TMA kernel of the 1D quantize
// (`k_mxfp8` takes both outputs when M * K is not a multiple of 64).
#include "qfp4_common.cuh"
#include "quantize1d.cuh"

namespace qfp4 {

struct Q2DParams {
    int64_t M, K;
    uint8_t *codes, *scales, *codesT, *scalesT;
    const float *partials;       // NVFP4: partial maxima of the amax pass
    int n_partials;
    float *tscale_out;
    uint64_t seed;
    int rule;                    // qfp4_scale_rule
    const float *amax_in;        // NVFP4: caller-supplied tensor amax (device), or NULL
};

// NVFP4 tensor scale s_t = amax_t / (6 * 448): amax_t from the caller or
// from the partial maxima of the amax pass (uniform over the block).
__device__ __forceinline__ float q2d_tensor_scale(const Q2DParams &p, float *red)
{
    if (p.amax_in) return __fdiv_rn(*p.amax_in, 2688.0f);
    return tensor_scale_from(p.partials, p.n_partials, red);
}

// 16 consecutive elements as raw words (bf16: 32 bytes, binary32: 64 bytes),
// so that the next task's loads can be in flight during this task's work.
template <typename T>
struct Raw16 {
    uint4 w[sizeof(T) == 4 ? 4 : 2];
};

template <typename T>
__device__ __forceinline__ void raw_load16(const T *x, int64_t off, bool valid, Raw16<T> &r)
{
    if (valid) {
        const uint4 *s = reinterpret_cast<const uint4 *>(x + off);
#pragma unroll
        for (int c = 0; c < (sizeof(T) == 4 ? 4 : 2); ++c) r.w[c] = s[c];
    } else {
#pragma unroll
        for (int c = 0; c < (sizeof(T) == 4 ? 4 : 2); ++c) r.w[c] = make_uint4(0u, 0u, 0u, 0u);
    }
}

template <typename T>
__device__ __forceinline__ void raw_to_f32(const Raw16<T> &r, float *v)
{
#pragma unroll
    for (int c = 0; c < (sizeof(T) == 4 ? 4 : 2); ++c) {
        const uint4 w = r.w[c];
        if (sizeof(T) == 4) {
            v[4 * c] = __uint_as_float(w.x);
            v[4 * c + 1] = __uint_as_float(w.y);
            v[4 * c + 2] = __uint_as_float(w.z);
            v[4 * c + 3] = __uint_as_float(w.w);
        } else {
            v[8 * c] = bf16lo(w.x);
            v[8 * c + 1] = bf16hi(w.x);
            v[8 * c + 2] = bf16lo(w.y);
            v[8 * c + 3] = bf16hi(w.y);
            v[8 * c + 4] = bf16lo(w.z);
            v[8 * c + 5] = bf16hi(w.z);
            v[8 * c + 6] = bf16lo(w.w);
            v[8 * c + 7] = bf16hi(w.w);
        }
    }
}

template <typename T>
__device__ __forceinline__ float ld1(const T *x, int64_t i)
{
    if (sizeof(T) == 4) return reinterpret_cast<const float *>(x)[i];
    return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t *>(x)[i]) << 16);
}

// Transpose a 16 x 16 nibble matrix held as one row per lane of a 16-lane
// group (lo = nibbles 0-7, hi = nibbles 8-15; nibble j of lane r = element
// (r, j)); afterwards nibble j of lane r is element (j, r).  Four block-swap
// stages with the partner lane r ^ s: for s = 8 the swapped halves are whole
// words, for s = 4 and 2 byte pairs and bytes (one byte permute packs what a
// lane sends, two put what it receives in place), for s = 1 the odd or even
// nibbles of every byte.  One shuffle a stage; shuffle partners stay inside
// the group.
__device__ __forceinline__ void transpose16x16_nibbles(uint32_t &lo, uint32_t &hi, int r)
{
    {   // s = 8: the lower lane's hi <-> the upper lane's lo
        const bool up = (r & 8) != 0;
        const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, up ? lo : hi, 8);
        if (up) lo = got;
        else hi = got;
    }
    {   // s = 4: bytes 2-3 of each word (lower lane) <-> bytes 0-1 (upper lane)
        const bool up = (r & 4) != 0;
        const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, __byte_perm(lo, hi, up ? 0x5410u : 0x7632u), 4);
        lo = __byte_perm(lo, got, up ? 0x3254u : 0x5410u);
        hi = __byte_perm(hi, got, up ? 0x3276u : 0x7610u);
    }
    {   // s = 2: bytes 1 and 3 (lower lane) <-> bytes 0 and 2 (upper lane)
        const bool up = (r & 2) != 0;
        const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, __byte_perm(lo, hi, up ? 0x6420u : 0x7531u), 2);
        lo = __byte_perm(lo, got, up ? 0x3514u : 0x5240u);
        hi = __byte_perm(hi, got, up ? 0x3716u : 0x7260u);
    }
    {   // s = 1: odd nibbles (lower lane) <-> even nibbles (upper lane); the
        // sent word holds lo's share in its low nibbles and hi's in its high ones
        const bool up = (r & 1) != 0;
        const uint32_t M = 0x0F0F0F0Fu, km = up ? ~M : M;
        const uint32_t send = ((lo >> (up ? 0 : 4)) & M) | ((hi << (up ? 4 : 0)) & ~M);
        const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
        lo = (lo & km) | ((got << (up ? 0 : 4)) & ~km);
        hi = (hi & km) | ((got >> (up ? 4 : 0)) & ~km);
    }
}

// ---------------------------------------------------------------- 2D NVFP4
// A warp task is 64 rows x 32 columns: four 16-row bands of two 16 x 16
// tiles.  Lane (h, r) = (lane / 16, lane % 16) holds row r of tile (b, h) for
// each band b (16 values; 32 contiguous bytes of bf16).  After rounding, the
// nibble transpose of each band gives lane (h, r) column r of tile (b, h):
// 16 consecutive elements of X^T row j = 16 tc + r, so the four bands are 32
// contiguous bytes of that row (one full sector, two 16-byte stores) and its
// four scale bytes are contiguous in scalesT (one 4-byte store).  The four
// bands' shuffles are independent, which hides their latency.
template <bool SR, typename T>
__global__ void __launch_bounds__(256) k_quant2d(const T *__restrict__ x, Q2DParams p)
{
    __shared__ float red[32];
    const float s_t = q2d_tensor_scale(p, red);
    if (p.tscale_out && blockIdx.x == 0 && threadIdx.x == 0) *p.tscale_out = s_t;
    const NvScale nz = nv_scale_setup(s_t, p.rule);

    const int lane = threadIdx.x & 31, half = lane >> 4, r = lane & 15;
    const int64_t tiles_k = p.K / 16, bands = p.M / 16;
    const int64_t pairs = (tiles_k + 1) / 2, quads = (bands + 3) / 4;
    const int64_t tasks = quads * pairs;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    // task -> (band quad, tile column); tasks < 2^31 (checked on the host),
    // so the division runs in 32 bits
    auto task_pos = [&](int64_t task, int64_t &bq, int64_t &tc) {
        const uint32_t t32 = static_cast<uint32_t>(task), bq32 = t32 / static_cast<uint32_t>(pairs);
        bq = bq32;
        tc = static_cast<int64_t>(t32 - bq32 * static_cast<uint32_t>(pairs)) * 2 + half;
    };
    auto load_task = [&](int64_t task, Raw16<T> (&rw)[4]) {
        int64_t bq, tc;
        task_pos(task, bq, tc);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t band = bq * 4 + b;
            raw_load16(x, (band * 16 + r) * p.K + tc * 16, tc < tiles_k && band < bands, rw[b]);
        }
    };
    for (int64_t task = warp0; task < tasks; task += nwarps) {
        int64_t bq, tc;
        task_pos(task, bq, tc);
        const bool colv = tc < tiles_k;
        const int64_t j0 = tc * 16;
        Raw16<T> raw[4];
        bool bv[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) bv[b] = bq * 4 + b < bands;
        load_task(task, raw);
        uint32_t w[4][2], enc[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float v[16];
            raw_to_f32(raw[b], v);
            float amax = 0.0f;
#pragma unroll
            for (int t = 0; t < 16; ++t) amax = fmaxf(amax, fabsf(v[t]));
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            enc[b] = 0u;
            float S = 0.0f;
            if (s_t != 0.0f) {
                enc[b] = nv_scale_byte<true>(amax, nz);
                S = __fmul_rn(e4m3_value(enc[b]), s_t);
            }
            w[b][0] = w[b][1] = 0u;
            if (S != 0.0f) {
                if (SR) {
                    uint64_t pp[8], qq[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) pp[t] = f2pack(v[2 * t], v[2 * t + 1]);
                    nv_quot16_pairs(pp, S, amax, qq);
                    const int64_t i = (bq * 4 + b) * 16 + r;
                    sr_group_pairs<16>(qq, static_cast<uint64_t>(i * p.K + j0), p.seed, w[b]);
                } else {
                    nv_block_rne(v, S, amax, w[b], nullptr);
                }
            }
        }
        // row-wise outputs: 8 code bytes and one scale byte per band
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (colv && bv[b]) {
                const int64_t i = (bq * 4 + b) * 16 + r;
                *reinterpret_cast<uint2 *>(p.codes + (i * p.K + j0) / 2) = make_uint2(w[b][0], w[b][1]);
                p.scales[i * tiles_k + tc] = static_cast<uint8_t>(enc[b]);
            }
        }
        if (p.codesT) {
            uint64_t tw[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                uint32_t lo = w[b][0], hi = w[b][1];
                transpose16x16_nibbles(lo, hi, r);
                tw[b] = (static_cast<uint64_t>(hi) << 32) | lo;
            }
            if (colv) {
                const int64_t jr = j0 + r;                       // column of X = row of X^T
                const int64_t base = jr * p.M + bq * 64;         // X^T element index of band 0
                const bool full = bv[3];                         // all four bands inside M
                if (full && (p.M % 32) == 0) {                   // 32 contiguous bytes, 16-byte aligned
                    uint4 *dst = reinterpret_cast<uint4 *>(p.codesT + base / 2);
                    dst[0] = make_uint4(static_cast<uint32_t>(tw[0]), static_cast<uint32_t>(tw[0] >> 32),
                                        static_cast<uint32_t>(tw[1]), static_cast<uint32_t>(tw[1] >> 32));
                    dst[1] = make_uint4(static_cast<uint32_t>(tw[2]), static_cast<uint32_t>(tw[2] >> 32),
                                        static_cast<uint32_t>(tw[3]), static_cast<uint32_t>(tw[3] >> 32));
                } else {
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (bv[b])
                            *reinterpret_cast<uint2 *>(p.codesT + (base + 16 * b) / 2) =
                                make_uint2(static_cast<uint32_t>(tw[b]), static_cast<uint32_t>(tw[b] >> 32));
                }
                uint8_t *sdst = p.scalesT + jr * bands + bq * 4;
                if (full && (bands % 4) == 0) {
                    *reinterpret_cast<uint32_t *>(sdst) = enc[0] | (enc[1] << 8) | (enc[2] << 16) | (enc[3] << 24);
                } else {
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (bv[b]) sdst[b] = static_cast<uint8_t>(enc[b]);
                }
            }
        }
    }
}

// Transpose a 32 x 32 nibble matrix held as one 128-bit row per lane (4
// words, nibble j of lane r = element (r, j) in word j / 8); afterwards
// nibble j of lane r is element (j, r).  Block swaps of 16 and 8 nibbles move
// whole words; those of 4, 2 and 1 nibbles are the 16 x 16 transpose's
// stages on each pair of words.
__device__ __forceinline__ void transpose32x32_nibbles(uint32_t (&w)[4], int r)
{
    {   // 16: words {0,1} of the upper lane <-> words {2,3} of the lower lane
        const bool up = (r & 16) != 0;
        const uint32_t a = __shfl_xor_sync(0xFFFFFFFFu, up ? w[0] : w[2], 16);
        const uint32_t b = __shfl_xor_sync(0xFFFFFFFFu, up ? w[1] : w[3], 16);
        if (up) { w[0] = a; w[1] = b; } else { w[2] = a; w[3] = b; }
    }
    {   // 8: word 1 / 3 of the lower lane <-> word 0 / 2 of the upper lane
        const bool up = (r & 8) != 0;
        const uint32_t a = __shfl_xor_sync(0xFFFFFFFFu, up ? w[0] : w[1], 8);
        const uint32_t b = __shfl_xor_sync(0xFFFFFFFFu, up ? w[2] : w[3], 8);
        if (up) { w[0] = a; w[2] = b; } else { w[1] = a; w[3] = b; }
    }
    // 4, 2, 1: the byte-permute stages of the 16 x 16 transpose on the word
    // pairs (0, 1) and (2, 3): one shuffle a pair and stage
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
        {
            const bool up = (r & 4) != 0;
            const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, __byte_perm(w[k], w[k + 1], up ? 0x5410u : 0x7632u), 4);
            w[k] = __byte_perm(w[k], got, up ? 0x3254u : 0x5410u);
            w[k + 1] = __byte_perm(w[k + 1], got, up ? 0x3276u : 0x7610u);
        }
        {
            const bool up = (r & 2) != 0;
            const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, __byte_perm(w[k], w[k + 1], up ? 0x6420u : 0x7531u), 2);
            w[k] = __byte_perm(w[k], got, up ? 0x3514u : 0x5240u);
            w[k + 1] = __byte_perm(w[k + 1], got, up ? 0x3716u : 0x7260u);
        }
        {
            const bool up = (r & 1) != 0;
            const uint32_t M = 0x0F0F0F0Fu, km = up ? ~M : M;
            const uint32_t send = ((w[k] >> (up ? 0 : 4)) & M) | ((w[k + 1] << (up ? 4 : 0)) & ~M);
            const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
            w[k] = (w[k] & km) | ((got << (up ? 0 : 4)) & ~km);
            w[k + 1] = (w[k + 1] & km) | ((got >> (up ? 4 : 0)) & ~km);
        }
    }
}

// ---------------------------------------------------------------- 2D MXFP4 (32 x 32 tiles)
// A warp takes one 32 x 32 tile: lane r loads row r (32 elements), the tile
// amax is a 32-lane reduction, the E8M0 exponent follows the scale rule, each
// lane rounds its row once (RNE or Philox SR keyed on X's index) and stores
// its 16 code bytes; the nibble transpose then gives each lane one column of
// the tile, the codes of X^T.
template <bool SR, typename T>
__global__ void __launch_bounds__(256) k_quant2d_mx(const T *__restrict__ x, Q2DParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t tiles_k = p.K / 32, tasks = (p.M / 32) * tiles_k;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t task = warp0; task < tasks; task += nwarps) {
        const int64_t bi = (task / tiles_k) * 32, bj = (task % tiles_k) * 32;
        const int64_t i = bi + lane;
        float v[32];
        Raw16<T> r0, r1;
        raw_load16(x, i * p.K + bj, true, r0);
        raw_load16(x, i * p.K + bj + 16, true, r1);
        raw_to_f32(r0, v);
        raw_to_f32(r1, v + 16);
        float amax = 0.0f;
#pragma unroll
        for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(v[t]));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        uint32_t w[4] = {0u, 0u, 0u, 0u}, sbyte = 0u;
        if (amax != 0.0f) {
            const int k = mx_scale_exp(amax, p.rule);
            sbyte = static_cast<uint32_t>(k + 127);
            const float mul = exp2i(-k);
            float q[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) q[t] = __fmul_rn(v[t], mul);
            if (SR) {
                uint64_t qp[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) qp[t] = f2pack(q[2 * t], q[2 * t + 1]);
                sr_group_pairs<32>(qp, static_cast<uint64_t>(i * p.K + bj), p.seed, w);
            } else {
#pragma unroll
                for (int t = 0; t < 4; ++t) w[t] = e2m1x8_rne(q + 8 * t);
            }
        }
        *reinterpret_cast<uint4 *>(p.codes + (i * p.K + bj) / 2) = make_uint4(w[0], w[1], w[2], w[3]);
        p.scales[i * tiles_k + bj / 32] = static_cast<uint8_t>(sbyte);
        if (p.codesT) {
            transpose32x32_nibbles(w, lane);
            const int64_t jr = bj + lane;                     // column of X = row of X^T
            *reinterpret_cast<uint4 *>(p.codesT + (jr * p.M + bi) / 2) = make_uint4(w[0], w[1], w[2], w[3]);
            p.scalesT[jr * (p.M / 32) + bi / 32] = static_cast<uint8_t>(sbyte);
        }
    }
}

// ---------------------------------------------------------------- 1D column-wise (X^T baseline)
template <int FMT, bool SR, bool FOUR6, typename T>
__global__ void __launch_bounds__(256) k_quant_cols(const T *__restrict__ x, Q2DParams p)
{
    __shared__ float red[32];
    float s_t = 0.0f;
    if (FMT == QFP4_NVFP4) s_t = q2d_tensor_scale(p, red);
    const NvScale nz = nv_scale_setup(s_t, p.rule);
    constexpr int G = FMT == QFP4_MXFP4 ? 32 : 16;
    const int lane = threadIdx.x & 31;
    const int64_t col_blocks = (p.K + 31) / 32, row_blocks = (p.M + 31) / 32;
    const int64_t tasks = row_blocks * col_blocks;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t task = warp0; task < tasks; task += nwarps) {
        const int64_t i0 = (task / col_blocks) * 32, j = (task % col_blocks) * 32 + lane;
        const int rows = static_cast<int>(imin<int64_t>(32, p.M - i0));   // 32, or 16 (NVFP4 with M % 32 == 16)
        if (j >= p.K) continue;                     // no shuffles below: lanes are independent
        float v[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = r < rows ? ld1(x, (i0 + r) * p.K + j) : 0.0f;
        uint32_t cw[4];
        uint32_t sc = 0u;
#pragma unroll
        for (int g = 0; g < 32 / G; ++g) {
            const float *xg = v + g * G;
            uint32_t *wg = cw + g * (G / 8);
            float amax = 0.0f;
#pragma unroll
            for (int t = 0; t < G; ++t) amax = fmaxf(amax, fabsf(xg[t]));
            uint32_t sbyte = 0u;
            float S = 0.0f, mul = 0.0f;
            if (FMT == QFP4_MXFP4) {
                if (amax != 0.0f) {
                    const int k = mx_scale_exp(amax, p.rule);
                    sbyte = static_cast<uint32_t>(k + 127);
                    S = exp2i(k);
                    mul = exp2i(-k);
                }
            } else if (s_t != 0.0f) {
                sbyte = nv_scale_byte<true>(amax, nz);
                S = __fmul_rn(e4m3_value(sbyte), s_t);
            }
            if (FMT == QFP4_NVFP4 && FOUR6) {
                uint32_t w6[2], w4[2], enc4 = 0u;
                float sse6, sse4, S4 = 0.0f;
                if (s_t != 0.0f) {
                    enc4 = nv_scale_byte<false>(amax, nz);
                    S4 = __fmul_rn(e4m3_value(enc4), s_t);
                }
                nv_block_rne(xg, S, amax, w6, &sse6);
                nv_block_rne(xg, S4, amax, w4, &sse4);
                const bool pick4 = sse4 < sse6;
                wg[0] = pick4 ? w4[0] : w6[0];
                wg[1] = pick4 ? w4[1] : w6[1];
                sbyte = pick4 ? enc4 : sbyte;
            } else if (S == 0.0f) {
#pragma unroll
                for (int t = 0; t < G / 8; ++t) wg[t] = 0u;
            } else if (FMT == QFP4_NVFP4 && !SR) {
                nv_block_rne(xg, S, amax, wg, nullptr);
            } else {
                float q[G];
                if (FMT == QFP4_MXFP4) {
#pragma unroll
                    for (int t = 0; t < G; ++t) q[t] = __fmul_rn(xg[t], mul);
                } else {
                    uint64_t pp[G / 2], qq[G / 2];
#pragma unroll
                    for (int t = 0; t < G / 2; ++t) pp[t] = f2pack(xg[2 * t], xg[2 * t + 1]);
                    nv_quot16_pairs(pp, S, amax, qq);
#pragma unroll
                    for (int t = 0; t < G / 2; ++t) f2unpack(qq[t], q[2 * t], q[2 * t + 1]);
                }
                if (SR) {
#pragma unroll
                    for (int t = 0; t < G / 8; ++t) wg[t] = 0u;
#pragma unroll
                    for (int t = 0; t < G; ++t) {
                        const uint64_t e = static_cast<uint64_t>((i0 + g * G + t) * p.K + j);
                        const uint4 rw = sr_words4(p.seed, e >> 2);
                        const uint32_t word = (e & 3) == 0 ? rw.x : (e & 3) == 1 ? rw.y : (e & 3) == 2 ? rw.z : rw.w;
                        wg[t >> 3] |= e2m1_sr(q[t], word) << (4 * (t & 7));
                    }
                } else {
#pragma unroll
                    for (int t = 0; t < G / 8; ++t) wg[t] = e2m1x8_rne(q + 8 * t);
                }
            }
            sc |= sbyte << (8 * g);
        }
        // codes of column j, rows i0 .. i0+rows-1 (8-byte aligned: M % 16 == 0)
        uint2 *cdst = reinterpret_cast<uint2 *>(p.codesT + (j * p.M + i0) / 2);
        cdst[0] = make_uint2(cw[0], cw[1]);
        if (rows == 32) cdst[1] = make_uint2(cw[2], cw[3]);
        if (G == 32) {
            p.scalesT[j * (p.M / 32) + i0 / 32] = static_cast<uint8_t>(sc);
        } else {
            p.scalesT[j * (p.M / 16) + i0 / 16] = static_cast<uint8_t>(sc);
            if (rows == 32) p.scalesT[j * (p.M / 16) + i0 / 16 + 1] = static_cast<uint8_t>(sc >> 8);
        }
    }
}

// ---------------------------------------------------------------- MXFP8 (E4M3, g32)
// ROWS / COLS: emit the row-wise and / or the column-wise output.
template <bool SR, bool ROWS, bool COLS, typename T>
__global__ void __launch_bounds__(256) k_mxfp8(const T *__restrict__ x, Q2DParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t col_blocks = p.K / 32, row_blocks = (p.M + 31) / 32;
    const int64_t tasks = row_blocks * col_blocks;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t task = warp0; task < tasks; task += nwarps) {
        const int64_t i0 = (task / col_blocks) * 32, j = (task % col_blocks) * 32 + lane;
        const int rows = static_cast<int>(imin<int64_t>(32, p.M - i0));
        float v[32];
        uint32_t wd[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            v[r] = r < rows ? ld1(x, (i0 + r) * p.K + j) : 0.0f;
            if (SR) {
                const uint64_t e = static_cast<uint64_t>((i0 + r) * p.K + j);
                const uint4 rw = sr_words4(p.seed, e >> 2);
                wd[r] = (e & 3) == 0 ? rw.x : (e & 3) == 1 ? rw.y : (e & 3) == 2 ? rw.z : rw.w;
            }
        }
        // row groups: 32 lanes of one row
        uint8_t my_scale = 0;
#pragma unroll
        for (int r = 0; r < (ROWS ? 32 : 0); ++r) {
            float amax = fabsf(v[r]);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            uint32_t byte = 0u, sbyte = 0u;
            if (amax != 0.0f) {
                const int k = scale_exp(amax, 0x600000u, 8);
                sbyte = static_cast<uint32_t>(k + 127);
                const float q = __fmul_rn(v[r], exp2i(-k));
                byte = SR ? e4m3_sr(q, wd[r]) : e4m3_rne(q);
            }
            if (lane == r) my_scale = static_cast<uint8_t>(sbyte);
            if (r < rows) p.codes[(i0 + r) * p.K + j] = static_cast<uint8_t>(byte);
        }
        if (ROWS && lane < rows) p.scales[(i0 + lane) * (p.K / 32) + j / 32] = my_scale;
        if (COLS) {                                   // column group: this lane's 32 rows
            float amax = 0.0f;
#pragma unroll
            for (int r = 0; r < 32; ++r) amax = fmaxf(amax, fabsf(v[r]));
            uint32_t bytes[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sbyte = 0u;
            if (amax != 0.0f) {
                const int k = scale_exp(amax, 0x600000u, 8);
                sbyte = static_cast<uint32_t>(k + 127);
                const float m = exp2i(-k);
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    const float q = __fmul_rn(v[r], m);
                    bytes[r >> 2] |= (SR ? e4m3_sr(q, wd[r]) : e4m3_rne(q)) << (8 * (r & 3));
                }
            }
            uint4 *dst = reinterpret_cast<uint4 *>(p.codesT + j * p.M + i0);
            dst[0] = make_uint4(bytes[0], bytes[1], bytes[2], bytes[3]);
            dst[1] = make_uint4(bytes[4], bytes[5], bytes[6], bytes[7]);
            p.scalesT[j * (p.M / 32) + i0 / 32] = static_cast<uint8_t>(sbyte);
        }
    }
}

// ---------------------------------------------------------------- column-wise outputs, 4 columns a lane
// fl(x / S) for one value: division-free when the block is on the fast path
// (y = fl(1/S)), else the IEEE division; the sign of x is kept, also on zero.
__device__ __forceinline__ float nv_quot1(float x, float S, float y, bool fast)
{
    if (!fast) return __fdiv_rn(x, S);
    const float q = div_rn_by(x, y, -S);
    return __uint_as_float(__float_as_uint(q) | (__float_as_uint(x) & 0x80000000u));   // sign of x, also on zero
}

// Round-to-nearest column-wise outputs from bf16 input (stochastic rounding
// has k_cols_sr): a warp covers 32 rows x 128 columns, lane l the 4 adjacent
// columns jb = j0 + 4 l .. jb + 3, loaded as one 8-byte word per row (256
// bytes per warp instruction).  The 32 rows stay as raw bf16 pairs (64
// registers).  Per column: the group maxima, the scales, then the codes of
// X^T row jb + c (E2M1 nibbles, or E4M3 bytes for FMT_MXFP8).  Groups along M:
// 32 (MXFP4, MXFP8) or 16 (NVFP4, where the last row block may have 16 rows).
template <int FMT, bool FOUR6>
__global__ void __launch_bounds__(256) k_cols4(const uint16_t *__restrict__ x, Q2DParams p)
{
    constexpr bool MX8 = FMT == FMT_MXFP8, NV = FMT == QFP4_NVFP4;
    constexpr int G = NV ? 16 : 32, NG = 32 / G;
    __shared__ float red[32];
    float s_t = 0.0f;
    if (NV) s_t = q2d_tensor_scale(p, red);
    const NvScale nz = nv_scale_setup(s_t, p.rule);
    const int lane = threadIdx.x & 31;
    const int64_t col_blocks = (p.K + 127) / 128, row_blocks = (p.M + 31) / 32;
    const int64_t tasks = row_blocks * col_blocks;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t task = warp0; task < tasks; task += nwarps) {
        const int64_t i0 = (task / col_blocks) * 32, jb = (task % col_blocks) * 128 + 4 * lane;
        const int rows = static_cast<int>(imin<int64_t>(32, p.M - i0));   // 32, or 16 (NVFP4, M % 32 == 16)
        if (jb >= p.K) continue;                    // K % 4 == 0: a lane's columns are all in or all out
        uint32_t raw[32][2];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            if (r < rows) {
                const uint2 w = *reinterpret_cast<const uint2 *>(x + (i0 + r) * p.K + jb);
                raw[r][0] = w.x;
                raw[r][1] = w.y;
            } else {
                raw[r][0] = raw[r][1] = 0u;
            }
        }
        auto val = [&](int r, int c) -> float { return (c & 1) ? bf16hi(raw[r][c >> 1]) : bf16lo(raw[r][c >> 1]); };

        // scales per (group, column)
        float S[NG][4], Y[NG][4], A[NG][4], mul[4];
        bool fast[NG][4];
        uint32_t sb[NG][4], w[4][MX8 ? 8 : 4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int t = 0; t < (MX8 ? 8 : 4); ++t) w[c][t] = 0u;
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float amax = 0.0f;
#pragma unroll
                for (int r = 0; r < G; ++r) amax = fmaxf(amax, fabsf(val(G * g + r, c)));
                A[g][c] = amax;
                sb[g][c] = 0u;
                S[g][c] = 0.0f;
                Y[g][c] = 0.0f;
                fast[g][c] = false;
                if (!NV) {
                    mul[c] = 0.0f;
                    if (amax != 0.0f) {
                        const int k = MX8 ? scale_exp(amax, 0x600000u, 8) : mx_scale_exp(amax, p.rule);
                        sb[g][c] = static_cast<uint32_t>(k + 127);
                        S[g][c] = 1.0f;                      // marks a nonzero group
                        mul[c] = exp2i(-k);
                    }
                } else if (s_t != 0.0f) {
                    uint32_t enc = nv_scale_byte<true>(amax, nz);
                    float Sv = __fmul_rn(e4m3_value(enc), s_t);
                    if (FOUR6) {
                        float xg[16];
#pragma unroll
                        for (int r = 0; r < 16; ++r) xg[r] = val(16 * g + r, c);
                        const uint32_t enc4 = nv_scale_byte<false>(amax, nz);
                        const float S4 = __fmul_rn(e4m3_value(enc4), s_t);
                        uint32_t w6[2], w4[2];
                        float sse6, sse4;
                        nv_block_rne(xg, Sv, amax, w6, &sse6);
                        nv_block_rne(xg, S4, amax, w4, &sse4);
                        const bool pick4 = sse4 < sse6;
                        w[c][2 * g] = pick4 ? w4[0] : w6[0];
                        w[c][2 * g + 1] = pick4 ? w4[1] : w6[1];
                        enc = pick4 ? enc4 : enc;
                    }
                    sb[g][c] = enc;
                    S[g][c] = Sv;
                    fast[g][c] = Sv >= 0x1p-125f && Sv <= 0x1p125f && amax <= Sv * 0x1p100f;
                    Y[g][c] = fast[g][c] ? __frcp_rn(Sv) : 0.0f;
                }
            }

        // codes
        if (!FOUR6) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    if (S[g][c] == 0.0f) continue;
                    if (NV) {
                        float xg[16];
#pragma unroll
                        for (int r = 0; r < 16; ++r) xg[r] = val(16 * g + r, c);
                        nv_block_rne(xg, S[g][c], A[g][c], &w[c][2 * g], nullptr);
                    } else if (MX8) {
#pragma unroll
                        for (int t = 0; t < 8; ++t)
                            w[c][t] = e4m3x2_rne(__fmul_rn(val(4 * t, c), mul[c]), __fmul_rn(val(4 * t + 1, c), mul[c])) |
                                      (e4m3x2_rne(__fmul_rn(val(4 * t + 2, c), mul[c]),
                                                  __fmul_rn(val(4 * t + 3, c), mul[c])) << 16);
                    } else {
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            float q8[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u) q8[u] = __fmul_rn(val(8 * t + u, c), mul[c]);
                            w[c][t] = e2m1x8_rne(q8);
                        }
                    }
                }
            }
        }

        // stores: X^T rows jb .. jb + 3, elements i0 .. i0 + rows - 1
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t j = jb + c;
            if (MX8) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.codesT + j * p.M + i0);
                dst[0] = make_uint4(w[c][0], w[c][1], w[c][2], w[c][3]);
                dst[1] = make_uint4(w[c][4], w[c][5], w[c][6], w[c][7]);
                p.scalesT[j * (p.M / 32) + i0 / 32] = static_cast<uint8_t>(sb[0][c]);
            } else {
                // M % 32 == 0 (always for groups of 32): 16-byte code stores and
                // the two NVFP4 scale bytes in one 2-byte store, both aligned
                const bool whole = rows == 32 && (p.M % 32) == 0;
                if (whole) {
                    *reinterpret_cast<uint4 *>(p.codesT + (j * p.M + i0) / 2) =
                        make_uint4(w[c][0], w[c][1], w[c][2], w[c][3]);
                } else {
                    uint2 *dst = reinterpret_cast<uint2 *>(p.codesT + (j * p.M + i0) / 2);
                    dst[0] = make_uint2(w[c][0], w[c][1]);
                    if (rows == 32) dst[1] = make_uint2(w[c][2], w[c][3]);
                }
                if (G == 32) {
                    p.scalesT[j * (p.M / 32) + i0 / 32] = static_cast<uint8_t>(sb[0][c]);
                } else if (whole) {
                    *reinterpret_cast<uint16_t *>(p.scalesT + j * (p.M / 16) + i0 / 16) =
                        static_cast<uint16_t>(sb[0][c] | (sb[NG - 1][c] << 8));
                } else {
                    p.scalesT[j * (p.M / 16) + i0 / 16] = static_cast<uint8_t>(sb[0][c]);
                    if (rows == 32) p.scalesT[j * (p.M / 16) + i0 / 16 + 1] = static_cast<uint8_t>(sb[NG - 1][c]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------- host
// One resident wave of 256-thread blocks (8 warps each, one task per warp at
// a time): each block pays its prologue (the tensor-scale reduction) once,
// and its warps loop over their tasks.
template <auto Kern>
static int grid_for_warps(int64_t warp_tasks)
{
    static const int per_sm = [] {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, Kern, 256, 0) != cudaSuccess || b < 1) {
            (void)cudaGetLastError();
            b = 1;
        }
        return b;
    }();
    const int64_t blocks = (warp_tasks + 7) / 8;
    return static_cast<int>(imax<int64_t>(1, imin<int64_t>(blocks, static_cast<int64_t>(per_sm) * num_sms())));
}

// Launch one of the tile kernels with its resident-wave grid.
template <auto Kern, typename T>
static void launch_tiles(int64_t warp_tasks, const void *x, const Q2DParams &p, cudaStream_t stream)
{
    Kern<<<grid_for_warps<Kern>(warp_tasks), 256, 0, stream>>>(static_cast<const T *>(x), p);
}

// 2D blocks: NVFP4 16 x 16 (after the amax pass, unless the caller gives
// the tensor amax and does not ask for it back) or MXFP4 32 x 32 tiles.
int quantize2d(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_fmt fmt, qfp4_round rounding,
               uint64_t seed, uint8_t *codes, uint8_t *scales, uint8_t *codesT, uint8_t *scalesT, float *tscale,
               float *partials, cudaStream_t stream, const QuantOpts &opt)
{
    const bool sr = rounding == QFP4_SR;
    Q2DParams p{M, K, codes, scales, codesT, scalesT, partials, 0, tscale, seed, opt.rule, opt.amax_in};
    if (fmt == QFP4_MXFP4) {
        const int64_t tasks = (M / 32) * (K / 32);
        if (xdt == QFP4_BF16) {
            if (sr) launch_tiles<k_quant2d_mx<true, uint16_t>, uint16_t>(tasks, x, p, stream);
            else launch_tiles<k_quant2d_mx<false, uint16_t>, uint16_t>(tasks, x, p, stream);
        } else {
            if (sr) launch_tiles<k_quant2d_mx<true, float>, float>(tasks, x, p, stream);
            else launch_tiles<k_quant2d_mx<false, float>, float>(tasks, x, p, stream);
        }
        QFP4_LAUNCH_CHECK();
        return QFP4_OK;
    }
    const int64_t tasks = ((M / 16 + 3) / 4) * ((K / 16 + 1) / 2);     // 64 x 32 warp tasks
    if (tasks >= (int64_t(1) << 31)) return QFP4_ERR_SHAPE;            // the kernel indexes tasks in 32 bits
    if (!opt.amax_in || opt.amax_out) {
        int st = amax_partials(x, xdt, M * K, partials, &p.n_partials, stream);
        if (st != QFP4_OK) return st;
        if (opt.amax_out) {
            st = partials_max(partials, p.n_partials, opt.amax_out, stream);
            if (st != QFP4_OK) return st;
        }
    }
    if (xdt == QFP4_BF16) {
        if (sr) launch_tiles<k_quant2d<true, uint16_t>, uint16_t>(tasks, x, p, stream);
        else launch_tiles<k_quant2d<false, uint16_t>, uint16_t>(tasks, x, p, stream);
    } else {
        if (sr) launch_tiles<k_quant2d<true, float>, float>(tasks, x, p, stream);
        else launch_tiles<k_quant2d<false, float>, float>(tasks, x, p, stream);
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

// Stochastic rounding of the column-wise outputs from bf16 input.  A warp
// covers 32 rows x 64 columns; lanes 2p and 2p + 1 share the 4 adjacent
// columns jb = j0 + 4p .. jb + 3, lane q = lane & 1 taking columns jb + 2q
// and jb + 2q + 1, read as one 4-byte word per row (128 bytes per warp
// instruction, 32 registers for the tile, so two blocks fit an SM where the
// 4-columns-a-lane kernel fits one).  The Philox counter of a row's 4
// columns is ((i0 + r) K + jb) / 4: in step k the lower lane of a pair draws
// row k and the upper lane row 16 + k, each keeps the two words of its own
// columns and sends the other two to its partner, so each call still serves
// four elements.  The decision runs on the lane's two columns as a packed
// pair.  All-zero groups (and NVFP4 blocks whose scale is 0) get +0 codes.
// Groups along M: 32 (MXFP4, MXFP8) or 16 (NVFP4, whose last row block may
// have 16 rows).  No lane leaves the loop early: the shuffles need the whole
// warp, so lanes past K load zeros and store nothing.
template <int FMT>
__global__ void __launch_bounds__(256) k_cols_sr(const uint16_t *__restrict__ x, Q2DParams p)
{
    constexpr bool MX8 = FMT == FMT_MXFP8, NV = FMT == QFP4_NVFP4;
    constexpr int G = NV ? 16 : 32, NG = 32 / G, CW = MX8 ? 8 : 4;   // code words per column
    __shared__ float red[32];
    float s_t = 0.0f;
    if (NV) s_t = q2d_tensor_scale(p, red);
    const NvScale nz = nv_scale_setup(s_t, p.rule);
    const int lane = threadIdx.x & 31, q = lane & 1;
    const int64_t col_blocks = (p.K + 63) / 64, row_blocks = (p.M + 31) / 32;
    const int64_t tasks = row_blocks * col_blocks;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t task = warp0; task < tasks; task += nwarps) {
        const int64_t i0 = (task / col_blocks) * 32, jb = (task % col_blocks) * 64 + 4 * (lane >> 1);
        const int rows = static_cast<int>(imin<int64_t>(32, p.M - i0));   // 32, or 16 (NVFP4, M % 32 == 16)
        const bool colv = jb < p.K;                 // K % 4 == 0: a pair's columns are all in or all out
        const int64_t j = jb + 2 * q;               // this lane's first column
        uint32_t raw[32];
#pragma unroll
        for (int r = 0; r < 32; ++r)
            raw[r] = (colv && r < rows) ? *reinterpret_cast<const uint32_t *>(x + (i0 + r) * p.K + j) : 0u;

        // per group and column: the scale byte, the divisor (or multiplier)
        uint64_t mul2[NG], y2[NG], nS2[NG];
        bool fast2[NG], zero[NG][2];
        float Sg[NG][2], Yg[NG][2];
        uint32_t sb[NG][2];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            uint32_t m = 0u;                        // |bf16| maxima of both columns as 16-bit integers
#pragma unroll
            for (int r = 0; r < G; ++r) {
                uint32_t t;
                asm("max.u16x2 %0, %1, %2;" : "=r"(t) : "r"(m), "r"(raw[G * g + r] & 0x7FFF7FFFu));
                m = t;
            }
            const float amax[2] = {bf16lo(m), bf16hi(m)};
            float mulc[2] = {0.0f, 0.0f};
            bool fast[2] = {false, false};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                sb[g][c] = 0u;
                Sg[g][c] = 0.0f;
                Yg[g][c] = 0.0f;
                if (!NV) {
                    zero[g][c] = amax[c] == 0.0f;
                    if (!zero[g][c]) {
                        const int k = MX8 ? scale_exp(amax[c], 0x600000u, 8) : mx_scale_exp(amax[c], p.rule);
                        sb[g][c] = static_cast<uint32_t>(k + 127);
                        mulc[c] = exp2i(-k);
                    }
                } else {
                    if (s_t != 0.0f) {
                        sb[g][c] = nv_scale_byte<true>(amax[c], nz);
                        Sg[g][c] = __fmul_rn(e4m3_value(sb[g][c]), s_t);
                    }
                    zero[g][c] = Sg[g][c] == 0.0f;
                    fast[c] = Sg[g][c] >= 0x1p-125f && Sg[g][c] <= 0x1p125f && amax[c] <= Sg[g][c] * 0x1p100f;
                    Yg[g][c] = fast[c] ? __frcp_rn(Sg[g][c]) : 0.0f;
                }
            }
            mul2[g] = f2pack(mulc[0], mulc[1]);
            y2[g] = f2pack(Yg[g][0], Yg[g][1]);
            nS2[g] = f2pack(-Sg[g][0], -Sg[g][1]);
            fast2[g] = fast[0] && fast[1];
        }

        uint32_t code[2][CW];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int t = 0; t < CW; ++t) code[c][t] = 0u;
        // one element pair (row r, the lane's two columns) under words w0, w1
        auto round_pair = [&](int r, uint32_t w0, uint32_t w1) {
            const int g = r / G;
            const uint64_t v = f2pack(bf16lo(raw[r]), bf16hi(raw[r]));
            uint64_t qv;
            if (!NV) {
                qv = f2mul(v, mul2[g]);
            } else if (fast2[g]) {
                qv = div_rn_by2(v, y2[g], nS2[g]);
            } else {
                qv = f2pack(nv_quot1(bf16lo(raw[r]), Sg[g][0], Yg[g][0], Yg[g][0] != 0.0f),
                            nv_quot1(bf16hi(raw[r]), Sg[g][1], Yg[g][1], Yg[g][1] != 0.0f));
            }
            if (MX8) {
                float q0, q1;
                f2unpack(qv, q0, q1);
                const uint32_t b2 = e4m3_sr2(q0, q1, w0, w1);   // column 0 in the low byte
                code[0][r >> 2] |= (b2 & 0xFFu) << (8 * (r & 3));
                code[1][r >> 2] |= (b2 >> 8) << (8 * (r & 3));
            } else {
                float g0, g1;
                f2unpack(e2m1_sr_grid2(qv, w0, w1), g0, g1);
                uint32_t b;                         // low nibble: column 0, high nibble: column 1
                asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
                    : "=r"(b) : "f"(g1), "f"(g0));
                code[0][r >> 3] |= (b & 0xFu) << (4 * (r & 7));
                code[1][r >> 3] |= ((b >> 4) & 0xFu) << (4 * (r & 7));
            }
        };
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int rr = k + 16 * q;               // the row this lane draws
            const uint4 wd = sr_words4(p.seed, static_cast<uint64_t>((i0 + rr) * p.K + jb) >> 2);
            const uint32_t own0 = q ? wd.z : wd.x, own1 = q ? wd.w : wd.y;
            const uint32_t got0 = __shfl_xor_sync(0xFFFFFFFFu, q ? wd.x : wd.z, 1);
            const uint32_t got1 = __shfl_xor_sync(0xFFFFFFFFu, q ? wd.y : wd.w, 1);
            round_pair(k, q ? got0 : own0, q ? got1 : own1);                  // row k
            if (16 + k < rows) round_pair(16 + k, q ? own0 : got0, q ? own1 : got1);   // row 16 + k
        }
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int c = 0; c < 2; ++c)
                if (zero[g][c])
#pragma unroll
                    for (int t = g * CW / NG; t < (g + 1) * CW / NG; ++t) code[c][t] = 0u;

        // stores: X^T rows j, j + 1; elements i0 .. i0 + rows - 1
        if (colv) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int64_t jr = j + c;
                if (MX8) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.codesT + jr * p.M + i0);
                    dst[0] = make_uint4(code[c][0], code[c][1], code[c][2], code[c][3]);
                    dst[1] = make_uint4(code[c][4], code[c][5], code[c][6], code[c][7]);
                    p.scalesT[jr * (p.M / 32) + i0 / 32] = static_cast<uint8_t>(sb[0][c]);
                } else {
                    // M % 32 == 0 (always for groups of 32): 16-byte code stores and
                    // the two NVFP4 scale bytes in one 2-byte store, both aligned
                    const bool whole = rows == 32 && (p.M % 32) == 0;
                    if (whole) {
                        *reinterpret_cast<uint4 *>(p.codesT + (jr * p.M + i0) / 2) =
                            make_uint4(code[c][0], code[c][1], code[c][2], code[c][3]);
                    } else {
                        uint2 *dst = reinterpret_cast<uint2 *>(p.codesT + (jr * p.M + i0) / 2);
                        dst[0] = make_uint2(code[c][0], code[c][1]);
                        if (rows == 32) dst[1] = make_uint2(code[c][2], code[c][3]);
                    }
                    if (G == 32) {
                        p.scalesT[jr * (p.M / 32) + i0 / 32] = static_cast<uint8_t>(sb[0][c]);
                    } else if (whole) {
                        *reinterpret_cast<uint16_t *>(p.scalesT + jr * (p.M / 16) + i0 / 16) =
                            static_cast<uint16_t>(sb[0][c] | (sb[NG - 1][c] << 8));
                    } else {
                        p.scalesT[jr * (p.M / 16) + i0 / 16] = static_cast<uint8_t>(sb[0][c]);
                        if (rows == 32) p.scalesT[jr * (p.M / 16) + i0 / 16 + 1] = static_cast<uint8_t>(sb[NG - 1][c]);
                    }
                }
            }
        }
    }
}

// bf16: the lane-pair kernel for stochastic rounding (32 x 64 tasks), else the
// 4-columns-a-lane kernel (32 x 128 tasks); binary32: one column a lane.
template <int FMT, bool SR, bool FOUR6>
static int launch_cols(const void *x, qfp4_dtype xdt, const Q2DParams &p, cudaStream_t stream)
{
    if (xdt == QFP4_BF16) {
        if constexpr (SR)
            launch_tiles<k_cols_sr<FMT>, uint16_t>(((p.M + 31) / 32) * ((p.K + 63) / 64), x, p, stream);
        else
            launch_tiles<k_cols4<FMT, FOUR6>, uint16_t>(((p.M + 31) / 32) * ((p.K + 127) / 128), x, p, stream);
    } else
        launch_tiles<k_quant_cols<FMT, SR, FOUR6, float>, float>(((p.M + 31) / 32) * ((p.K + 31) / 32), x, p, stream);
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

int quantize_columns(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_fmt fmt, qfp4_round rounding, int four6,
                     uint64_t seed, uint8_t *codesT, uint8_t *scalesT, const float *partials, int n_partials,
                     cudaStream_t stream, const QuantOpts &opt)
{
    Q2DParams p{M, K, nullptr, nullptr, codesT, scalesT, partials, n_partials, nullptr, seed, opt.rule, opt.amax_in};
    const bool sr = rounding == QFP4_SR;
    if (fmt == QFP4_MXFP4)
        return sr ? launch_cols<QFP4_MXFP4, true, false>(x, xdt, p, stream)
                  : launch_cols<QFP4_MXFP4, false, false>(x, xdt, p, stream);
    if (four6) return launch_cols<QFP4_NVFP4, false, true>(x, xdt, p, stream);
    return sr ? launch_cols<QFP4_NVFP4, true, false>(x, xdt, p, stream)
              : launch_cols<QFP4_NVFP4, false, false>(x, xdt, p, stream);
}

int quantize_mxfp8(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_round rounding, uint64_t seed,
                   uint8_t *codes, uint8_t *scales, uint8_t *codesT, uint8_t *scalesT, cudaStream_t stream)
{
    Q2DParams p{M, K, codes, scales, codesT, scalesT, nullptr, 0, nullptr, seed, QFP4_SCALE_DEFAULT, nullptr};
    const int64_t tasks = ((M + 31) / 32) * (K / 32);
    const bool sr = rounding == QFP4_SR, cols = codesT != nullptr;
    if (xdt == QFP4_BF16 && (M * K) % 64 == 0) {
        // row-wise output through the TMA-fed 1D kernel; the column-wise one
        // (if asked for) by the tile kernel without its row part
        int st = mxfp8_rows(x, M * K, sr, seed, codes, scales, stream);
        if (st != QFP4_OK || !cols) return st;
        if (sr) launch_tiles<k_cols_sr<FMT_MXFP8>, uint16_t>(((M + 31) / 32) * ((K + 63) / 64), x, p, stream);
        else launch_tiles<k_cols4<FMT_MXFP8, false>, uint16_t>(((M + 31) / 32) * ((K + 127) / 128), x, p, stream);
        QFP4_LAUNCH_CHECK();
        return QFP4_OK;
    }
#define QFP4_MX8(SRV, COLV)                                                                     \
    do {                                                                                        \
        if (xdt == QFP4_BF16) launch_tiles<k_mxfp8<SRV, true, COLV, uint16_t>, uint16_t>(tasks, x, p, stream); \
        else launch_tiles<k_mxfp8<SRV, true, COLV, float>, float>(tasks, x, p, stream);          \
    } while (0)
    if (sr) {
        if (cols) QFP4_MX8(true, true);
        else QFP4_MX8(true, false);
    } else {
        if (cols) QFP4_MX8(false, true);
        else QFP4_MX8(false, false);
    }
#undef QFP4_MX8
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

// MXFP8 column-wise output alone (groups of 32 along M, K x M codes): the
// transposed operands of the FP8 backward GEMMs.  Needs M % 32 == 0.
int quantize_mxfp8_columns(const void *x, qfp4_dtype xdt, int64_t M, int64_t K, qfp4_round rounding, uint64_t seed,
                           uint8_t *codesT, uint8_t *scalesT, cudaStream_t stream)
{
    Q2DParams p{M, K, nullptr, nullptr, codesT, scalesT, nullptr, 0, nullptr, seed, QFP4_SCALE_DEFAULT, nullptr};
    const bool sr = rounding == QFP4_SR;
    if (xdt == QFP4_BF16) {
        if (sr) launch_tiles<k_cols_sr<FMT_MXFP8>, uint16_t>(((M + 31) / 32) * ((K + 63) / 64), x, p, stream);
        else launch_tiles<k_cols4<FMT_MXFP8, false>, uint16_t>(((M + 31) / 32) * ((K + 127) / 128), x, p, stream);
    } else {
        const int64_t tasks = ((M + 31) / 32) * (K / 32);
        if (sr) launch_tiles<k_mxfp8<true, false, true, float>, float>(tasks, x, p, stream);
        else launch_tiles<k_mxfp8<false, false, true, float>, float>(tasks, x, p, stream);
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

}  // namespace qfp4
