// qfp4_common.cuh -- shared device/host helpers of libqfp4 (sm_100a only).
//
// Holds: the status plumbing, PTX wrappers for mbarriers and TMA, the
// tensor-map encoder (reached through the driver entry point, so the
// library does not link libcuda), and the device numerics of the method:
// Philox4x32-10, the E2M1 / E4M3 conversions, the truncation-free E8M0
// exponent and the Walsh-Hadamard butterflies.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/qfp4.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "libqfp4 is built for sm_100a only"
#endif

namespace qfp4 {

template <class T>
__host__ __device__ __forceinline__ T imin(T a, T b) { return a < b ? a : b; }
template <class T>
__host__ __device__ __forceinline__ T imax(T a, T b) { return a < b ? b : a; }

// ------------------------------------------------------------------ errors
// Device-side sticky error word: the code of the first bounded wait that gave
// up (QFP4_DEV_ERR_TIMEOUT), read and cleared by qfp4_last_device_error.
enum : int { DEV_ERR_NONE = 0, DEV_ERR_TIMEOUT = QFP4_DEV_ERR_TIMEOUT };
static __device__ int g_dev_error = 0;   // one copy: the library is a single translation unit

// A spin on an mbarrier gives up after this many polls (seconds of wall
// time), records DEV_ERR_TIMEOUT and lets the kernel return.
constexpr uint32_t kSpinLimit = 1u << 28;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_dev_error, 0, code); }

// ------------------------------------------------------------------ PTX: mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// After a wait gave up: let copies this thread already started (TMA loads,
// at most a few stages) land before the CTA leaves, for at most `ns`.
__device__ __forceinline__ void settle_ns(uint64_t ns)
{
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < ns) {
    }
}
constexpr uint64_t kSettleNs = 100000ull;

// Bounded wait: true when the phase completed, false (error recorded) when
// limit_ns of wall time (or kSpinLimit polls) ran out.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && global_ns() - t0 > limit_ns) break;
    }
    record_error(DEV_ERR_TIMEOUT);
    return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// ------------------------------------------------------------------ dependent launches
// Kernels are launched with programmatic stream serialization: a kernel may
// start (run its prologue: barrier setup, tensor-map prefetch, tensor-memory
// allocation) while the previous kernel in the stream is finishing.  Every
// thread calls pdl_wait() before its first global-memory access; it returns
// once the previous grid has completed and its writes are visible (at once
// when there is no such grid).  pdl_trigger() lets the next kernel be
// scheduled as soon as every CTA of this grid has issued it or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// ------------------------------------------------------------------ PTX: TMA
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ numerics
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): multipliers 0xD2511F53
// and 0xCD9E8D57, Weyl increments 0x9E3779B9 / 0xBB67AE85, ten rounds.
// Counter (c0, c1, 0, 0); key (k0, k1).
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t k0, uint32_t k1)
{
    uint32_t c2 = 0u, c3 = 0u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
        const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return make_uint4(c0, c1, c2, c3);
}

// The four random words of elements 4q .. 4q+3 (counter q = e / 4).
__device__ __forceinline__ uint4 sr_words4(uint64_t seed, uint64_t q)
{
    return philox4x32_10(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32), static_cast<uint32_t>(seed),
                         static_cast<uint32_t>(seed >> 32));
}

// Two bf16 packed in a 32-bit word -> binary32 (exact widening).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E2M1 round-to-nearest-even with saturation to +-6, eight values packed
// into one 32-bit word (element t in nibble t), by the sm_100 hardware
// conversion.  The conversion keeps the sign of zero (-0.0 and negative
// values that round to zero give code 0x8), which is the rule this library
// follows; an exhaustive sweep of all finite binary32 inputs on B200 agrees
// with the nearest / ties-to-even / saturating definition bit for bit.
__device__ __forceinline__ uint32_t e2m1x8_rne(const float *v)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// ------------------------------------------------------------------ packed binary32 pairs
// Two binary32 values in one 64-bit register pair (low = the even element);
// sm_100's f32x2 arithmetic does two IEEE round-to-nearest operations per
// instruction.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t p, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// two bf16 (one 32-bit word) -> a packed pair, exact
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w)
{
    return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// E2M1 RNE of four packed pairs (8 values) -> one word of nibbles
__device__ __forceinline__ uint32_t e2m1x8_rne_pairs(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3)
{
    float v[8];
    f2unpack(p0, v[0], v[1]);
    f2unpack(p1, v[2], v[3]);
    f2unpack(p2, v[4], v[5]);
    f2unpack(p3, v[6], v[7]);
    return e2m1x8_rne(v);
}

// The eight E2M1 values of a word of nibbles as binary32 (exact: binary16
// holds every E2M1 value, and the widening is exact).
__device__ __forceinline__ void e2m1x8_values(uint32_t w, uint64_t *g4)
{
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[q]));
        g4[q] = f2pack(f.x, f.y);
    }
}

// E2M1 stochastic rounding of one value (|v| <= 6 or saturating):
// lo <= |v| < hi adjacent grid values, up iff u < (|v| - lo) / (hi - lo)
// with u = (w >> 8) * 2^-24.  Returns the 4-bit code.
__device__ __forceinline__ float e2m1_sr_grid(float v, uint32_t w)
{
    // Grid spacing sp = 2^(m - 128) with m = clamp(biased exponent of |v|, 127, 129):
    // 0.5 below 2, 1 in [2, 4), 2 from 4 on.  Everything below is exact binary32:
    //   q24 = |v| / sp * 2^24                      (scaling by a power of two)
    //   fl24 = floor(q24 / 2^24) * 2^24            (round-toward-zero add of 1.5 * 2^47,
    //                                               whose ulp is 2^24, then its removal)
    //   frac24 = q24 - fl24 = ((|v| - lo) / sp) * 2^24
    // so u < (|v| - lo) / sp with u = (w >> 8) * 2^-24 is (w >> 8) < frac24, and the
    // result is (fl24 or fl24 + 2^24) * sp * 2^-24, saturated at 6.
    const float a = fabsf(v);
    const int m = imin(imax(static_cast<int>(__float_as_uint(a) >> 23), 127), 129);
    const float inv24 = __uint_as_float(static_cast<uint32_t>(279 - m) << 23);   // 2^24 / sp
    const float sp24 = __uint_as_float(static_cast<uint32_t>(m - 25) << 23);     // sp / 2^24
    const float q24 = __fmul_rn(a, inv24);
    const float fl24 = __fsub_rn(__fadd_rz(q24, 211106232532992.0f), 211106232532992.0f);   // 1.5 * 2^47
    const float frac24 = __fsub_rn(q24, fl24);
    const float r24 = (static_cast<float>(w >> 8) < frac24) ? __fadd_rn(fl24, 16777216.0f) : fl24;
    const float r = fminf(__fmul_rn(r24, sp24), 6.0f);
    return __uint_as_float(__float_as_uint(r) | (__float_as_uint(v) & 0x80000000u));   // sign kept, also on zero
}

// add.rz on a packed binary32 pair.
__device__ __forceinline__ uint64_t f2add_rz(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// e2m1_sr_grid on two values held as a packed binary32 pair (the even
// element low) with random words w0 / w1, the pair's arithmetic on the
// f32x2 pipe.  The grid spacing's exponent is clamped below only: |v| >= 8
// keeps its own binade (spacing >= 4), so its grid value is >= 8, and grid
// values above 6 are left for the saturating conversion that follows (all
// are finite).  Same codes as e2m1_sr on each value.
__device__ __forceinline__ uint64_t e2m1_sr_grid2(uint64_t vv, uint32_t w0, uint32_t w1)
{
    float v0, v1;
    f2unpack(vv, v0, v1);
    const uint32_t b0 = __float_as_uint(v0) & 0x7FFFFFFFu, b1 = __float_as_uint(v1) & 0x7FFFFFFFu;
    const uint32_t m0 = imax(b0 >> 23, 127u), m1 = imax(b1 >> 23, 127u);
    const uint64_t inv = f2pack(__uint_as_float((279u - m0) << 23), __uint_as_float((279u - m1) << 23));
    const uint64_t sp = f2pack(__uint_as_float((m0 - 25u) << 23), __uint_as_float((m1 - 25u) << 23));
    const uint64_t C = f2pack(211106232532992.0f, 211106232532992.0f);   // 1.5 * 2^47
    const uint64_t q24 = f2mul(f2pack(__uint_as_float(b0), __uint_as_float(b1)), inv);
    const uint64_t fl24 = f2sub(f2add_rz(q24, C), C);
    float f0, f1;
    f2unpack(f2sub(q24, fl24), f0, f1);
    const uint64_t up = f2pack(static_cast<float>(w0 >> 8) < f0 ? 16777216.0f : 0.0f,
                               static_cast<float>(w1 >> 8) < f1 ? 16777216.0f : 0.0f);
    float r0, r1;
    f2unpack(f2mul(f2add(fl24, up), sp), r0, r1);
    return f2pack(__uint_as_float(__float_as_uint(r0) | (__float_as_uint(v0) & 0x80000000u)),
                  __uint_as_float(__float_as_uint(r1) | (__float_as_uint(v1) & 0x80000000u)));
}

// The same rule as a 4-bit code.
__device__ __forceinline__ uint32_t e2m1_sr(float v, uint32_t w)
{
    const float r = e2m1_sr_grid(v, w);
    uint32_t code;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %1;\n\tcvt.u32.u8 %0, b;\n\t}" : "=r"(code) : "f"(r));
    return code & 0xFu;
}

// E4M3 (OCP) round-to-nearest-even, saturating to +-448: returns the byte.
__device__ __forceinline__ uint32_t e4m3_rne(float v)
{
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(out) : "f"(v));
    return out & 0xFFu;
}

// Two values -> two E4M3 bytes (a in the low byte).
__device__ __forceinline__ uint32_t e4m3x2_rne(float a, float b)
{
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(b), "f"(a));
    return out;
}

// E4M3 stochastic rounding: lo <= |v| < hi adjacent E4M3 values (subnormal
// spacing 2^-9 below 2^-6, else 2^(e-3)), up iff (w >> 8) * 2^-24 < (|v|-lo)/(hi-lo);
// saturates at 448.  Returns the byte.
__device__ __forceinline__ uint32_t e4m3_sr(float v, uint32_t w)
{
    const uint32_t sign = (__float_as_uint(v) >> 24) & 0x80u;
    const float a = fabsf(v);
    float lo, sp, inv_sp;
    if (a >= 0.015625f) {                                    // 2^-6: normal binade
        const uint32_t spb = (__float_as_uint(a) & 0x7F800000u) - (3u << 23);
        lo = __uint_as_float(__float_as_uint(a) & 0x7FF00000u);
        sp = __uint_as_float(spb);
        inv_sp = __uint_as_float((254u << 23) - spb);
    } else {
        lo = __fmul_rn(truncf(__fmul_rn(a, 512.0f)), 0.001953125f);   // exact: multiples of 2^-9
        sp = 0.001953125f;
        inv_sp = 512.0f;
    }
    const float p = __fmul_rn(__fsub_rn(a, lo), inv_sp);
    const float u = __fmul_rn(static_cast<float>(w >> 8), 5.9604644775390625e-08f);
    float rr = (u < p) ? __fadd_rn(lo, sp) : lo;
    rr = fminf(rr, 448.0f);
    return e4m3_rne(rr) | sign;
}

// e4m3_sr on two values at once (a in the low byte), without a branch: in
// the normal binades (|v| >= 2^-6) the grid keeps 3 of the 23 mantissa bits
// and up iff (w >> 8) < 16 * (the 20 dropped bits), i.e. (w >> 12) < them,
// so adding 0xFFFFF - (w >> 12) to the bits and clearing the low 20 rounds
// (a carry moves into the exponent); below 2^-6 the spacing is 2^-9 and the
// fraction is compared as in e4m3_sr.  Saturates at 448.
__device__ __forceinline__ uint32_t e4m3_sr2(float a, float b, uint32_t wa, uint32_t wb)
{
    const float v[2] = {a, b};
    const uint32_t w[2] = {wa, wb};
    float r[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const uint32_t bits = __float_as_uint(v[t]) & 0x7FFFFFFFu;
        const uint32_t rn = (bits + (0xFFFFFu - (w[t] >> 12))) & 0xFFF00000u;
        const float t9 = __fmul_rn(__uint_as_float(bits), 512.0f), f9 = truncf(t9);
        const float frac24 = __fmul_rn(__fsub_rn(t9, f9), 16777216.0f);
        const float rs = __fmul_rn(static_cast<float>(w[t] >> 8) < frac24 ? __fadd_rn(f9, 1.0f) : f9, 0.001953125f);
        const float rr = fminf(bits >= 0x3C800000u ? __uint_as_float(rn) : rs, 448.0f);
        r[t] = __uint_as_float(__float_as_uint(rr) | (__float_as_uint(v[t]) & 0x80000000u));
    }
    return e4m3x2_rne(r[0], r[1]);
}

// E4M3 byte -> binary32 (exact), from the bit fields.
__device__ __forceinline__ float e4m3_value(uint32_t b)
{
    const uint32_t E = (b >> 3) & 15u, m = b & 7u;
    // E == 0: m * 2^-9 (2^-9 has binary32 exponent field 118); E > 0: (1 + m/8) 2^(E-7)
    const float mag = (E == 0) ? static_cast<float>(m) * __uint_as_float(118u << 23)
                               : __uint_as_float(((E + 120u) << 23) | (m << 20));
    return (b & 0x80u) ? -mag : mag;
}

// Least k in [-127, 127] with top * 2^k >= amax, top = top_m * 2^top_e with
// top_m in [1, 2) given by its 23-bit fraction (6 = 1.5 * 2^2: 0x400000, 2;
// 448 = 1.75 * 2^8: 0x600000, 8).  amax = m * 2^e: k = e - top_e when
// m <= top_m, else e - top_e + 1.  amax == 0 gives -127.
__device__ __forceinline__ int scale_exp(float amax, uint32_t top_frac, int top_e)
{
    const uint32_t u = __float_as_uint(amax) & 0x7FFFFFFFu;
    if (u == 0) return -127;
    int e;
    uint32_t f;
    const uint32_t E = u >> 23;
    if (E == 0) {                                  // subnormal: normalise
        const int lead = 31 - __clz(u);
        e = lead - 149;
        f = (u << (23 - lead)) & 0x7FFFFFu;
    } else {
        e = static_cast<int>(E) - 127;
        f = u & 0x7FFFFFu;
    }
    const int k = (f <= top_frac) ? e - top_e : e - top_e + 1;
    return max(-127, min(127, k));
}

// The OCP microscaling exponent: k = floor(log2(amax)) - emax (emax = 2 for
// E2M1), the largest k with 2^(k + emax) <= amax, clamped to [-127, 127];
// amax / 2^k lies in [2^emax, 2^(emax+1)), so magnitudes above the format's
// largest value clip.  amax == 0 gives -127.
__device__ __forceinline__ int scale_exp_floor(float amax, int emax)
{
    const uint32_t u = __float_as_uint(amax) & 0x7FFFFFFFu;
    if (u == 0) return -127;
    const uint32_t E = u >> 23;
    const int e = E == 0 ? (31 - __clz(u)) - 149 : static_cast<int>(E) - 127;
    return max(-127, min(127, e - emax));
}

// Scale rules (qfp4_scale_rule): the E8M0 exponent of an MXFP4 group.
__device__ __forceinline__ int mx_scale_exp(float amax, int rule)
{
    return rule == QFP4_SCALE_OCP_FLOOR ? scale_exp_floor(amax, 2) : scale_exp(amax, 0x400000u, 2);
}

// E4M3 byte of t >= 0 rounded up: the least finite E4M3 value >= t,
// saturating at 448.  Non-negative E4M3 bytes 0x00 .. 0x7E increase with
// their value, so one step up from the nearest byte when it lies below t.
__device__ __forceinline__ uint32_t e4m3_up_byte(float t, uint32_t nearest)
{
    return (nearest < 0x7Eu && e4m3_value(nearest) < t) ? nearest + 1u : nearest;
}

// 2^k as binary32 for k in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float exp2i(int k)
{
    return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// binary32 constant nearest 1/sqrt(128) = 2^-3.5.
__device__ __forceinline__ float inv_sqrt128() { return __uint_as_float(0x3DB504F3u); }

}  // namespace qfp4

// ------------------------------------------------------------------ host side
namespace qfp4 {

int encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, int rank, void *gaddr, const uint64_t *dims,
                      const uint64_t *strides_bytes /* rank-1 entries */, const uint32_t *box,
                      CUtensorMapSwizzle swizzle);

int num_sms();

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raise kernel Kern's dynamic shared-memory limit to `bytes` on the current
// device.  The attribute is per device, so it is recorded per device (and
// per kernel: one set of flags per template instance); devices beyond the
// table set it on every call.
template <auto Kern>
int ensure_dyn_smem(int bytes)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];       // static storage: starts at zero
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    const bool tracked = dev >= 0 && dev < kMaxDevices;
    if (tracked && done[dev].load(std::memory_order_acquire) >= bytes) return QFP4_OK;
    if (cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    if (tracked) done[dev].store(bytes, std::memory_order_release);
    return QFP4_OK;
}

}  // namespace qfp4

namespace qfp4 {
void count_launch();
}

// After every kernel launch: count it, and turn a launch error into a status.
#define QFP4_LAUNCH_CHECK()                                                                        \
    do {                                                                                           \
        qfp4::count_launch();                                                                      \
        if (cudaPeekAtLastError() != cudaSuccess) {                                                \
            (void)cudaGetLastError();                                                              \
            return QFP4_ERR_CUDA;                                                                  \
        }                                                                                          \
    } while (0)
