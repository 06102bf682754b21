// calib.cu -- KL-divergence clip calibration of an activation tensor ([LB]
// §5, the TensorRT method: for each candidate clip point T, P = the
// histogram of |x| cut at T with the tail counted in the last kept bin, Q =
// the kept histogram quantized to the levels and spread back over P's bins;
// the T with the least D_KL(P || Q) loses the least information).
//
// Three launches after the tensor-amax pass: a histogram of |x| over [0,
// amax] privatized in shared memory; one thread per candidate computing its
// KL (the level of a bin never decreases with the bin, so a level's bins are
// one contiguous run: a first walk over the run gathers its kept mass and
// the count of P's nonzero bins, a second adds the run's terms, bins in
// ascending order); one block taking the least KL (smallest candidate on a
// tie) and writing the clip point T = fl(i * fl(amax / bins)).
#include <math_constants.h>

#include "qfp4_common.cuh"
#include "quantize1d.cuh"

namespace qfp4 {

constexpr int KL_MAX_BINS = 8192;               // 32 KiB of shared counters

template <typename T>
__global__ void __launch_bounds__(256) k_abs_hist(const T *__restrict__ x, int64_t n, int bins, const float *amax_p,
                                                  unsigned long long *hist)
{
    extern __shared__ uint32_t counts[];
    pdl_wait();
    pdl_trigger();
    for (int b = threadIdx.x; b < bins; b += blockDim.x) counts[b] = 0u;
    __syncthreads();
    const float amax = *amax_p;
    const bool zero = !(amax > 0.0f);
    const float inv = zero ? 0.0f : __fdiv_rn(static_cast<float>(bins), amax);
    auto bin = [&](float v) -> int {
        if (zero) return 0;
        const int b = __float2int_rz(__fmul_rn(fabsf(v), inv));
        return b < bins - 1 ? b : bins - 1;
    };
    constexpr int VEC = 16 / sizeof(T);                   // elements per 16-byte load
    const int64_t nvec = n / VEC;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec; v += stride) {
        const uint4 w = reinterpret_cast<const uint4 *>(x)[v];
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (sizeof(T) == 4) {
                atomicAdd(&counts[bin(__uint_as_float(u[k]))], 1u);
            } else {
                atomicAdd(&counts[bin(bf16lo(u[k]))], 1u);
                atomicAdd(&counts[bin(bf16hi(u[k]))], 1u);
            }
        }
    }
    for (int64_t e = nvec * VEC + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += stride) {
        const float v = sizeof(T) == 4 ? reinterpret_cast<const float *>(x)[e]
                                       : __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t *>(x)[e]) << 16);
        atomicAdd(&counts[bin(v)], 1u);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < bins; b += blockDim.x)
        if (counts[b]) atomicAdd(&hist[b], static_cast<unsigned long long>(counts[b]));
}

__global__ void k_zero_u64(unsigned long long *p, int n)
{
    pdl_wait();
    pdl_trigger();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = 0ull;
}

// E2M1 magnitude index (0..7) nearest to bin b's centre 6 (2b + 1) / (2i),
// ties to the even code, decided in integers against the midpoints x 8.
__device__ __forceinline__ int e2m1_level_of_bin(int64_t b, int64_t i)
{
    const int64_t num = 24 * (2 * b + 1);
    const int64_t mid8[7] = {2, 6, 10, 14, 20, 28, 40};
    int level = 0;
#pragma unroll
    for (int t = 0; t < 7; ++t) {
        const int64_t rhs = mid8[t] * i;
        if (num > rhs) {
            level = t + 1;
        } else {
            if (num == rhs) level = (t & 1) ? t + 1 : t;   // tie between t and t + 1: the even one
            break;
        }
    }
    return level;
}

__device__ __forceinline__ int kl_level(int b, int i, int levels, int grid)
{
    if (grid) return e2m1_level_of_bin(b, i);
    const int per = i / levels;
    const int l = b / per;
    return l < levels ? l : levels - 1;
}

// KL of candidate i = first + thread index; +inf when Q is zero where P is not.
__global__ void __launch_bounds__(128) k_kl(const unsigned long long *__restrict__ hist, int bins, int levels, int grid,
                                            double *kl)
{
    pdl_wait();
    pdl_trigger();
    const int first = grid ? 8 : levels;
    const int i = first + static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
    if (i > bins) return;
    unsigned long long outliers = 0ull, kept = 0ull;
    for (int b = i; b < bins; ++b) outliers += hist[b];
    for (int b = 0; b < i; ++b) kept += hist[b];
    const double total_p = static_cast<double>(kept + outliers), total_q = static_cast<double>(kept);
    double d = 0.0;
    if (total_p != 0.0) {
        if (total_q == 0.0) {
            d = CUDART_INF;
        } else {
            int b0 = 0;
            while (b0 < i && d != CUDART_INF) {
                const int l = kl_level(b0, i, levels, grid);
                int b1 = b0 + 1;
                while (b1 < i && kl_level(b1, i, levels, grid) == l) ++b1;
                unsigned long long mass = 0ull;
                long long nz = 0;
                for (int b = b0; b < b1; ++b) {
                    mass += hist[b];
                    nz += (hist[b] + (b == i - 1 ? outliers : 0ull)) != 0ull;
                }
                const double qb = nz ? static_cast<double>(mass) / static_cast<double>(nz) : 0.0;
                for (int b = b0; b < b1; ++b) {
                    const double pb = static_cast<double>(hist[b] + (b == i - 1 ? outliers : 0ull));
                    if (pb == 0.0) continue;
                    if (qb == 0.0) {
                        d = CUDART_INF;
                        break;
                    }
                    const double p = pb / total_p, q = qb / total_q;
                    d += p * log(p / q);
                }
                b0 = b1;
            }
        }
    }
    kl[i - first] = d;
}

// least KL (smallest candidate on a tie) -> clip point and winning candidate
__global__ void __launch_bounds__(256) k_kl_pick(const double *kl, int count, int first, int bins, const float *amax_p,
                                                  float *clip, int *best_out)
{
    __shared__ double sv[256];
    __shared__ int si[256];
    pdl_wait();
    pdl_trigger();
    double v = CUDART_INF;
    int idx = count - 1;                                 // all rejected: keep every bin
    for (int k = threadIdx.x; k < count; k += blockDim.x)
        if (kl[k] < v) {
            v = kl[k];
            idx = k;
        }
    sv[threadIdx.x] = v;
    si[threadIdx.x] = idx;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) {
            const double ov = sv[threadIdx.x + s];
            const int oi = si[threadIdx.x + s];
            if (ov < sv[threadIdx.x] || (ov == sv[threadIdx.x] && oi < si[threadIdx.x])) {
                sv[threadIdx.x] = ov;
                si[threadIdx.x] = oi;
            }
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const int i = first + si[0];
        const float w = __fdiv_rn(*amax_p, static_cast<float>(bins));
        *clip = __fmul_rn(static_cast<float>(i), w);
        if (best_out) *best_out = i;
    }
}

struct KlLayout {
    size_t partials, amax, hist, kl, total;
};

static KlLayout kl_layout(int bins, int levels, int grid)
{
    const int first = grid ? 8 : levels;
    auto a256 = [](size_t v) { return (v + 255) & ~size_t(255); };
    KlLayout L;
    L.partials = 0;
    L.amax = a256(sizeof(float) * kMaxPartials);
    L.hist = L.amax + 256;
    L.kl = L.hist + a256(sizeof(unsigned long long) * bins);
    L.total = L.kl + a256(sizeof(double) * (bins - first + 1));
    return L;
}

template <auto Kern, typename... Args>
static int launch_simple(dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args)
{
    if (launch_pdl(Kern, grid, block, smem, stream, args...) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

}  // namespace qfp4

using namespace qfp4;

static int kl_args_ok(int bins, int levels, int grid)
{
    if (grid != 0 && grid != 1) return QFP4_ERR_ARG;
    if (bins < 8 || bins > KL_MAX_BINS) return QFP4_ERR_ARG;
    if (!grid && (levels < 2 || levels > bins)) return QFP4_ERR_ARG;
    return QFP4_OK;
}

extern "C" size_t qfp4_kl_calibrate_workspace_bytes(int bins, int levels, int grid)
{
    if (kl_args_ok(bins, levels, grid) != QFP4_OK) return 0;
    return kl_layout(bins, levels, grid).total;
}

extern "C" int qfp4_kl_calibrate(const void *x, qfp4_dtype xdt, int64_t n, int bins, int levels, int grid,
                                 float *clip_out, int *best_bins_out, double *kl_out, uint64_t *hist_out,
                                 void *workspace, size_t workspace_bytes, qfp4_stream_t stream_)
{
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int st = kl_args_ok(bins, levels, grid);
    if (st != QFP4_OK) return st;
    if (xdt != QFP4_BF16 && xdt != QFP4_F32) return QFP4_ERR_ARG;
    if (n < 0) return QFP4_ERR_SHAPE;
    if (!clip_out || (n > 0 && !x)) return QFP4_ERR_ARG;
    if (!aligned16(x) || !aligned16(workspace) || !aligned16(kl_out) || !aligned16(hist_out)) return QFP4_ERR_ALIGN;
    const KlLayout L = kl_layout(bins, levels, grid);
    if (!workspace || workspace_bytes < L.total) return QFP4_ERR_ARG;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *partials = reinterpret_cast<float *>(ws + L.partials);
    float *amax = reinterpret_cast<float *>(ws + L.amax);
    auto *hist = reinterpret_cast<unsigned long long *>(hist_out ? static_cast<void *>(hist_out) : ws + L.hist);
    double *kl = kl_out ? kl_out : reinterpret_cast<double *>(ws + L.kl);
    const int first = grid ? 8 : levels, count = bins - first + 1;

    int n_parts = 0;
    if (n > 0) {
        st = amax_partials(x, xdt, n, partials, &n_parts, stream);
        if (st != QFP4_OK) return st;
    } else {
        st = launch_simple<k_zero_u64>(dim3(1), dim3(32), 0, stream, reinterpret_cast<unsigned long long *>(partials), 1);
        if (st != QFP4_OK) return st;
        n_parts = 1;                                      // a zero partial: amax 0
    }
    st = partials_max(partials, n_parts, amax, stream);
    if (st != QFP4_OK) return st;
    st = launch_simple<k_zero_u64>(dim3((bins + 255) / 256), dim3(256), 0, stream, hist, bins);
    if (st != QFP4_OK) return st;
    if (n > 0) {
        const int blocks = static_cast<int>(imin<int64_t>((n + 4095) / 4096, 4 * num_sms()));
        const size_t smem = sizeof(uint32_t) * bins;
        st = xdt == QFP4_BF16
                 ? launch_simple<k_abs_hist<uint16_t>>(dim3(blocks), dim3(256), smem, stream,
                                                       static_cast<const uint16_t *>(x), n, bins,
                                                       static_cast<const float *>(amax), hist)
                 : launch_simple<k_abs_hist<float>>(dim3(blocks), dim3(256), smem, stream,
                                                    static_cast<const float *>(x), n, bins,
                                                    static_cast<const float *>(amax), hist);
        if (st != QFP4_OK) return st;
    }
    st = launch_simple<k_kl>(dim3((count + 127) / 128), dim3(128), 0, stream,
                             static_cast<const unsigned long long *>(hist), bins, levels, grid, kl);
    if (st != QFP4_OK) return st;
    return launch_simple<k_kl_pick>(dim3(1), dim3(256), 0, stream, static_cast<const double *>(kl), count, first, bins,
                                    static_cast<const float *>(amax), clip_out, best_bins_out);
}
