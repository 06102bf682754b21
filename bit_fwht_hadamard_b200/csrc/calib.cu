// calib.cu -- KL-divergence clip calibration of an activation tensor ([LB]
// §5, the TensorRT method: for each candidate clip point T, P = the
// histogram of |x| cut at T with the tail counted in the last kept bin, Q =
// the kept histogram quantized to the levels and spread back over P's bins;
// the T with the least D_KL(P || Q) loses the least information).
//
// Four launches after the tensor-amax pass: a histogram of |x| over [0,
// amax] privatized in shared memory; prefix sums of the histogram and of its
// nonzero bins; one warp per candidate computing its KL (the level of a bin
// never decreases with the bin, so a level's bins are one contiguous run
// whose kept mass and nonzero count are two prefix lookups; the lanes form
// the terms of 32 bins at a time and one lane adds them in ascending bin
// order); one block taking the least KL (smallest candidate on a tie) and
// writing the clip point T = fl(i * fl(amax / bins)).
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

// Prefix sums of the histogram and of its count of nonzero bins, so that a
// level's kept mass and nonzero count are two lookups: ph[b] = sum of
// hist[0 .. b), pnz[b] = number of nonzero bins in [0, b), b = 0 .. bins.
// One block of 1024 threads, each summing 8 consecutive bins (bins <= 8192).
__global__ void __launch_bounds__(1024) k_hist_prefix(const unsigned long long *__restrict__ hist, int bins,
                                                      unsigned long long *ph, int *pnz)
{
    __shared__ unsigned long long sh[1024];
    __shared__ int sn[1024];
    pdl_wait();
    pdl_trigger();
    const int t = threadIdx.x, b0 = 8 * t;
    unsigned long long h = 0ull;
    int c = 0;
    for (int b = b0; b < b0 + 8 && b < bins; ++b) {
        h += hist[b];
        c += hist[b] != 0ull;
    }
    sh[t] = h;
    sn[t] = c;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {          // inclusive scan of the per-thread sums
        const unsigned long long hv = t >= off ? sh[t - off] : 0ull;
        const int cv = t >= off ? sn[t - off] : 0;
        __syncthreads();
        sh[t] += hv;
        sn[t] += cv;
        __syncthreads();
    }
    unsigned long long run = t ? sh[t - 1] : 0ull;        // exclusive prefix of this thread's first bin
    int runc = t ? sn[t - 1] : 0;
    for (int b = b0; b < b0 + 8 && b < bins; ++b) {
        ph[b] = run;
        pnz[b] = runc;
        run += hist[b];
        runc += hist[b] != 0ull;
    }
    if (t == 1023) {                                      // the totals
        ph[bins] = sh[1023];
        pnz[bins] = sn[1023];
    }
}

// KL of candidate i, one warp per candidate; +inf when Q is zero where P is
// not.  The level runs of candidate i are contiguous: uniform levels from
// per = floor(i / levels), the E2M1 ones from the smallest bin of each level
// (a binary search on e2m1_level_of_bin, which is monotone in the bin), so a
// level's kept mass and nonzero count come from the prefix sums (the last
// kept bin also holds the tail beyond i, which can make it nonzero).  The
// lanes compute the terms p log(p / q) of 32 consecutive bins; lane 0 adds
// them in ascending bin order, the order of the plain loop.
__global__ void __launch_bounds__(256) k_kl(const unsigned long long *__restrict__ hist,
                                            const unsigned long long *__restrict__ ph, const int *__restrict__ pnz,
                                            int bins, int levels, int grid, double *kl)
{
    __shared__ double terms[8][32];
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int first = grid ? 8 : levels;
    const int i = first + static_cast<int>(blockIdx.x) * 8 + warp;
    if (i > bins) return;                                 // the whole warp
    const unsigned long long kept = ph[i], outliers = ph[bins] - ph[i];
    const double total_p = static_cast<double>(kept + outliers), total_q = static_cast<double>(kept);
    // E2M1 run starts: start[l] = smallest bin of level >= l (start[0] = 0, start[8] = i)
    int bound = i;
    if (grid && lane < 7) {                               // lane t: smallest b with level(b) >= t + 1
        int lo = 0, hi = i;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (e2m1_level_of_bin(mid, i) >= lane + 1) hi = mid;
            else lo = mid + 1;
        }
        bound = lo;
    }
    int start[9];
    start[0] = 0;
#pragma unroll
    for (int t = 0; t < 7; ++t) start[t + 1] = __shfl_sync(0xFFFFFFFFu, bound, t);
    start[8] = i;
    const int per = grid ? 1 : i / levels;
    double d = 0.0;
    if (total_p != 0.0) {
        if (total_q == 0.0) {
            d = CUDART_INF;
        } else {
            for (int c0 = 0; c0 < i; c0 += 32) {
                const int b = c0 + lane;
                double term = 0.0;
                if (b < i) {
                    const unsigned long long pb_u = hist[b] + (b == i - 1 ? outliers : 0ull);
                    if (pb_u != 0ull) {
                        int b0, b1;
                        if (grid) {
                            const int l = e2m1_level_of_bin(b, i);
                            b0 = 0;
                            b1 = i;
#pragma unroll
                            for (int t = 0; t < 8; ++t)
                                if (t == l) {
                                    b0 = start[t];
                                    b1 = start[t + 1];
                                }
                        } else {
                            const int l = imin(b / per, levels - 1);
                            b0 = l * per;
                            b1 = l == levels - 1 ? i : b0 + per;
                        }
                        const unsigned long long mass = ph[b1] - ph[b0];
                        long long nz = pnz[b1] - pnz[b0];
                        if (b1 == i && hist[i - 1] == 0ull && outliers != 0ull) ++nz;   // the tail makes bin i - 1 nonzero
                        const double qb = nz ? static_cast<double>(mass) / static_cast<double>(nz) : 0.0;
                        if (qb == 0.0) {
                            term = CUDART_INF;
                        } else {
                            const double pp = static_cast<double>(pb_u) / total_p, qq = qb / total_q;
                            term = pp * log(pp / qq);
                        }
                    }
                }
                terms[warp][lane] = term;
                __syncwarp();
                if (lane == 0)
#pragma unroll 8
                    for (int k = 0; k < 32; ++k) d += terms[warp][k];
                __syncwarp();
            }
        }
    }
    if (lane == 0) kl[i - first] = d;
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
    size_t partials, amax, hist, kl, ph, pnz, total;
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
    L.ph = L.kl + a256(sizeof(double) * (bins - first + 1));
    L.pnz = L.ph + a256(sizeof(unsigned long long) * (bins + 1));
    L.total = L.pnz + a256(sizeof(int) * (bins + 1));
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
    if (n < 0 || n > (int64_t(1) << 38)) return QFP4_ERR_SHAPE;   // the library's element limit
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
    auto *ph = reinterpret_cast<unsigned long long *>(ws + L.ph);
    int *pnz = reinterpret_cast<int *>(ws + L.pnz);
    st = launch_simple<k_hist_prefix>(dim3(1), dim3(1024), 0, stream, static_cast<const unsigned long long *>(hist),
                                      bins, ph, pnz);
    if (st != QFP4_OK) return st;
    st = launch_simple<k_kl>(dim3((count + 7) / 8), dim3(256), 0, stream, static_cast<const unsigned long long *>(hist),
                             static_cast<const unsigned long long *>(ph), static_cast<const int *>(pnz), bins, levels,
                             grid, kl);
    if (st != QFP4_OK) return st;
    return launch_simple<k_kl_pick>(dim3(1), dim3(256), 0, stream, static_cast<const double *>(kl), count, first, bins,
                                    static_cast<const float *>(amax), clip_out, best_bins_out);
}
