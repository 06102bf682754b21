// gemm_noalloc.cu -- qfp4_gemm_blockscaled_noalloc: the block-scaled FP4 GEMM
// for callers that cannot allocate device memory.
//
// Who needs it: code that runs where no allocator may be called -- inside a
// framework's custom-op or plugin hook that forbids allocation while it is
// enqueuing work, in real-time or embedded loops that must not touch the
// allocator after start-up, or in libraries that are handed only input and
// output buffers and no workspace.  qfp4_gemm_blockscaled needs a caller-given
// workspace for the rearranged scales; this entry point instead uses one
// fixed scratch array compiled into the library.
//
// The scratch is a file-scope device array of kNoallocScratchBytes (16 MiB).
// Every GPU on which the library's kernels are loaded keeps those 16 MiB
// until the process exits.  Its device address is looked up once per device
// (cudaGetSymbolAddress with that device current) on the first call made on
// that device; make that first call before any stream capture.  All calls
// share the one array and it keeps the last call's contents: nothing in it has
// to start at zero (the scale prepass rewrites every byte the GEMM reads), but
// two calls whose work overlaps on the GPU -- on different streams without
// ordering between them -- race on it.
#include <mutex>

#include "qfp4_common.cuh"

namespace qfp4 {

constexpr size_t kNoallocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

size_t gemm_workspace(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt);

// Device address of the scratch array on the current device, looked up once
// per device.  Returns nullptr when the lookup fails.
static void *noalloc_scratch_ptr()
{
    constexpr int kMaxDevices = 64;
    static void *ptrs[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        ptrs[dev] = p;
    }
    return ptrs[dev];
}

}  // namespace qfp4

extern "C" int qfp4_gemm_blockscaled_noalloc(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale,
                                             const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale,
                                             int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, qfp4_dtype out_dt,
                                             void *out, qfp4_stream_t stream)
{
    using namespace qfp4;
    // The checks qfp4_gemm_blockscaled makes first (enums, then shape rules
    // including M, N, K < 2^30), so the scratch size below cannot overflow and
    // an invalid call gets the same status from both entry points.
    if (fmt != QFP4_MXFP4 && fmt != QFP4_NVFP4 && fmt != QFP4_MXFP8) return QFP4_ERR_ARG;
    if (out_dt != QFP4_BF16 && out_dt != QFP4_F32) return QFP4_ERR_ARG;
    const int shape = gemm_shape_check(M, N, K, out_dt);
    if (shape != QFP4_OK) return shape;
    if (M * N > 0 && K > 0 && gemm_workspace(M, N, K, fmt) > kNoallocScratchBytes) return QFP4_ERR_SHAPE;
    void *scratch = noalloc_scratch_ptr();
    if (!scratch) return QFP4_ERR_CUDA;
    // Same validation and kernels as qfp4_gemm_blockscaled, with the built-in
    // scratch in place of a caller's workspace.
    return qfp4_gemm_blockscaled(A_codes, A_scales, A_tscale, B_codes, B_scales, B_tscale, M, N, K, fmt, out_dt, out,
                                 scratch, kNoallocScratchBytes, stream);
}
