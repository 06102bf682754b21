// runtime.cu -- host runtime of libqfp4: the device error word, the
// tensor-map encoder (driver entry point looked up once, no libcuda link),
// SM counts, status strings.
#include <atomic>
#include <mutex>

#include "qfp4_common.cuh"

namespace qfp4 {



typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode()
{
    static PFN_encodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(p);
    });
    return fn;
}

int encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, int rank, void *gaddr, const uint64_t *dims,
                      const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swizzle)
{
    PFN_encodeTiled enc = get_encode();
    if (!enc) return QFP4_ERR_CUDA;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(map, dtype, static_cast<cuuint32_t>(rank), gaddr, reinterpret_cast<const cuuint64_t *>(dims),
                     reinterpret_cast<const cuuint64_t *>(strides_bytes), reinterpret_cast<const cuuint32_t *>(box),
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QFP4_OK : QFP4_ERR_CUDA;
}

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int num_sms()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace qfp4

extern "C" const char *qfp4_status_string(int status)
{
    switch (status) {
    case QFP4_OK: return "ok";
    case QFP4_ERR_ARG: return "invalid argument (NULL buffer, bad enum value or short workspace)";
    case QFP4_ERR_SHAPE: return "shape violates the call's divisibility or size rules";
    case QFP4_ERR_UNSUPPORTED: return "unsupported option combination";
    case QFP4_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QFP4_ERR_CUDA: return "CUDA launch or driver call failed";
    case QFP4_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    default: return "unknown status";
    }
}

extern "C" int qfp4_last_device_error(void)
{
    int v = 0, zero = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(&v, qfp4::g_dev_error, sizeof v) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(qfp4::g_dev_error, &zero, sizeof zero);
    return v;
}

// One thread waits on an mbarrier that expects an arrival nobody makes, with
// no copy or MMA in flight, so only the bounded wait's give-up path runs.
__global__ void k_wait_timeout(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    qfp4::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    (void)qfp4::mbar_wait_for(&bar, 0, limit_ns);
}

extern "C" int qfp4_selftest_wait_timeout(int64_t limit_us, qfp4_stream_t stream)
{
    if (limit_us < 1 || limit_us > 1000000) return QFP4_ERR_ARG;
    k_wait_timeout<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_us) * 1000u);
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

extern "C" int qfp4_version(void) { return 200; }

extern "C" uint64_t qfp4_launch_count(void) { return qfp4::g_launches.load(std::memory_order_relaxed); }
