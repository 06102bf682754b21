// pending.cu -- entry points whose kernels are not built yet.
#include "qfp4_common.cuh"

namespace qfp4 {
int quantize_columns(const void *, qfp4_dtype, int64_t, int64_t, qfp4_fmt, qfp4_round, int, uint64_t, uint8_t *,
                     uint8_t *, const float *, int, cudaStream_t)
{
    return QFP4_ERR_UNSUPPORTED;
}
int quantize2d(const void *, qfp4_dtype, int64_t, int64_t, qfp4_round, uint64_t, uint8_t *, uint8_t *, uint8_t *,
               uint8_t *, float *, float *, cudaStream_t)
{
    return QFP4_ERR_UNSUPPORTED;
}
int quantize_mxfp8(const void *, qfp4_dtype, int64_t, int64_t, qfp4_round, uint64_t, uint8_t *, uint8_t *, uint8_t *,
                   uint8_t *, cudaStream_t)
{
    return QFP4_ERR_UNSUPPORTED;
}
}  // namespace qfp4
