// pending.cu -- entry points whose kernels are not built yet.
#include "qfp4_common.cuh"

namespace qfp4 {
}  // namespace qfp4
