// libqfp4.cu -- single translation unit of the library (so the device-side
// error word and the inline helpers need no relocatable device code).
#include "runtime.cu"
#include "quantize1d.cu"
#include "dequant_fp32scale.cu"
#include "quantize2d.cu"
#include "gemm.cu"
#include "api.cu"
#include "gemm_noalloc.cu"
#include "linear.cu"
#include "calib.cu"
