// quantize1d.cuh -- interface between the 1D quantize kernels and the C ABI.
#pragma once
#include "qfp4_common.cuh"

namespace qfp4 {

enum { MODE_AMAX = 0, MODE_QUANT = 1 };

// Element format of the 1D kernels besides QFP4_MXFP4 / QFP4_NVFP4: MXFP8
// (E4M3 elements, E8M0 scale per 32), row-wise.
constexpr int FMT_MXFP8 = QFP4_MXFP8;

// Upper bound on the number of partial tensor maxima a pass writes.
constexpr int kMaxPartials = 1024;

struct QuantParams {
    int64_t n;                 // elements of this launch
    uint64_t e_base;           // logical index of its first element
    uint8_t *codes;            // whole-tensor outputs (indexed by logical element)
    uint8_t *scales;
    uint64_t seed;
    const float *partials;     // NVFP4 quantize: partial maxima of the amax pass
    int n_partials;
    float *partials_out;       // amax pass: where this launch writes its partials
    float *tscale_out;         // NVFP4: s_t output
    bool write_tscale;         // this launch's block 0 writes *tscale_out
    int rule;                  // qfp4_scale_rule
    const float *amax_in;      // NVFP4 quantize pass: caller-supplied tensor amax (device), or NULL
};

// Options beyond the defaults: the scale rule, and for NVFP4 a caller-supplied
// tensor amax (device pointer; the tensor scale is fl(amax / 2688)) and where
// to write this tensor's own (rotated) amax.
struct QuantOpts {
    int rule = QFP4_SCALE_DEFAULT;
    const float *amax_in = nullptr;
    float *amax_out = nullptr;
};

int quantize1d(const void *x, qfp4_dtype xdt, int64_t n, qfp4_fmt fmt, qfp4_round rounding, int rotate, int four6,
               uint64_t seed, uint8_t *codes, uint8_t *scales, float *tscale, float *partials, int *n_parts_out,
               cudaStream_t stream, const QuantOpts &opt = QuantOpts{});

// *amax_out = max(partials[0 .. n)) (one block, dependent launch).
int partials_max(const float *partials, int n, float *amax_out, cudaStream_t stream);

// MXFP8 row-wise over a bf16 stream of n elements (n % 64 == 0) through the
// TMA kernel.
int mxfp8_rows(const void *x, int64_t n, bool sr, uint64_t seed, uint8_t *codes, uint8_t *scales,
               cudaStream_t stream);

int amax_partials(const void *x, qfp4_dtype xdt, int64_t n, float *partials, int *n_parts, cudaStream_t stream);

}  // namespace qfp4
