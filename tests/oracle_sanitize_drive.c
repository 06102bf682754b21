/* Drives every oracle entry point over small and ragged shapes and every
 * option combination (invalid ones included, which must return an error
 * without touching the buffers), with output buffers of the exact sizes the
 * header states.  Built with AddressSanitizer and UndefinedBehaviorSanitizer
 * by tests/test_oracle_sanitized.py, so an out-of-bounds access or undefined
 * arithmetic in the oracle stops the run.  Prints the number of calls that
 * returned OR_OK. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include "qfp4_oracle.h"

static uint16_t to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

static void *buf(int64_t n) { return malloc(n > 0 ? (size_t)n : 1); }

int main(void)
{
    static const int64_t shapes[][2] = {{1, 16}, {1, 32}, {3, 128}, {16, 16}, {32, 32},
                                        {48, 64}, {37, 384}, {64, 256}, {5, 48}};
    long ok = 0;
    srand(1);
    for (size_t s = 0; s < sizeof shapes / sizeof shapes[0]; ++s) {
        const int64_t M = shapes[s][0], K = shapes[s][1], n = M * K;
        uint16_t *xb = buf(2 * n);
        float *xf = buf(4 * n);
        for (int64_t i = 0; i < n; ++i) {
            xf[i] = (float)((rand() / (double)RAND_MAX - 0.5) * 8.0);
            xb[i] = to_bf16(xf[i]);
        }
        for (int opt = 0; opt < 128; ++opt) {
            const int fmt = opt & 1, rnd = (opt >> 1) & 1, rot = (opt >> 2) & 1, b2 = (opt >> 3) & 1,
                      f6 = (opt >> 4) & 1, tr = (opt >> 5) & 1, dt = (opt >> 6) & 1;
            const int g = fmt == OR_MXFP4 ? 32 : 16;
            uint8_t *c = buf(n / 2), *sc = buf(n / g), *cT = tr ? buf(n / 2) : NULL, *sT = tr ? buf(n / g) : NULL;
            float ts = 0.0f;
            ok += or_quantize(dt ? (const void *)xf : (const void *)xb, dt, M, K, fmt, rnd, rot, b2, f6, 7, c, sc, cT,
                              sT, &ts) == OR_OK;
            free(c); free(sc); free(cT); free(sT);
        }
        for (int opt = 0; opt < 4; ++opt) {
            const int rnd = opt & 1, tr = opt >> 1;
            uint8_t *c = buf(n), *sc = buf(n / 32), *cT = tr ? buf(n) : NULL, *sT = tr ? buf(n / 32) : NULL;
            ok += or_quantize_mxfp8(xb, OR_BF16, M, K, rnd, 3, c, sc, cT, sT) == OR_OK;
            free(c); free(sc); free(cT); free(sT);
        }
        for (int gran = 0; gran < 4; ++gran) {
            const int64_t ns = gran == OR_GRAN_TENSOR ? 1 : gran == OR_GRAN_ROW ? M : n / (gran == OR_GRAN_GROUP16 ? 16 : 32);
            uint8_t *c = buf(n / 2);
            float *sc = buf(4 * ns);
            ok += or_quantize_fp32scale(xb, OR_BF16, M, K, gran, c, sc) == OR_OK;
            free(c); free(sc);
        }
        if (K % 32 == 0) {
            for (int fmt = 0; fmt < 3; ++fmt) {
                const int g = fmt == OR_NVFP4 ? 16 : 32;
                const int64_t cb = fmt == OR_MXFP8 ? n : n / 2, no = M * M;
                uint8_t *c = buf(cb), *sc = buf(n / g);
                for (int64_t i = 0; i < cb; ++i) c[i] = (uint8_t)(fmt == OR_MXFP8 ? (rand() & 0x7E) : rand());
                for (int64_t i = 0; i < n / g; ++i)
                    sc[i] = (uint8_t)(fmt == OR_NVFP4 ? (rand() & 0x7E) : 120 + rand() % 10);
                const float t = 0.01f;
                int64_t *r = buf(8 * no), *cc = buf(8 * no);
                for (int64_t i = 0; i < no; ++i) {
                    r[i] = i / M;
                    cc[i] = i % M;
                }
                double *o = buf(8 * no), *mag = buf(8 * no), *dq = buf(8 * n);
                ok += or_gemm_sampled(c, sc, &t, c, sc, &t, M, M, K, fmt, r, cc, no, o, mag) == OR_OK;
                ok += (fmt == OR_MXFP8 ? or_dequantize_mxfp8(c, sc, M, K, dq)
                                       : or_dequantize(c, sc, &t, M, K, fmt, dq)) == OR_OK;
                free(c); free(sc); free(r); free(cc); free(o); free(mag); free(dq);
            }
        }
        free(xb);
        free(xf);
    }
    for (int bins = 8; bins <= 2048; bins *= 4) {
        uint64_t *h = buf(8 * bins);
        uint16_t xs[1000];
        for (int i = 0; i < 1000; ++i) xs[i] = to_bf16((float)(rand() % 1000) / 100.0f);
        ok += or_abs_histogram(xs, OR_BF16, 1000, bins, 9.99f, h) == OR_OK;
        for (int grid = 0; grid < 2; ++grid) {
            const int first = grid ? 8 : 4;
            int best = 0;
            double *kl = buf(8 * (bins - first + 1));
            ok += or_kl_calibrate(h, bins, 4, grid, kl, &best) == OR_OK;
            free(kl);
        }
        free(h);
    }
    printf("%ld\n", ok);
    return 0;
}
