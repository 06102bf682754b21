// gemm.cu -- block-scaled FP4 GEMM on 5th-generation tensor cores:
// Y[m][n] = sum_k deqA[m][k] deqB[n][k]  (A: M x K, B: N x K, both K-major
// packed E2M1 codes with row-major scales as qfp4_quantize writes them).
//
// Method: [QN] §QuTLASS (MXFP4 / NVFP4 operands, FP32 accumulation);
// [LB] §FP4 (Blackwell FP4 tensor cores).  Hardware path (sm_100a):
//   * tcgen05.mma.cta_group::1 kind::mxf4 (E8M0 scale per 32, MXFP4) or
//     kind::mxf4nvf4 (E4M3 scale per 16, NVFP4), M=128 x N=256 x K=64 per
//     instruction, fp32 accumulators in tensor memory (TMEM);
//   * operands staged in shared memory by TMA (128-byte swizzle, no
//     multicast), scale factors staged by 1D bulk copies and moved to TMEM
//     with tcgen05.cp (32x128b, replicated to the four lane quadrants);
//   * persistent, warp-specialised CTA: warp 0 produces (TMA), warp 1
//     issues MMAs (one elected lane), warps 2-9 drain the accumulator
//     (tcgen05.ld) and store; the accumulator is released as soon as the
//     tile is in registers, so the next tile's MMAs overlap the stores.
// The row-major scales are first rearranged by a small prepass into
// 512-byte chunks in the tcgen05.cp source layout (128 rows x 4 scales:
// byte (r%32)*16 + (r/32)*4 + j), so the main loop loads them with plain
// contiguous bulk copies; the chunks live in the caller's workspace.
#include "qfp4_common.cuh"
#include "quantize1d.cuh"

namespace qfp4 {

constexpr int GM_BM = 128, GM_BN = 256, GM_BK = 256;      // tile (elements)
constexpr int GM_BKB = GM_BK / 2;                         // bytes of one row per stage
constexpr int GM_STAGES = 4;
constexpr int GM_A_BYTES = GM_BM * GM_BKB;                // 16 KiB
constexpr int GM_B_BYTES = GM_BN * GM_BKB;                // 32 KiB
constexpr int GM_SFA_BYTES = 4 * 512;                     // up to 4 chunks (NVFP4)
constexpr int GM_SFB_BYTES = 8 * 512;                     // 2 row blocks x 4 chunks
constexpr int GM_STAGE_BYTES = GM_A_BYTES + GM_B_BYTES + GM_SFA_BYTES + GM_SFB_BYTES;
constexpr int GM_SMEM = GM_STAGES * GM_STAGE_BYTES + 1024;
constexpr int GM_EPI_WARPS = 8;
constexpr int GM_THREADS = 32 * (2 + GM_EPI_WARPS);
constexpr uint32_t GM_TMEM_COLS = 512;
constexpr uint32_t GM_SF_COL = 256;                       // scale factors after the accumulator
constexpr int GM_GROUP_M = 8;                             // tile raster: 8 m-blocks per band

// chunks of 4 scale groups per stage and 128-row block
__host__ __device__ constexpr int gm_cps(int fmt) { return fmt == QFP4_NVFP4 ? 4 : 2; }

struct GemmParams {
    int M, N, K;
    int KT;                 // k tiles of 256
    int tiles_m, tiles_n;
    int NC;                 // scale chunks per 128-row block (KT * cps)
    const uint8_t *sfa;     // rearranged scales (workspace)
    const uint8_t *sfb;
    const float *tA, *tB;   // NVFP4 tensor scales
    void *out;
};

// ------------------------------------------------------------------ PTX: tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// arrive on `bar` once every tcgen05 operation issued so far by this thread completes
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// shared -> tensor memory: 32 rows x 128 bits, replicated into all four lane quadrants
__device__ __forceinline__ void utccp_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

template <int FMT>
__device__ __forceinline__ void umma_blockscaled(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                                 uint32_t sfb, uint32_t accumulate)
{
    if (FMT == QFP4_NVFP4)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
}

// 32 lanes x 32 consecutive fp32 columns (lane quadrant of the calling warp)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// 16 lanes x 128 consecutive fp32 columns (16x256b shape, 16 repetitions):
// thread t gets, for repetition j, columns 8j + 2(t%4) + {0,1} of lane
// base + t/4 (r[4j], r[4j+1]) and of lane base + 8 + t/4 (r[4j+2], r[4j+3]).
__device__ __forceinline__ void tmem_ld16x256b_x16(uint32_t taddr, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,"
        "%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
          "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
          "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
          "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
          "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Ties registers filled by tcgen05.ld to a point after tcgen05.wait::ld, so
// no use of them can be scheduled before the wait.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t *r)
{
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// 1D bulk copy global -> shared, completing on an mbarrier
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128 B,
// 8-row groups 1024 B apart (SBO), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t desc_k_sw128(const void *p)
{
    return static_cast<uint64_t>((smem_u32(p) >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Source descriptor of a scale chunk for tcgen05.cp: 32 rows of 16 B,
// no swizzle, 8-row core matrices 128 B apart.
__device__ __forceinline__ uint64_t desc_sf_chunk(const void *p)
{
    return static_cast<uint64_t>((smem_u32(p) >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128 >> 4) << 32) |
           (static_cast<uint64_t>(1) << 46);
}

// Instruction descriptor of the block-scaled MMA: E2M1 A and B, K-major,
// N >> 3 at bit 17, scale format (0 = UE4M3, 1 = UE8M0) at bit 23,
// M >> 4 at bit 24, scale-factor byte selectors at bits 4 (B) and 29 (A).
__host__ __device__ constexpr uint32_t idesc_blockscaled(int fmt, int M, int N, uint32_t sf_id)
{
    return (sf_id << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           ((fmt == QFP4_NVFP4 ? 0u : 1u) << 23) | (static_cast<uint32_t>(M >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int &mb, int &nb)
{
    const int per_group = GM_GROUP_M * tiles_n;
    const int group = t / per_group;
    const int first_m = group * GM_GROUP_M;
    const int gm = min(tiles_m - first_m, GM_GROUP_M);
    const int r = t - group * per_group;
    mb = first_m + r % gm;
    nb = r / gm;
}

// ------------------------------------------------------------------ scale prepass
// One thread per 16-byte line of a chunk: rows rb*128 + r0 + 32*rr (rr = 0..3),
// scale groups c*4 + j (j = 0..3); zero beyond R rows or Kg groups.
__global__ void __launch_bounds__(256) k_sf_rearrange(const uint8_t *__restrict__ sc, int R, int Kg, int NC,
                                                      int n_lines, uint8_t *__restrict__ dst)
{
    const int line = blockIdx.x * blockDim.x + threadIdx.x;
    if (line >= n_lines) return;
    const int r0 = line & 31;
    const int chunk = line >> 5;
    const int c = chunk % NC, rb = chunk / NC;
    uint32_t w[4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int row = rb * 128 + r0 + 32 * rr;
        uint32_t v = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int grp = c * 4 + j;
            const uint32_t b = (row < R && grp < Kg) ? sc[static_cast<int64_t>(row) * Kg + grp] : 0u;
            v |= b << (8 * j);
        }
        w[rr] = v;
    }
    *reinterpret_cast<uint4 *>(dst + static_cast<int64_t>(line) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
}

// ------------------------------------------------------------------ main kernel
template <int FMT, int OUT>
__global__ void __launch_bounds__(GM_THREADS, 1)
    k_gemm_blockscaled(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[GM_STAGES], empty[GM_STAGES], acc_full, acc_empty;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_flag;

    constexpr int CPS = gm_cps(FMT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = p.tiles_m * p.tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < GM_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, GM_EPI_WARPS);
        abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, GM_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    auto stage_a = [&](int s) { return smem + s * GM_STAGE_BYTES; };
    auto stage_b = [&](int s) { return smem + s * GM_STAGE_BYTES + GM_A_BYTES; };
    auto stage_sfa = [&](int s) { return smem + s * GM_STAGE_BYTES + GM_A_BYTES + GM_B_BYTES; };
    auto stage_sfb = [&](int s) { return smem + s * GM_STAGE_BYTES + GM_A_BYTES + GM_B_BYTES + GM_SFA_BYTES; };

    if (warp == 0) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            const uint32_t bytes = GM_A_BYTES + GM_B_BYTES + 3 * CPS * 512;
            int it = 0;
            for (int t = blockIdx.x; t < ntiles && !abort_flag; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p.tiles_m, p.tiles_n, mb, nb);
                for (int kt = 0; kt < p.KT; ++kt, ++it) {
                    const int s = it % GM_STAGES;
                    const uint32_t ph = (it / GM_STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u)) { abort_flag = 1; break; }
                    mbar_arrive_expect_tx(&full[s], bytes);
                    tma_load_2d(stage_a(s), &tmA, &full[s], kt * GM_BKB, mb * GM_BM);
                    tma_load_2d(stage_b(s), &tmB, &full[s], kt * GM_BKB, nb * GM_BN);
                    const int64_t ca = (static_cast<int64_t>(mb) * p.NC + kt * CPS) * 512;
                    const int64_t cb0 = (static_cast<int64_t>(2 * nb) * p.NC + kt * CPS) * 512;
                    const int64_t cb1 = (static_cast<int64_t>(2 * nb + 1) * p.NC + kt * CPS) * 512;
                    bulk_g2s(stage_sfa(s), p.sfa + ca, CPS * 512, &full[s]);
                    bulk_g2s(stage_sfb(s), p.sfb + cb0, CPS * 512, &full[s]);
                    bulk_g2s(stage_sfb(s) + CPS * 512, p.sfb + cb1, CPS * 512, &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, ti = 0;
            for (int t = blockIdx.x; t < ntiles && !abort_flag; t += gridDim.x, ++ti) {
                if (!mbar_wait(&acc_empty, (ti & 1) ^ 1u)) { abort_flag = 1; break; }
                tc_fence_after();
                for (int kt = 0; kt < p.KT; ++kt, ++it) {
                    const int s = it % GM_STAGES;
                    const uint32_t ph = (it / GM_STAGES) & 1u;
                    if (!mbar_wait(&full[s], ph)) { abort_flag = 1; break; }
                    tc_fence_after();
                    const uint32_t sfa_col = tmem + GM_SF_COL + (it & 1) * 48;
                    const uint32_t sfb_col = sfa_col + 16;
#pragma unroll
                    for (int j = 0; j < CPS; ++j) utccp_sf(sfa_col + 4 * j, desc_sf_chunk(stage_sfa(s) + 512 * j));
#pragma unroll
                    for (int b = 0; b < 2; ++b)
#pragma unroll
                        for (int j = 0; j < CPS; ++j)
                            utccp_sf(sfb_col + 8 * j + 4 * b, desc_sf_chunk(stage_sfb(s) + 512 * (b * CPS + j)));
                    const uint64_t adesc = desc_k_sw128(stage_a(s));
                    const uint64_t bdesc = desc_k_sw128(stage_b(s));
#pragma unroll
                    for (int k = 0; k < GM_BK / 64; ++k) {
                        uint32_t sfa, sfb, id;
                        if (FMT == QFP4_NVFP4) {
                            sfa = sfa_col + 4 * k;
                            sfb = sfb_col + 8 * k;
                            id = idesc_blockscaled(FMT, GM_BM, GM_BN, 0);
                        } else {
                            const uint32_t sel = 2u * (k & 1);
                            sfa = (sfa_col + 4 * (k >> 1)) | (sel << 30);
                            sfb = (sfb_col + 8 * (k >> 1)) | (sel << 30);
                            id = idesc_blockscaled(FMT, GM_BM, GM_BN, sel);
                        }
                        umma_blockscaled<FMT>(tmem, adesc + 2 * k, bdesc + 2 * k, id, sfa, sfb, (kt | k) != 0);
                    }
                    umma_commit(&empty[s]);
                }
                umma_commit(&acc_full);
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                   // TMEM lane quadrant of this warp
        const int h = (warp - 2) >> 2;            // column half
        float alpha = 1.0f;
        if (FMT == QFP4_NVFP4) alpha = __fmul_rn(*p.tA, *p.tB);
        int ti = 0;
        for (int t = blockIdx.x; t < ntiles && !abort_flag; t += gridDim.x, ++ti) {
            int mb, nb;
            tile_coords(t, p.tiles_m, p.tiles_n, mb, nb);
            if (!mbar_wait(&acc_full, ti & 1)) { abort_flag = 1; break; }
            tc_fence_after();
            // two 16-lane halves of this warp's quadrant, 128 columns each
            uint32_t r[128];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                tmem_ld16x256b_x16(tmem + (static_cast<uint32_t>(32 * q + 16 * hh) << 16) + 128 * h, r + 64 * hh);
            tmem_ld_wait();
            reg_fence<128>(r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty);

            // r[64hh + 4j + {0,1}]: row 32q + 16hh + lane/4, columns 8j + 2(lane%4) + {0,1};
            // r[64hh + 4j + {2,3}]: the row 8 below.  Four lanes cover 32 contiguous bytes.
            const int col0 = nb * GM_BN + 128 * h + 2 * (lane & 3);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int row = mb * GM_BM + 32 * q + 16 * hh + 8 * e + (lane >> 2);
                    if (row >= p.M) continue;
                    if (OUT == QFP4_F32) {
                        float *o = static_cast<float *>(p.out) + static_cast<int64_t>(row) * p.N + col0;
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (col0 + 8 * j < p.N)
                                *reinterpret_cast<float2 *>(o + 8 * j) =
                                    make_float2(__fmul_rn(__uint_as_float(r[64 * hh + 4 * j + 2 * e]), alpha),
                                                __fmul_rn(__uint_as_float(r[64 * hh + 4 * j + 2 * e + 1]), alpha));
                    } else {
                        uint16_t *o = static_cast<uint16_t *>(p.out) + static_cast<int64_t>(row) * p.N + col0;
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (col0 + 8 * j < p.N) {
                                const __nv_bfloat162 b2 =
                                    __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[64 * hh + 4 * j + 2 * e]), alpha),
                                                          __fmul_rn(__uint_as_float(r[64 * hh + 4 * j + 2 * e + 1]), alpha));
                                *reinterpret_cast<__nv_bfloat162 *>(o + 8 * j) = b2;
                            }
                    }
                }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, GM_TMEM_COLS);
}

// ------------------------------------------------------------------ host
struct GemmLayout {
    int MB, NT, KT, NC;
    size_t sfa_bytes, sfb_bytes;
};

static GemmLayout gemm_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    GemmLayout L;
    L.MB = static_cast<int>((M + GM_BM - 1) / GM_BM);
    L.NT = static_cast<int>((N + GM_BN - 1) / GM_BN);
    L.KT = static_cast<int>((K + GM_BK - 1) / GM_BK);
    L.NC = L.KT * gm_cps(fmt);
    L.sfa_bytes = static_cast<size_t>(L.MB) * L.NC * 512;
    L.sfb_bytes = static_cast<size_t>(2 * L.NT) * L.NC * 512;
    return L;
}

size_t gemm_workspace(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    const GemmLayout L = gemm_layout(M, N, K, fmt);
    return L.sfa_bytes + L.sfb_bytes;
}

int rearrange_scales(const uint8_t *scales, int64_t R, int64_t K, qfp4_fmt fmt, int n_blocks128, int NC, uint8_t *dst,
                     cudaStream_t stream)
{
    const int g = fmt == QFP4_MXFP4 ? 32 : 16;
    const int n_lines = n_blocks128 * NC * 32;
    k_sf_rearrange<<<(n_lines + 255) / 256, 256, 0, stream>>>(scales, static_cast<int>(R), static_cast<int>(K / g), NC,
                                                             n_lines, dst);
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

template <int FMT, int OUT>
static int launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p, int grid, cudaStream_t s)
{
    static bool configured = false;
    auto kern = k_gemm_blockscaled<FMT, OUT>;
    if (!configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GM_SMEM) != cudaSuccess)
            return QFP4_ERR_CUDA;
        configured = true;
    }
    kern<<<grid, GM_THREADS, GM_SMEM, s>>>(ta, tb, p);
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

// Main kernel on already rearranged scales (sfa / sfb in the chunk layout).
int gemm_core(const uint8_t *A_codes, const uint8_t *sfa, const float *A_tscale, const uint8_t *B_codes,
              const uint8_t *sfb, const float *B_tscale, int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
              qfp4_dtype out_dt, void *out, cudaStream_t stream)
{
    const GemmLayout L = gemm_layout(M, N, K, fmt);
    CUtensorMap ta, tb;
    {
        const uint64_t dims[2] = {static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M)};
        const uint64_t strides[1] = {static_cast<uint64_t>(K / 2)};
        const uint32_t box[2] = {GM_BKB, GM_BM};
        int st = encode_tensor_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(A_codes), dims,
                                   strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != QFP4_OK) return st;
    }
    {
        const uint64_t dims[2] = {static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N)};
        const uint64_t strides[1] = {static_cast<uint64_t>(K / 2)};
        const uint32_t box[2] = {GM_BKB, GM_BN};
        int st = encode_tensor_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(B_codes), dims,
                                   strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != QFP4_OK) return st;
    }
    GemmParams p;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.KT = L.KT;
    p.tiles_m = L.MB;
    p.tiles_n = L.NT;
    p.NC = L.NC;
    p.sfa = sfa;
    p.sfb = sfb;
    p.tA = A_tscale;
    p.tB = B_tscale;
    p.out = out;
    const int grid = static_cast<int>(imin<int64_t>(static_cast<int64_t>(L.MB) * L.NT, num_sms()));
    if (fmt == QFP4_NVFP4)
        return out_dt == QFP4_F32 ? launch_gemm<QFP4_NVFP4, QFP4_F32>(ta, tb, p, grid, stream)
                                  : launch_gemm<QFP4_NVFP4, QFP4_BF16>(ta, tb, p, grid, stream);
    return out_dt == QFP4_F32 ? launch_gemm<QFP4_MXFP4, QFP4_F32>(ta, tb, p, grid, stream)
                              : launch_gemm<QFP4_MXFP4, QFP4_BF16>(ta, tb, p, grid, stream);
}

int gemm_blockscaled(const uint8_t *A_codes, const uint8_t *A_scales, const float *A_tscale, const uint8_t *B_codes,
                     const uint8_t *B_scales, const float *B_tscale, int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
                     qfp4_dtype out_dt, void *out, void *workspace, cudaStream_t stream)
{
    const GemmLayout L = gemm_layout(M, N, K, fmt);
    uint8_t *sfa = static_cast<uint8_t *>(workspace);
    uint8_t *sfb = sfa + L.sfa_bytes;
    int st = rearrange_scales(A_scales, M, K, fmt, L.MB, L.NC, sfa, stream);
    if (st != QFP4_OK) return st;
    st = rearrange_scales(B_scales, N, K, fmt, 2 * L.NT, L.NC, sfb, stream);
    if (st != QFP4_OK) return st;
    return gemm_core(A_codes, sfa, A_tscale, B_codes, sfb, B_tscale, M, N, K, fmt, out_dt, out, stream);
}

// ------------------------------------------------------------------ fused rotate + quantize + GEMM
// Workspace: quantized A (codes M*K/2, row-major scales M*K/g), its tensor
// scale, the partial maxima of the amax pass, then the scale chunks of A and B.
struct FusedLayout {
    size_t codes, scales, tscale, partials, chunks, total;
};

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

static FusedLayout fused_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    const int g = fmt == QFP4_MXFP4 ? 32 : 16;
    FusedLayout L;
    L.codes = 0;
    L.scales = align256(static_cast<size_t>(M) * K / 2);
    L.tscale = L.scales + align256(static_cast<size_t>(M) * K / g);
    L.partials = L.tscale + 256;
    L.chunks = L.partials + align256(sizeof(float) * kMaxPartials);
    L.total = L.chunks + align256(gemm_workspace(M, N, K, fmt));
    return L;
}

size_t gemm_fused_rq_workspace(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return fused_layout(M, N, K, fmt).total;
}

int gemm_fused_rq(const void *A_bf16, int64_t M, int64_t K, int rotate, int four6, qfp4_fmt fmt,
                  const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale, int64_t N, void *workspace,
                  qfp4_dtype out_dt, void *out, cudaStream_t stream)
{
    const FusedLayout F = fused_layout(M, N, K, fmt);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *a_codes = ws + F.codes, *a_scales = ws + F.scales;
    float *a_tscale = reinterpret_cast<float *>(ws + F.tscale);
    float *partials = reinterpret_cast<float *>(ws + F.partials);
    int st = quantize1d(A_bf16, QFP4_BF16, M * K, fmt, QFP4_RNE, rotate, four6, 0, a_codes, a_scales, a_tscale,
                        partials, nullptr, stream);
    if (st != QFP4_OK) return st;
    const GemmLayout L = gemm_layout(M, N, K, fmt);
    uint8_t *sfa = ws + F.chunks, *sfb = sfa + L.sfa_bytes;
    st = rearrange_scales(a_scales, M, K, fmt, L.MB, L.NC, sfa, stream);
    if (st != QFP4_OK) return st;
    st = rearrange_scales(B_scales, N, K, fmt, 2 * L.NT, L.NC, sfb, stream);
    if (st != QFP4_OK) return st;
    return gemm_core(a_codes, sfa, a_tscale, B_codes, sfb, B_tscale, M, N, K, fmt, out_dt, out, stream);
}

}  // namespace qfp4
