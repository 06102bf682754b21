// gemm.cu -- block-scaled FP4 (and MXFP8) GEMM on 5th-generation tensor
// cores: Y[m][n] = sum_k deqA[m][k] deqB[n][k]  (A: M x K, B: N x K, both
// K-major: packed E2M1 codes, or E4M3 bytes for MXFP8, with row-major
// scales as qfp4_quantize / qfp4_quantize_mxfp8 write them).
//
// Method: [QN] §QuTLASS (MXFP4 / NVFP4 operands, FP32 accumulation; FP8
// for the backward); [LB] §FP4 (Blackwell FP4 tensor cores).  Two
// persistent, warp-specialised kernels on sm_100a, both with fp32
// accumulators in tensor memory (TMEM), operands staged by TMA with 128-byte
// swizzle and no multicast:
//   * k_gemm_bs2 (M > 128): a cluster of two CTAs computes a 256 x 256 tile
//     with tcgen05.mma.cta_group::2 (kind::mxf4 block32 for MXFP4,
//     kind::mxf4nvf4 block16 for NVFP4, kind::mxf8f6f4 block32 with E4M3
//     operands for MXFP8).  The leader's one MMA lane issues;
//     a scale producer and four scale warps per CTA move each k-tile's scale
//     words into a ring of TMEM buffers with tcgen05.st; eight epilogue warps
//     per CTA read the accumulator (tcgen05.ld), hand it back, then store.
//   * k_gemm_blockscaled (M <= 128): one CTA per 128 x 256 tile; the MMA lane
//     moves the scale chunks to TMEM with tcgen05.cp (32x128b.warpx4).
// Both hand the accumulator back as soon as it is in registers, so the next
// tile's MMAs overlap the stores.  The row-major scales are first rearranged
// by a small prepass into 512-byte chunks (128 rows x 4 scales: byte
// (r%32)*16 + (r/32)*4 + j), which the main loops load with plain TMA or
// bulk copies; the chunks live in the caller's workspace.
#include "qfp4_common.cuh"
#include "quantize1d.cuh"

namespace qfp4 {

constexpr int GM_BM = 128, GM_BN = 256;                  // tile rows / columns
constexpr int GM_BKB = 128;                               // bytes of one operand row per stage
// Element format of the GEMM besides QFP4_MXFP4 / QFP4_NVFP4: MXFP8 (E4M3
// bytes under E8M0 scales per 32) is QFP4_MXFP8.
// k-tile length in elements: 128 bytes of a row hold 256 FP4 or 128 FP8 values.
__host__ __device__ constexpr int gm_bk(int fmt) { return fmt == QFP4_MXFP8 ? 128 : 256; }
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
__host__ __device__ constexpr int gm_cps(int fmt) { return fmt == QFP4_NVFP4 ? 4 : fmt == QFP4_MXFP4 ? 2 : 1; }

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
    if (FMT == QFP4_MXFP8)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    else if (FMT == QFP4_NVFP4)
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

// Instruction descriptor of the block-scaled MMA: A and B types at bits 7
// and 10 (E2M1 = 1 for kind::mxf4 / mxf4nvf4; E4M3 = 0 for kind::mxf8f6f4),
// K-major, N >> 3 at bit 17, scale format (0 = UE4M3, 1 = UE8M0) at bit 23,
// M >> 4 at bit 24, scale-factor byte selectors at bits 4 (B) and 29 (A).
__host__ __device__ constexpr uint32_t idesc_blockscaled(int fmt, int M, int N, uint32_t sf_id)
{
    const uint32_t ty = fmt == QFP4_MXFP8 ? 0u : 1u;
    return (sf_id << 4) | (ty << 7) | (ty << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           ((fmt == QFP4_NVFP4 ? 0u : 1u) << 23) | (static_cast<uint32_t>(M >> 4) << 24) | (sf_id << 29);
}

// wait of a whole warp before a .sync.aligned tcgen05 instruction: either
// every lane saw the phase complete or every lane gives up
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity)) != 0;
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
// The GEMM reads scales in 512-byte chunks, one per (128-row block rb, group
// of four scale columns c), chunk index rb * NC + c: byte (r % 32) * 16 +
// (r / 32) * 4 + j holds the scale of row rb * 128 + r, column 4c + j; zero
// beyond R rows or Kg columns.  A block takes one 128-row block and eight
// chunks: it reads the 128 x 32 scale bytes row by row (16-byte loads where
// the rows allow them) into shared memory and writes the eight chunks, 4 KiB
// that are contiguous in the output, as 16-byte stores.  Both operands go in
// one launch: blockIdx.y runs over A's row blocks, then B's.
struct SfJob {
    const uint8_t *sc;
    int R, nblk;
    uint8_t *dst;
};
constexpr int SF_CHUNKS_PER_BLOCK = 8;

__global__ void __launch_bounds__(256) k_sf_chunks(SfJob ja, SfJob jb, int Kg, int NC)
{
    __shared__ uint32_t tile[128 * 9];                    // 128 rows x 32 bytes, row stride 36 bytes
    pdl_wait();
    pdl_trigger();
    const bool is_a = static_cast<int>(blockIdx.y) < ja.nblk;
    const SfJob j = is_a ? ja : jb;
    const int rb = is_a ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y) - ja.nblk;
    const int c0 = static_cast<int>(blockIdx.x) * SF_CHUNKS_PER_BLOCK;
    const int t = threadIdx.x;
    {
        const int row = t >> 1, gs = 4 * c0 + 16 * (t & 1);
        const int64_t grow = static_cast<int64_t>(rb) * 128 + row;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (grow < j.R) {
            const uint8_t *src = j.sc + grow * Kg + gs;
            if (gs + 16 <= Kg && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
                const uint4 v = *reinterpret_cast<const uint4 *>(src);
                w[0] = v.x;
                w[1] = v.y;
                w[2] = v.z;
                w[3] = v.w;
            } else {
                for (int i = 0; i < 16; ++i)
                    if (gs + i < Kg) w[i >> 2] |= static_cast<uint32_t>(src[i]) << (8 * (i & 3));
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) tile[row * 9 + 4 * (t & 1) + i] = w[i];
    }
    __syncthreads();
    const int ci = t >> 5, r0 = t & 31;
    if (c0 + ci < NC) {
        const uint4 o = make_uint4(tile[r0 * 9 + ci], tile[(r0 + 32) * 9 + ci], tile[(r0 + 64) * 9 + ci],
                                   tile[(r0 + 96) * 9 + ci]);
        *reinterpret_cast<uint4 *>(j.dst + (static_cast<int64_t>(rb) * NC + c0 + ci) * 512 + r0 * 16) = o;
    }
}

// ------------------------------------------------------------------ main kernel
template <int FMT, int OUT>
__global__ void __launch_bounds__(GM_THREADS, 1)
    k_gemm_blockscaled(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[GM_STAGES], empty[GM_STAGES], acc_full, acc_empty, drain;
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
        mbar_init(&drain, 1);
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
    pdl_wait();
    pdl_trigger();

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
            if (abort_flag) settle_ns(kSettleNs);   // loads already issued may still be landing
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
                    for (int k = 0; k < 4; ++k) {       // four MMAs of 64 (FP4) or 32 (FP8) elements
                        uint32_t sfa, sfb, id;
                        if (FMT == QFP4_NVFP4) {
                            sfa = sfa_col + 4 * k;
                            sfb = sfb_col + 8 * k;
                            id = idesc_blockscaled(FMT, GM_BM, GM_BN, 0);
                        } else if (FMT == QFP4_MXFP8) {
                            // one chunk per k-tile; MMA k takes byte k (its one block-32 scale)
                            const uint32_t sel = static_cast<uint32_t>(k);
                            sfa = sfa_col | (sel << 30);
                            sfb = sfb_col | (sel << 30);
                            id = idesc_blockscaled(FMT, GM_BM, GM_BN, sel);
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
            // every MMA and scale copy this thread issued has finished before the CTA can leave
            umma_commit(&drain);
            if (!mbar_wait(&drain, 0)) abort_flag = 1;
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
            if (!warp_wait(&acc_full, ti & 1)) { abort_flag = 1; break; }
            tc_fence_after();
            // two 16-lane halves of this warp's quadrant, 128 columns each
            uint32_t r[128];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                tmem_ld16x256b_x16(tmem + (static_cast<uint32_t>(32 * q + 16 * hh) << 16) + 128 * h, r + 64 * hh);
            tmem_ld_wait();
            reg_fence<128>(r);
            // the accumulator is in registers: hand it back before the stores
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

// ------------------------------------------------------------------ 2-CTA kernel
// A cluster of two CTAs on two SMs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256: each CTA holds 128 rows of A and of the
// accumulator, and half (128 rows) of the tile's B, which the pair shares).
// Each CTA loads its A half and B half with cta_group::2 TMA loads that
// complete on the leader CTA's barrier; the leader alone issues the MMAs and
// its commits arrive in both CTAs.  Compared with the 1-CTA tile each SM
// stages 38 KiB instead of 54 KiB per k-tile and issues half the MMAs per unit
// of work.
//
// Scale factors do not go through tcgen05.cp: every copy instruction costs
// about as much issue time as an MMA of a quarter k-tile, and the twelve an
// NVFP4 k-tile needs would cap the tensor pipe near 60 %.  Instead a second
// producer thread loads each k-tile's scale chunks (plain TMA into this CTA's
// own ring of scale slots, which runs ahead of the operand stages) and four
// scale warps (one per TMEM lane quadrant) write them into a ring of TMEM
// buffers with tcgen05.st, concurrently with the MMAs.  The MMA for rows in
// quadrant q reads the A scale of row r at lane r, column addr + q and the
// B scale of column n at lane (n mod 32) + 32 q, column addr + n / 32, and
// the MMA takes scale addresses on 4-column (A) and 8-column (B) boundaries.
// Each of a k-tile's four MMAs (K = 64) gets a scale word of its own: the
// four E4M3 scales of its K (NVFP4), or its two E8M0 scales in bytes 0-1
// (MXFP4, so no MMA reads a word through the byte selector):
//   A: lane r, columns bufA + 4 k + (0..3) = scale word of MMA k for row r
//   B: lane l + 32 q, column bufB + 8 k + m = scale word of MMA k for column l + 32 m
// Only column bufA + 4 k + q of a quadrant-q lane is read; the other three
// hold copies so that one store writes a quadrant's A scales.  A k-tile takes
// 16 + 32 columns; the 256 columns after the accumulator hold 5 such buffers,
// which is how far the scale warps may run ahead of the MMAs.  Every store
// starts on a multiple of its own width.
// No TMA multicast.
constexpr int G2_BM = 256, G2_BN = 256;                   // cluster tile
// warp roles by warpgroup: 0 operand producer, 1 MMA issuer, 2 scale producer
// (3 idle); 4..7 scale warps; 8..15 epilogue.  setmaxnreg moves registers from the first two
// warpgroups to the epilogue: 128 x 48 + 128 x 80 + 256 x 184 = 63488 of the
// 512 x 128 = 65536 the block is launched with.
constexpr int G2_SF_WARPS = 4;
constexpr int G2_THREADS = 512;
constexpr int G2_SF_WARP0 = 4, G2_EPI_WARP0 = 8;
constexpr int G2_A_BYTES = 128 * GM_BKB;                  // this CTA's A rows
constexpr int G2_B_BYTES = 128 * GM_BKB;                  // this CTA's half of B
constexpr int G2_STAGE_BYTES = G2_A_BYTES + G2_B_BYTES;
constexpr int G2_STAGES = 6;
constexpr int G2_SF_SLOT_BYTES = 12 * 512;                // A: CPS chunks, B: 2 x CPS chunks (CPS <= 4)
constexpr int G2_SF_SLOTS = 5;
constexpr int G2_SMEM = G2_STAGES * G2_STAGE_BYTES + G2_SF_SLOTS * G2_SF_SLOT_BYTES + 1024;
__host__ __device__ constexpr int g2_sf_bufs(int) { return 5; }
constexpr int G2_SF_BUFS_MAX = 5;
static_assert(256 + G2_SF_BUFS_MAX * 48 <= GM_TMEM_COLS, "TMEM columns");

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared variable in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on a barrier of the leader CTA, given by its shared::cluster address
// (the partner's arrivals cross CTAs).  Default semantics, release at CTA
// scope: what an arrival publishes is tensor-memory state whose accesses
// tcgen05.wait::st / wait::ld already completed in the arriving thread before
// the arrive issues, and the pair's tcgen05.fence::before / after_thread_sync
// bracket the hand-off; no generic-memory data crosses CTAs through these
// barriers.  The cluster-scope release puts a cluster-wide fence in every
// arrival: it took the 8192 x 11008 x 4096 GEMM from 199 us to 361 us.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tma_load_2d_cg2(void *smem_dst, const CUtensorMap *map, uint32_t leader_bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_cg2(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_cg2()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_cg2(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// arrive on `bar` (same offset) in both CTAs once this thread's tcgen05 work completes
__device__ __forceinline__ void umma_commit_cg2_both(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}
template <int FMT>
__device__ __forceinline__ void umma_blockscaled_cg2(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                                     uint32_t sfb, uint32_t accumulate)
{
    if (FMT == QFP4_MXFP8)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    else if (FMT == QFP4_NVFP4)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
}

#define QFP4_R8(b) "r"(v[b]), "r"(v[b + 1]), "r"(v[b + 2]), "r"(v[b + 3]), "r"(v[b + 4]), "r"(v[b + 5]), "r"(v[b + 6]), "r"(v[b + 7])
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t *v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
                 "%14, %15, %16};" ::"r"(taddr),
                 QFP4_R8(0), QFP4_R8(8)
                 : "memory");
}
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t *v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
                 "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
                     taddr),
                 QFP4_R8(0), QFP4_R8(8), QFP4_R8(16), QFP4_R8(24)
                 : "memory");
}
#undef QFP4_R8
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// end of every role of the 2-CTA kernel: no CTA leaves while its partner may
// still signal it; the allocating warp then frees the pair's tensor memory
__device__ __forceinline__ void g2_exit(uint32_t tmem, bool dealloc)
{
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (dealloc) tmem_dealloc_cg2(tmem, GM_TMEM_COLS);
}

template <int FMT, int OUT>
__global__ void __launch_bounds__(G2_THREADS, 1)
    k_gemm_bs2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB, GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[G2_STAGES], empty[G2_STAGES], sfs_full[G2_SF_SLOTS], sfs_empty[G2_SF_SLOTS];
    __shared__ __align__(8) uint64_t sf_full[G2_SF_BUFS_MAX], sf_empty[G2_SF_BUFS_MAX], acc_full, acc_empty, drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_flag;

    constexpr int CPS = gm_cps(FMT);
    constexpr int NBUF = g2_sf_bufs(FMT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int tiles_m = (p.M + G2_BM - 1) / G2_BM, tiles_n = (p.N + G2_BN - 1) / G2_BN;
    const int ntiles = tiles_m * tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < G2_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < G2_SF_SLOTS; ++s) {
            mbar_init(&sfs_full[s], 1);
            mbar_init(&sfs_empty[s], G2_SF_WARPS);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&sf_full[b], 2 * G2_SF_WARPS);
            mbar_init(&sf_empty[b], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, 2 * GM_EPI_WARPS);
        mbar_init(&drain, 1);
        abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmSA);
        prefetch_tensormap(&tmSB);
    }
    if (warp == 1) {
        tmem_alloc_cg2(&tmem_base_sh, GM_TMEM_COLS);
        tmem_relinquish_cg2();
    }
    tc_fence_before();
    cluster_sync();                          // barriers of both CTAs initialised before any remote use
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    pdl_wait();
    pdl_trigger();

    auto stage_a = [&](int s) { return smem + s * G2_STAGE_BYTES; };
    auto stage_b = [&](int s) { return smem + s * G2_STAGE_BYTES + G2_A_BYTES; };
    auto slot_sfa = [&](int s) { return smem + G2_STAGES * G2_STAGE_BYTES + s * G2_SF_SLOT_BYTES; };
    auto slot_sfb = [&](int s) { return slot_sfa(s) + CPS * 512; };
    auto buf_b = [&](int b) { return tmem + 256 + b * 32; };
    auto buf_a = [&](int b) { return tmem + 256 + NBUF * 32 + b * 16; };

    // Each role ends with its own copy of the exit sequence, so that the
    // register-count regions set by setmaxnreg never merge again.
    if (warp < G2_SF_WARP0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 48;");
        if (warp == 0) {
        // ------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            const uint32_t ab_bytes = G2_A_BYTES + G2_B_BYTES;
            int it = 0;
            for (int t = cluster; t < ntiles && !abort_flag; t += nclusters) {
                int mb, nb;
                tile_coords(t, tiles_m, tiles_n, mb, nb);
                const int rb_a = 2 * mb + static_cast<int>(rank);   // this CTA's 128-row block of A
                for (int kt = 0; kt < p.KT; ++kt, ++it) {
                    const int s = it % G2_STAGES;
                    const uint32_t ph = (it / G2_STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u)) { abort_flag = 1; break; }
                    const uint32_t lbar = mapa_shared(smem_u32(&full[s]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * ab_bytes);
                    tma_load_2d_cg2(stage_a(s), &tmA, lbar, kt * GM_BKB, rb_a * 128);
                    tma_load_2d_cg2(stage_b(s), &tmB, lbar, kt * GM_BKB, nb * G2_BN + 128 * static_cast<int>(rank));
                }
            }
            // wait until the leader's commits have released every stage, so no
            // arrival is still on its way to this CTA when it leaves
            for (int i = 0; i < G2_STAGES && !abort_flag; ++i, ++it)
                if (!mbar_wait(&empty[it % G2_STAGES], ((it / G2_STAGES) & 1u) ^ 1u)) abort_flag = 1;
            if (abort_flag) settle_ns(kSettleNs);   // loads already issued may still be landing
        }
        } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA only)
        if (leader && lane == 0) {
            int it = 0, ti = 0;
            for (int t = cluster; t < ntiles && !abort_flag; t += nclusters, ++ti) {
                if (!mbar_wait(&acc_empty, (ti & 1) ^ 1u)) { abort_flag = 1; break; }
                tc_fence_after();
                for (int kt = 0; kt < p.KT; ++kt, ++it) {
                    const int s = it % G2_STAGES, b = it % NBUF;
                    if (!mbar_wait(&full[s], (it / G2_STAGES) & 1u)) { abort_flag = 1; break; }
                    if (!mbar_wait(&sf_full[b], (it / NBUF) & 1u)) { abort_flag = 1; break; }
                    tc_fence_after();
                    const uint64_t adesc = desc_k_sw128(stage_a(s));
                    const uint64_t bdesc = desc_k_sw128(stage_b(s));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {       // four MMAs of 64 (FP4) or 32 (FP8) elements
                        umma_blockscaled_cg2<FMT>(tmem, adesc + 2 * k, bdesc + 2 * k,
                                                  idesc_blockscaled(FMT, G2_BM, G2_BN, 0), buf_a(b) + 4 * k,
                                                  buf_b(b) + 8 * k, (kt | k) != 0);
                    }
                    umma_commit_cg2_both(&empty[s]);
                    umma_commit_cg2_both(&sf_empty[b]);
                }
                umma_commit_cg2_both(&acc_full);
            }
            // every MMA this thread issued has finished before either CTA can leave
            umma_commit_cg2_both(&drain);
            if (!mbar_wait(&drain, 0)) abort_flag = 1;
        } else if (!leader && lane == 0) {
            // the partner waits for the leader's drain arrival (multicast into this CTA)
            if (!mbar_wait(&drain, 0)) abort_flag = 1;
        }
        } else if (warp == 2) {
        // ------------------------------------------------ scale producer (both CTAs)
        if (lane == 0) {
            int it = 0;
            for (int t = cluster; t < ntiles && !abort_flag; t += nclusters) {
                int mb, nb;
                tile_coords(t, tiles_m, tiles_n, mb, nb);
                const int rb_a = 2 * mb + static_cast<int>(rank);
                for (int kt = 0; kt < p.KT; ++kt, ++it) {
                    const int s = it % G2_SF_SLOTS;
                    if (!mbar_wait(&sfs_empty[s], ((it / G2_SF_SLOTS) & 1u) ^ 1u)) { abort_flag = 1; break; }
                    // scale chunks (rows of 128 B, 4 per 512-byte chunk, CPS chunks per k-tile)
                    mbar_arrive_expect_tx(&sfs_full[s], 3 * CPS * 512);
                    tma_load_2d(slot_sfa(s), &tmSA, &sfs_full[s], 0, (rb_a * p.NC + kt * CPS) * 4);
                    tma_load_2d(slot_sfb(s), &tmSB, &sfs_full[s], 0, ((2 * nb) * p.NC + kt * CPS) * 4);
                    tma_load_2d(slot_sfb(s) + CPS * 512, &tmSB, &sfs_full[s], 0, ((2 * nb + 1) * p.NC + kt * CPS) * 4);
                }
            }
            if (abort_flag) settle_ns(kSettleNs);   // loads already issued may still be landing
        }
        }
        g2_exit(tmem, warp == 1);
        return;
    }
    if (warp < G2_EPI_WARP0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
        // ------------------------------------------------ scale warps (both CTAs: own TMEM quadrant)
        const int q = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        int it = 0;
        for (int t = cluster; t < ntiles && !abort_flag; t += nclusters) {
            for (int kt = 0; kt < p.KT; ++kt, ++it) {
                const int s = it % G2_SF_SLOTS, b = it % NBUF;
                if (!warp_wait(&sfs_full[s], (it / G2_SF_SLOTS) & 1u)) { abort_flag = 1; break; }
                if (!warp_wait(&sf_empty[b], ((it / NBUF) & 1u) ^ 1u)) { abort_flag = 1; break; }
                tc_fence_after();
                // raw scale words of this k-tile: word w = the four scales of
                // k-groups 4w .. 4w + 3 (CPS words per row)
                uint32_t ra[CPS], rb[2][CPS][4];
                const uint8_t *sa = slot_sfa(s) + lane * 16 + q * 4;
#pragma unroll
                for (int w = 0; w < CPS; ++w) ra[w] = *reinterpret_cast<const uint32_t *>(sa + 512 * w);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int w = 0; w < CPS; ++w) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(slot_sfb(s) + 512 * (h * CPS + w) + lane * 16);
                        rb[h][w][0] = u.x;
                        rb[h][w][1] = u.y;
                        rb[h][w][2] = u.z;
                        rb[h][w][3] = u.w;
                    }
                // The slot is refilled by the scale producer's next TMA load (an
                // async-proxy write); the reads above are generic-proxy accesses
                // that may still be outstanding when the release below issues.
                // The proxy fence in every lane orders them before the refill.
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfs_empty[s]);
                // one TMEM word per MMA k: NVFP4 (K = 64) uses a whole raw word,
                // MXFP4 (K = 64) the half of one (its two block-32 scales, in
                // bytes 0-1), MXFP8 (K = 32) one byte (its one block-32 scale)
                auto mma_word = [&](const uint32_t *raw, int k) -> uint32_t {
                    if constexpr (FMT == QFP4_NVFP4) return raw[k];
                    else if constexpr (FMT == QFP4_MXFP4) return (raw[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
                    else return (raw[0] >> (8 * k)) & 0xFFu;
                };
                uint32_t av[16], bv[32];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t wa = mma_word(ra, k);
#pragma unroll
                    for (int c = 0; c < 4; ++c) av[4 * k + c] = wa;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) {
                            uint32_t col[CPS];
#pragma unroll
                            for (int w = 0; w < CPS; ++w) col[w] = rb[h][w][mm];
                            bv[8 * k + 4 * h + mm] = mma_word(col, k);
                        }
                }
                tmem_st_x16(buf_a(b) + lane_base, av);
                tmem_st_x32(buf_b(b) + lane_base, bv);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&sf_full[b]), 0));
            }
        }
        // the leader's last releases of the scale buffers are multicast into
        // this CTA too: let them land before the CTA can leave
        for (int i = 0; i < NBUF && !abort_flag; ++i, ++it)
            if (!warp_wait(&sf_empty[it % NBUF], ((it / NBUF) & 1u) ^ 1u)) abort_flag = 1;
        g2_exit(tmem, false);
        return;
    }
    {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 184;");
        // ------------------------------------------------ epilogue (both CTAs: own 128 rows)
        const int q = warp & 3;
        const int h = (warp - G2_EPI_WARP0) >> 2;
        const uint32_t acc_empty_leader = mapa_shared(smem_u32(&acc_empty), 0);
        float alpha = 1.0f;
        if (FMT == QFP4_NVFP4) alpha = __fmul_rn(*p.tA, *p.tB);
        int ti = 0;
        for (int t = cluster; t < ntiles && !abort_flag; t += nclusters, ++ti) {
            int mb, nb;
            tile_coords(t, tiles_m, tiles_n, mb, nb);
            if (!warp_wait(&acc_full, ti & 1)) { abort_flag = 1; break; }
            tc_fence_after();
            uint32_t r[128];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                tmem_ld16x256b_x16(tmem + (static_cast<uint32_t>(32 * q + 16 * hh) << 16) + 128 * h, r + 64 * hh);
            tmem_ld_wait();
            reg_fence<128>(r);
            // the accumulator is in registers: hand it back at once, so the
            // next tile's MMAs overlap these stores
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);

            const int col0 = nb * G2_BN + 128 * h + 2 * (lane & 3);
            const int row_base = mb * G2_BM + 128 * static_cast<int>(rank);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int row = row_base + 32 * q + 16 * hh + 8 * e + (lane >> 2);
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
    g2_exit(tmem, false);
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
    L.KT = static_cast<int>((K + gm_bk(fmt) - 1) / gm_bk(fmt));
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

// Scale chunks of A (n_blocks_a 128-row blocks) and B (n_blocks_b) in one launch.
int rearrange_scales(const uint8_t *a_scales, int64_t M, int n_blocks_a, uint8_t *sfa, const uint8_t *b_scales,
                     int64_t N, int n_blocks_b, uint8_t *sfb, int64_t K, qfp4_fmt fmt, int NC, cudaStream_t stream)
{
    const int g = fmt == QFP4_NVFP4 ? 16 : 32;
    const SfJob ja{a_scales, static_cast<int>(M), n_blocks_a, sfa};
    const SfJob jb{b_scales, static_cast<int>(N), n_blocks_b, sfb};
    const dim3 grid((NC + SF_CHUNKS_PER_BLOCK - 1) / SF_CHUNKS_PER_BLOCK, n_blocks_a + n_blocks_b);
    if (launch_pdl(k_sf_chunks, grid, dim3(256), 0, stream, ja, jb, static_cast<int>(K / g), NC) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

template <int FMT, int OUT>
static int launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p, int grid, cudaStream_t s)
{
    auto kern = k_gemm_blockscaled<FMT, OUT>;
    if (ensure_dyn_smem<k_gemm_blockscaled<FMT, OUT>>(GM_SMEM) != QFP4_OK) return QFP4_ERR_CUDA;
    if (launch_pdl(kern, dim3(grid), dim3(GM_THREADS), GM_SMEM, s, ta, tb, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

template <int FMT, int OUT>
static int launch_gemm2(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa, const CUtensorMap &tsb,
                        const GemmParams &p, int grid, cudaStream_t s)
{
    auto kern = k_gemm_bs2<FMT, OUT>;
    if (ensure_dyn_smem<k_gemm_bs2<FMT, OUT>>(G2_SMEM) != QFP4_OK) return QFP4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(G2_THREADS, 1, 1);
    cfg.dynamicSmemBytes = G2_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return QFP4_ERR_CUDA;
    }
    QFP4_LAUNCH_CHECK();
    return QFP4_OK;
}

// Main kernel on already rearranged scales (sfa / sfb in the chunk layout).
// Problems taller than one 128-row block run on CTA pairs (256 x 256 tiles),
// the rest on single CTAs (128 x 256 tiles).
int gemm_core(const uint8_t *A_codes, const uint8_t *sfa, const float *A_tscale, const uint8_t *B_codes,
              const uint8_t *sfb, const float *B_tscale, int64_t M, int64_t N, int64_t K, qfp4_fmt fmt,
              qfp4_dtype out_dt, void *out, cudaStream_t stream)
{
    const GemmLayout L = gemm_layout(M, N, K, fmt);
    const bool pair = M > GM_BM;
    CUtensorMap ta, tb;
    const uint64_t row_bytes = static_cast<uint64_t>(fmt == QFP4_MXFP8 ? K : K / 2);
    {
        const uint64_t dims[2] = {row_bytes, static_cast<uint64_t>(M)};
        const uint64_t strides[1] = {row_bytes};
        const uint32_t box[2] = {GM_BKB, GM_BM};
        int st = encode_tensor_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(A_codes), dims,
                                   strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != QFP4_OK) return st;
    }
    {
        const uint64_t dims[2] = {row_bytes, static_cast<uint64_t>(N)};
        const uint64_t strides[1] = {row_bytes};
        const uint32_t box[2] = {GM_BKB, static_cast<uint32_t>(pair ? 128 : GM_BN)};
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
    if (pair) {
        // scale chunks viewed as rows of 128 B (4 rows per 512-byte chunk)
        const int cps = gm_cps(fmt);
        CUtensorMap tsa, tsb;
        // rows past the last 128-row block of A (odd block counts) read as zeros
        {
            const uint64_t dims[2] = {128, static_cast<uint64_t>(L.MB) * L.NC * 4};
            const uint64_t strides[1] = {128};
            const uint32_t box[2] = {128, static_cast<uint32_t>(4 * cps)};
            int st = encode_tensor_map(&tsa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(sfa), dims,
                                       strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
            if (st != QFP4_OK) return st;
        }
        {
            const uint64_t dims[2] = {128, static_cast<uint64_t>(2 * L.NT) * L.NC * 4};
            const uint64_t strides[1] = {128};
            const uint32_t box[2] = {128, static_cast<uint32_t>(4 * cps)};
            int st = encode_tensor_map(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(sfb), dims,
                                       strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
            if (st != QFP4_OK) return st;
        }
        const int ntiles = static_cast<int>(((M + G2_BM - 1) / G2_BM) * ((N + G2_BN - 1) / G2_BN));
        const int grid = 2 * imin<int>(ntiles, num_sms() / 2);
        if (fmt == QFP4_MXFP8)
            return out_dt == QFP4_F32 ? launch_gemm2<QFP4_MXFP8, QFP4_F32>(ta, tb, tsa, tsb, p, grid, stream)
                                      : launch_gemm2<QFP4_MXFP8, QFP4_BF16>(ta, tb, tsa, tsb, p, grid, stream);
        if (fmt == QFP4_NVFP4)
            return out_dt == QFP4_F32 ? launch_gemm2<QFP4_NVFP4, QFP4_F32>(ta, tb, tsa, tsb, p, grid, stream)
                                      : launch_gemm2<QFP4_NVFP4, QFP4_BF16>(ta, tb, tsa, tsb, p, grid, stream);
        return out_dt == QFP4_F32 ? launch_gemm2<QFP4_MXFP4, QFP4_F32>(ta, tb, tsa, tsb, p, grid, stream)
                                  : launch_gemm2<QFP4_MXFP4, QFP4_BF16>(ta, tb, tsa, tsb, p, grid, stream);
    }
    const int grid = static_cast<int>(imin<int64_t>(static_cast<int64_t>(L.MB) * L.NT, num_sms()));
    if (fmt == QFP4_MXFP8)
        return out_dt == QFP4_F32 ? launch_gemm<QFP4_MXFP8, QFP4_F32>(ta, tb, p, grid, stream)
                                  : launch_gemm<QFP4_MXFP8, QFP4_BF16>(ta, tb, p, grid, stream);
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
    const int st = rearrange_scales(A_scales, M, L.MB, sfa, B_scales, N, 2 * L.NT, sfb, K, fmt, L.NC, stream);
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

void gemm_fused_rq_layout(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt, size_t *codes, size_t *scales,
                          size_t *tscale)
{
    const FusedLayout F = fused_layout(M, N, K, fmt);
    *codes = F.codes;
    *scales = F.scales;
    *tscale = F.tscale;
}

size_t gemm_fused_rq_workspace(int64_t M, int64_t N, int64_t K, qfp4_fmt fmt)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return fused_layout(M, N, K, fmt).total;
}

// A is rotated and quantized once by the 1D quantize kernel into the
// workspace, then the scale prepass and the CTA-pair GEMM run; the kernels
// follow each other through dependent launches.  NVFP4 measures A's tensor
// amax first unless the caller supplies it (one read of A instead of two).
int gemm_fused_rq(const void *A_bf16, int64_t M, int64_t K, int rotate, int four6, qfp4_fmt fmt,
                  const uint8_t *B_codes, const uint8_t *B_scales, const float *B_tscale, int64_t N, void *workspace,
                  qfp4_dtype out_dt, void *out, cudaStream_t stream, const float *amax_in, float *amax_out)
{
    const FusedLayout F = fused_layout(M, N, K, fmt);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *a_codes = ws + F.codes, *a_scales = ws + F.scales;
    float *a_tscale = reinterpret_cast<float *>(ws + F.tscale);
    float *partials = reinterpret_cast<float *>(ws + F.partials);
    QuantOpts opt;
    opt.amax_in = amax_in;
    opt.amax_out = amax_out;
    int st = quantize1d(A_bf16, QFP4_BF16, M * K, fmt, QFP4_RNE, rotate, four6, 0, a_codes, a_scales, a_tscale,
                        partials, nullptr, stream, opt);
    if (st != QFP4_OK) return st;
    const GemmLayout L = gemm_layout(M, N, K, fmt);
    uint8_t *sfa = ws + F.chunks, *sfb = sfa + L.sfa_bytes;
    st = rearrange_scales(a_scales, M, L.MB, sfa, B_scales, N, 2 * L.NT, sfb, K, fmt, L.NC, stream);
    if (st != QFP4_OK) return st;
    return gemm_core(a_codes, sfa, a_tscale, B_codes, sfb, B_tscale, M, N, K, fmt, out_dt, out, stream);
}

}  // namespace qfp4
