// gemm.cu -- block-scaled GEMM on the fifth-generation tensor cores (tcgen05), taking
// the codes and GEMM-layout block scales of bq_quantize as they are.
//
// D[m, n] = sum_k A[m, k] B[n, k] with A and B quantized along k: MXFP8 (E4M3 or E5M2
// elements, one UE8M0 scale per 32 elements) or NVFP4 (E2M1 elements, one E4M3 scale per
// 16 elements and an fp32 tensor scale per operand). This is the consumer the pages
// quantize for: "Quantization survey" §4.3 (MX and NV block scaling feed Blackwell's
// block-scaled tensor cores) and the FP8-training recipe's fp8_matmul of two FP8 operands
// with fp32 accumulation. The tensor cores apply the block scales themselves; the
// epilogue applies NV's two tensor scales (D = acc * S_a * S_b).
//
// One CTA per SM, persistent over 128 x BN tiles of D (taken in a grouped order that keeps
// a few bands of A and B in L2), with 7 warps:
//  - warp 0, one lane: loads, one stage ring running across the CTA's tiles (the next
//    tile's stages fill while the current one finishes). Per stage (128 bytes of k: 128
//    FP8 or 256 FP4 elements) a tensor-map copy of the A tile [128 rows x 128 B] and the B
//    tile [BN rows x 128 B] (128-byte swizzle), and bulk copies of the scale tiles: the GEMM
//    layout keeps the scales of 128 rows x 4 blocks in one 512-byte tile, which is exactly
//    the shared-memory form tcgen05.cp's 32x128b.warpx4 shape moves into tensor memory;
//  - warp 6, one lane: per stage, once its copies landed, the scale tiles into tensor
//    memory (tcgen05.cp), then a commit that lets the stage's MMAs start (a separate
//    issuer: NVFP4 moves 12 scale tiles a stage);
//  - warp 1, one lane: tensor memory allocation; per tile, once the epilogue has read the
//    previous accumulator, per stage 4 MMAs (k of 32 FP8 or 64 FP4 elements each) into the
//    fp32 accumulator; a commit per stage frees the stage, one per tile hands the
//    accumulator to the epilogue;
//  - warps 2-5: the epilogue. Each reads its 32-lane quarter of the accumulator
//    (tcgen05.ld) 32 columns at a time, scales (NV), rounds to bf16 through a small
//    swizzled staging buffer into row pieces of D, and releases the accumulator as soon as
//    its last columns are read (fp32 output: straight from registers).
// Every wait on an mbarrier gives up after about a second (counted in g_gemm_wait_timeouts);
// the CTA then lets its copies and MMAs in flight finish (bounded), frees its tensor
// memory and returns, leaving D incomplete.
#include "internal.h"
#include "tma.cuh"

#include <atomic>
#include <cstring>

namespace bq {

__device__ unsigned int g_gemm_wait_timeouts = 0;

namespace {

constexpr int GEMM_THREADS = 224;
constexpr uint32_t TMEM_COLS = 512;          // the whole tensor memory of the SM (one CTA per SM)
constexpr uint32_t SF_TMEM_COL = 256;        // scale-factor columns start here (accumulator below)
constexpr uint32_t GEMM_GROUP_M = 8;         // row tiles per group of the tile order

// The bf16 epilogue's staging buffer: per epilogue warp, 32 rows x 32 columns (64-byte
// rows; 16-byte granule g of row r at g ^ ((r >> 1) & 3), so that a warp's row-wise
// writes and its row-block reads both touch 8 distinct 16-byte bank groups per 8 lanes).
// Small, so that the stage ring keeps four stages of 256-column tiles.
constexpr uint32_t OUT_WARP_BYTES = 32u * 64u;
constexpr uint32_t OUT_BYTES = 4u * OUT_WARP_BYTES;

template <int KIND, int BN>
struct GemmCfg {
    static constexpr uint32_t A_BYTES = 128u * 128u;
    static constexpr uint32_t B_BYTES = (uint32_t)BN * 128u;
    // 512-byte scale tiles per 128 rows per stage: 4 blocks of 32 (MX) or 16 blocks of 16 (NV)
    static constexpr uint32_t SFT = KIND == GEMM_MXF8 ? 1u : 4u;
    static constexpr uint32_t BT = (uint32_t)BN / 128u;          // 128-row tiles of B
    static constexpr uint32_t SFA_BYTES = SFT * 512u;
    static constexpr uint32_t SFB_BYTES = BT * SFT * 512u;
    // bytes a stage's copies deliver (the stage's mbarrier transaction count)
    static constexpr uint32_t TX_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    // a stage starts on a 1024-byte boundary: the 128-byte swizzle repeats every 1024 bytes
    // and the operand descriptors assume the tiles start on it
    static constexpr uint32_t STAGE = (TX_BYTES + 1023u) & ~1023u;
    static constexpr uint32_t SF_COLS = 4u * SFT * (1u + BT);    // tensor-memory columns of a stage's scales
    // as many stages as shared memory (less the epilogue buffer, the alignment slack and
    // the barriers) and tensor memory hold, at most 6
    static constexpr uint32_t NS_SMEM = (232448u - OUT_BYTES - 1024u - 512u) / STAGE;
    static constexpr uint32_t NS_TMEM = (TMEM_COLS - SF_TMEM_COL) / SF_COLS;
    static constexpr int NS = (int)(NS_SMEM < NS_TMEM ? (NS_SMEM < 6u ? NS_SMEM : 6u) : (NS_TMEM < 6u ? NS_TMEM : 6u));
    static constexpr uint32_t SMEM = (uint32_t)NS * STAGE + OUT_BYTES + 1024u;
    static_assert(NS >= 2, "pipeline depth");
    static_assert(SF_TMEM_COL + NS * SF_COLS <= TMEM_COLS, "tensor memory");
    static_assert(SMEM <= 232448u, "shared memory");
};

// Shared-memory matrix descriptor (sm_100): start address, leading / stride byte offsets
// (all >> 4), descriptor version 1 at bit 46, layout type at bits 61-63 (2: 128-byte
// swizzle, 0: none).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// K-major operand tile, 128-byte rows, 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr) { return smem_desc(addr, 16u, 1024u, 2u); }

// A 512-byte scale tile: 32 rows of 16 bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t scale_desc(uint32_t addr) { return smem_desc(addr, 0u, 128u, 0u); }

// Instruction descriptor of the block-scaled MMA (M = 128, N = BN, both operands K-major):
// element formats at bits 7-9 / 10-12, N / 8 at 17-22, the scale format at 23 (1: UE8M0,
// 0: E4M3), M / 16 at 24-28, the scale-factor byte of A at 29-30 and of B at 4-5.
template <int KIND, int BN>
__device__ __forceinline__ uint32_t instr_desc(uint32_t elem_fmt, uint32_t sf_id)
{
    const uint32_t scale_fmt = KIND == GEMM_MXF8 ? 1u : 0u;
    return (elem_fmt << 7) | (elem_fmt << 10) | ((uint32_t)(BN >> 3) << 17) | (scale_fmt << 23) |
           ((128u >> 4) << 24) | (sf_id << 29) | (sf_id << 4);
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_cp_scales(uint32_t taddr, uint64_t desc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(desc) : "memory");
}

template <int KIND>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t accumulate)
{
    if constexpr (KIND == GEMM_MXF8) {
        asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
                     "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}"
                     :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb) : "memory");
    } else {
        asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
                     "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}"
                     :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb) : "memory");
    }
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

// The tile order: groups of GEMM_GROUP_M row tiles, column by column inside a group, so
// the tiles in flight at a time share a few bands of A and of B (they stay in L2).
__device__ __forceinline__ void tile_coords(uint32_t t, uint32_t num_m, uint32_t num_n, uint32_t& m_tile,
                                            uint32_t& n_tile)
{
    const uint32_t per_group = GEMM_GROUP_M * num_n, grp = t / per_group;
    const uint32_t first_m = grp * GEMM_GROUP_M, gm = min(GEMM_GROUP_M, num_m - first_m);
    const uint32_t local = t - grp * per_group;
    m_tile = first_m + local % gm;
    n_tile = local / gm;
}

template <int KIND, int BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1) k_bs_gemm(const __grid_constant__ CUtensorMap amap,
                                                           const __grid_constant__ CUtensorMap bmap,
                                                           const GemmArgs g)
{
    using C = GemmCfg<KIND, BN>;
    extern __shared__ uint8_t gemm_smem[];
    __shared__ __align__(8) uint64_t full_bar[C::NS], sf_bar[C::NS], empty_bar[C::NS], acc_full, acc_empty, done_bar, sf_done;
    __shared__ uint32_t tmem_holder;
    __shared__ volatile int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t base = (smem_addr(gemm_smem) + 1023u) & ~1023u;
    const uint32_t out_base = base + C::NS * C::STAGE;
    const uint32_t num_m = g.m / 128u, num_n = g.n / (uint32_t)BN, num_tiles = num_m * num_n;
    const uint32_t KT = g.k_stages;

    auto a_smem = [&](uint32_t s) { return base + s * C::STAGE; };
    auto b_smem = [&](uint32_t s) { return base + s * C::STAGE + C::A_BYTES; };
    auto sfa_smem = [&](uint32_t s) { return base + s * C::STAGE + C::A_BYTES + C::B_BYTES; };
    auto sfb_smem = [&](uint32_t s) { return base + s * C::STAGE + C::A_BYTES + C::B_BYTES + C::SFA_BYTES; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(smem_addr(&full_bar[s]), 1);
            mbar_init(smem_addr(&sf_bar[s]), 1);
            mbar_init(smem_addr(&empty_bar[s]), 1);
        }
        mbar_init(smem_addr(&acc_full), 1);
        mbar_init(smem_addr(&acc_empty), 4);          // one arrival per epilogue warp
        mbar_init(smem_addr(&done_bar), 1);
        mbar_init(smem_addr(&sf_done), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_addr(&tmem_holder)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_holder;

    if (warp == 0 && lane == 0) {
        // ---- loads: one stage ring over all of the CTA's tiles ----
        uint32_t it = 0;
        for (uint32_t t = blockIdx.x; t < num_tiles && !abort_flag; t += gridDim.x) {
            uint32_t m_tile, n_tile;
            tile_coords(t, num_m, num_n, m_tile, n_tile);
            const uint8_t* sfa_row = g.sfa + (size_t)m_tile * g.sf_tiles_per_row * 512u;
            for (uint32_t kk = 0; kk < KT; ++kk, ++it) {
                const uint32_t s = it % C::NS;
                if (it >= C::NS && !mbar_wait(smem_addr(&empty_bar[s]), ((it / C::NS) - 1) & 1u)) {
                    abort_flag = 1;
                    break;
                }
                if (abort_flag) break;
                const uint32_t fb = smem_addr(&full_bar[s]);
                mbar_arrive_expect_tx(fb, C::TX_BYTES);
                tma_load_2d(a_smem(s), &amap, fb, (int)(kk * 128u), (int)(m_tile * 128u));
                tma_load_2d(b_smem(s), &bmap, fb, (int)(kk * 128u), (int)(n_tile * (uint32_t)BN));
                bulk_load(sfa_smem(s), sfa_row + (size_t)kk * C::SFT * 512u, C::SFA_BYTES, fb);
                for (uint32_t i = 0; i < C::BT; ++i) {
                    const uint8_t* src = g.sfb + ((size_t)(n_tile * C::BT + i) * g.sf_tiles_per_row + kk * C::SFT) * 512u;
                    bulk_load(sfb_smem(s) + i * C::SFT * 512u, src, C::SFT * 512u, fb);
                }
            }
        }
        if (abort_flag) {
            // let the copies in flight land before the CTA can exit (bounded)
            const uint32_t first = it > (uint32_t)C::NS ? it - C::NS : 0u;
            for (uint32_t j = first; j < it; ++j)
                (void)mbar_wait(smem_addr(&full_bar[j % C::NS]), (j / C::NS) & 1u);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMAs: a tile's k stages into the accumulator, once the epilogue has read
        // the previous tile's; a stage is taken once its scale tiles are in tensor memory
        // (which the scale warp moves only after the stage's copies landed) ----
        uint32_t it = 0, i = 0;
        for (uint32_t t = blockIdx.x; t < num_tiles && !abort_flag; t += gridDim.x, ++i) {
            if (i > 0 && !mbar_wait(smem_addr(&acc_empty), (i - 1) & 1u)) { abort_flag = 1; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            uint32_t acc = 0;
            for (uint32_t kk = 0; kk < KT; ++kk, ++it) {
                const uint32_t s = it % C::NS;
                if (!mbar_wait(smem_addr(&sf_bar[s]), (it / C::NS) & 1u)) { abort_flag = 1; break; }
                if (abort_flag) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t sf = tmem + SF_TMEM_COL + s * C::SF_COLS;
                const uint32_t sfb_col = 4u * C::SFT;
                const uint64_t ad = operand_desc(a_smem(s)), bd = operand_desc(b_smem(s));
#pragma unroll
                for (uint32_t k = 0; k < 4; ++k) {
                    // MX: one 32-bit scale column per 128 rows holds the 4 blocks of the
                    // stage, MMA k reads byte k; NV: MMA k reads all 4 bytes of tile k
                    const uint32_t id = KIND == GEMM_MXF8 ? k : 0u;
                    const uint32_t ta = sf + (KIND == GEMM_MXF8 ? 0u : 4u * k);
                    const uint32_t tb = sf + sfb_col + (KIND == GEMM_MXF8 ? 0u : 4u * k * C::BT);
                    tc_mma<KIND>(tmem, ad + 2u * k, bd + 2u * k, instr_desc<KIND, BN>(g.elem_fmt, id),
                                 ta | (id << 30), tb | (id << 30), acc);
                    acc = 1;
                }
                tc_commit(smem_addr(&empty_bar[s]));     // the stage is free once these MMAs are done
            }
            if (abort_flag) break;
            tc_commit(smem_addr(&acc_full));             // the tile's accumulator is complete
        }
        // every MMA issued so far completes before done_bar's phase does
        tc_commit(smem_addr(&done_bar));
        if (!mbar_wait(smem_addr(&done_bar), 0u)) abort_flag = 1;
    } else if (warp == 6 && lane == 0) {
        // ---- scale tiles into tensor memory, a stage at a time once its copies landed:
        // A's tiles j at columns 4 j, B's (row tile b, tile j) at 4 (j BT + b), so the
        // BN / 128 tiles of one block group sit side by side. The stage's tensor-memory
        // columns are free: its previous MMAs completed before the loads refilled it ----
        uint32_t it = 0;
        for (uint32_t t = blockIdx.x; t < num_tiles && !abort_flag; t += gridDim.x) {
            for (uint32_t kk = 0; kk < KT; ++kk, ++it) {
                const uint32_t s = it % C::NS;
                if (!mbar_wait(smem_addr(&full_bar[s]), (it / C::NS) & 1u)) { abort_flag = 1; break; }
                if (abort_flag) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t sf = tmem + SF_TMEM_COL + s * C::SF_COLS;
                const uint32_t sfb_col = 4u * C::SFT;
                for (uint32_t j = 0; j < C::SFT; ++j) {
                    tc_cp_scales(sf + 4u * j, scale_desc(sfa_smem(s) + 512u * j));
                    for (uint32_t b = 0; b < C::BT; ++b)
                        tc_cp_scales(sf + sfb_col + 4u * (j * C::BT + b), scale_desc(sfb_smem(s) + (b * C::SFT + j) * 512u));
                }
                tc_commit(smem_addr(&sf_bar[s]));        // the MMAs of the stage may start
            }
        }
        // every copy issued so far completes before sf_done's phase does
        tc_commit(smem_addr(&sf_done));
        if (!mbar_wait(smem_addr(&sf_done), 0u)) abort_flag = 1;
    } else if (warp >= 2 && warp <= 5) {
        // ---- epilogue: warp w reads lanes 32 (w % 4) .. + 31 of the accumulator ----
        const uint32_t q = (uint32_t)warp & 3u;
        const uint32_t ob = out_base + q * OUT_WARP_BYTES;
        const float sc = KIND == GEMM_NVF4 ? __fmul_rn(g.a_tensor_scale ? *g.a_tensor_scale : 1.0f,
                                                        g.b_tensor_scale ? *g.b_tensor_scale : 1.0f) : 1.0f;
        uint32_t i = 0;
        for (uint32_t t = blockIdx.x; t < num_tiles; t += gridDim.x, ++i) {
            uint32_t m_tile, n_tile;
            tile_coords(t, num_m, num_n, m_tile, n_tile);
            bool ok = mbar_wait(smem_addr(&acc_full), i & 1u);
            ok = __all_sync(0xFFFFFFFFu, ok) && !abort_flag;
            if (!ok) { abort_flag = 1; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t row0 = m_tile * 128u + q * 32u;
            if (g.d_bf16) {
                // chunks of 32 columns: accumulator -> bf16 -> staging buffer -> whole
                // 64-byte row pieces of D; the accumulator is released once its last
                // columns are read, before that chunk's stores
#pragma unroll 1
                for (uint32_t c0 = 0; c0 < (uint32_t)BN; c0 += 32u) {
                    uint32_t r[32];
                    tmem_ld32(tmem + ((q * 32u) << 16) + c0, r);
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
                        if (KIND == GEMM_NVF4) { x0 = __fmul_rn(x0, sc); x1 = __fmul_rn(x1, sc); }
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                        w[e] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
                    if (c0 + 32u == (uint32_t)BN) {
                        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_addr(&acc_empty));
                    }
                    // row = lane: its 4 granules
                    const uint32_t sw = ((uint32_t)lane >> 1) & 3u;
#pragma unroll
                    for (uint32_t e = 0; e < 4; ++e)
                        sts_v4(ob + (uint32_t)lane * 64u + ((e ^ sw) * 16u), w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                    __syncwarp();
                    // 8 rows per store: lane l takes granule l % 4 of row 8 j + l / 4
#pragma unroll
                    for (uint32_t j = 0; j < 4; ++j) {
                        const uint32_t rr = 8u * j + ((uint32_t)lane >> 2), gi = (uint32_t)lane & 3u;
                        uint32_t v0, v1, v2, v3;
                        lds_v4(ob + rr * 64u + ((gi ^ ((rr >> 1) & 3u)) * 16u), v0, v1, v2, v3);
                        const uint32_t v[4] = {v0, v1, v2, v3};
                        const size_t off = (size_t)(row0 + rr) * g.ldd + n_tile * (uint32_t)BN + c0 + 8u * gi;
                        st_v4(reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(g.d) + off), v);
                    }
                    __syncwarp();        // the buffer is read before the next chunk refills it
                }
            } else {
                const uint32_t row = row0 + (uint32_t)lane;
#pragma unroll 1
                for (uint32_t c0 = 0; c0 < (uint32_t)BN; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem + ((q * 32u) << 16) + c0, r);
                    const size_t off = (size_t)row * g.ldd + n_tile * (uint32_t)BN + c0;
                    uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<float*>(g.d) + off);
#pragma unroll
                    for (int e8 = 0; e8 < 8; ++e8) {
                        uint32_t v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            v[e] = KIND == GEMM_NVF4 ? __float_as_uint(__fmul_rn(__uint_as_float(r[4 * e8 + e]), sc))
                                                     : r[4 * e8 + e];
                        st_v4(dst + 4 * e8, v);
                    }
                }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&acc_empty));
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0 && abort_flag) atomicAdd(&g_gemm_wait_timeouts, 1u);
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// Operand codes [rows, kb] bytes, K-major: boxes of 128 bytes x box_rows rows, 128-byte swizzle.
cudaError_t operand_map(const void* p, uint32_t rows, uint32_t kb, uint32_t box_rows, CUtensorMap* map)
{
    *map = CUtensorMap{};
    const EncodeTiled enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {kb, rows};
    const cuuint64_t strides[1] = {kb};
    const cuuint32_t box[2] = {128, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(p), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int KIND, int BN>
cudaError_t run_gemm(const GemmArgs& g, cudaStream_t st)
{
    using C = GemmCfg<KIND, BN>;
    constexpr auto kern = k_bs_gemm<KIND, BN>;
    static std::atomic<bool> attr_set{false};
    if (!attr_set.load(std::memory_order_acquire)) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set.store(true, std::memory_order_release);
    }
    CUtensorMap am, bm;
    cudaError_t e = operand_map(g.a, g.m, g.kb, 128u, &am);
    if (e != cudaSuccess) return e;
    e = operand_map(g.b, g.n, g.kb, (uint32_t)BN, &bm);
    if (e != cudaSuccess) return e;
    // persistent: a CTA per SM (tensor memory and shared memory admit one), tiles strided
    const unsigned tiles = (g.n / BN) * (g.m / 128u);
    const unsigned sms = (unsigned)device_sm_count();
    const unsigned grid = tiles < sms ? tiles : sms;
    kern<<<grid, GEMM_THREADS, C::SMEM, st>>>(am, bm, g);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(int kind, const GemmArgs& g, cudaStream_t st)
{
    const bool wide = g.n % 256u == 0;
    if (kind == GEMM_MXF8) return wide ? run_gemm<GEMM_MXF8, 256>(g, st) : run_gemm<GEMM_MXF8, 128>(g, st);
    if (kind == GEMM_NVF4) return wide ? run_gemm<GEMM_NVF4, 256>(g, st) : run_gemm<GEMM_NVF4, 128>(g, st);
    return cudaErrorInvalidValue;
}

cudaError_t gemm_wait_timeouts(unsigned int* count, bool reset)
{
    cudaError_t e = cudaMemcpyFromSymbol(count, g_gemm_wait_timeouts, sizeof(unsigned int));
    if (e == cudaSuccess && reset) {
        const unsigned int zero = 0u;
        e = cudaMemcpyToSymbol(g_gemm_wait_timeouts, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace bq
