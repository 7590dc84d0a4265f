// quant_row.cu -- per-row quantize (one scale per row: an output channel of a weight
// [out, in], or a token of an activation [tokens, hidden]).
//
// Steps (source pages): per-channel weights and per-token dynamic activation scales
// ("FP8 vs INT8" commentary §3.2; 2025 trend article §三, dynamic scales computed at
// run time); AbsMax scale s = max|x_row| / Qmax and q = clamp(round(x/s))
// ("INT vs FP at fine granularity" §2.1); asymmetric rows with a zero point
// ("INT4/INT8/FP8 quantization" §INT8).
//
// A CTA owns a row at a time (persistent over rows). Each thread holds K chunks of 16
// elements of the row (256-bit loads); the next row's chunks are loaded before the
// current row is reduced and quantized, so the loads of one row overlap the work on
// the previous one. The row range is reduced with warp shuffles and one barrier
// through double-buffered shared memory, and the codes come from registers: one read
// of x. Rows longer than 4 chunks per thread of a 256-thread CTA are read twice
// (range pass, then quantize pass; the second read comes from L2).
#include "quant_ops.cuh"
#include "internal.h"

#include <atomic>

namespace bq {

template <int FMT, bool HAD, bool STATS, int K>
__global__ void __launch_bounds__(256) k_quant_row(const RowArgs a)
{
    pdl_wait();
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    __shared__ float red[2][8][4];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const uint32_t B = blockDim.x;
    const bool fp16 = a.scale_fp16 != 0;
    Acc acc;
    int it = 0;
    constexpr int KK = K > 0 ? K : 1;
    uint32_t cur[KK][8];

    auto load_row = [&](uint32_t r, uint32_t (&dst)[KK][8]) {
        const uint32_t c_row = r * a.cpr;
#pragma unroll
        for (int k = 0; k < KK; ++k) {
            const uint32_t c = tid + k * B;
            if (c < a.cpr) ld_nc_v8(a.x + (size_t)(c_row + c) * 8, dst[k]);
            else {
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[k][i] = 0u;
            }
        }
    };

    uint32_t r = blockIdx.x;
    if constexpr (K > 0) {
        if (r < a.rows) load_row(r, cur);
    }
    for (; r < a.rows; r += gridDim.x, ++it) {
        const uint32_t c_row = r * a.cpr;
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
        uint32_t nxt[KK][8];

        // range of this thread's part of the row: raw bf16 words, or rotated values
        if constexpr (K > 0) {
            const uint32_t rn = r + gridDim.x;
            if (rn < a.rows) load_row(rn, nxt);
            if constexpr (HAD) {
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    float2 v[8];
                    widen16x2(cur[k], v);
                    fwht16x2(v);
                    if constexpr (F::asym) chunk_minmax(v, mn, mx);
                    else amax = chunk_amax(v, amax);
                }
            } else if constexpr (F::asym) {
                uint32_t lo = 0u, hi = 0u;
#pragma unroll
                for (int k = 0; k < K; ++k) words_minmax(cur[k], lo, hi);
                mn = pair_min(lo);
                mx = pair_max(hi);
            } else {
                uint32_t m = 0u;
#pragma unroll
                for (int k = 0; k < K; ++k) m = words_absmax(cur[k], m);
                amax = pair_absmax(m);
            }
        } else {
            for (uint32_t c = tid; c < a.cpr; c += B) {
                uint32_t w[8];
                float2 v[8];
                ld_nc_v8(a.x + (size_t)(c_row + c) * 8, w);
                widen16x2(w, v);
                if constexpr (HAD) fwht16x2(v);
                if constexpr (F::asym) chunk_minmax(v, mn, mx);
                else amax = chunk_amax(v, amax);
            }
        }

        if constexpr (F::asym) { mn = warp_minf(mn); mx = warp_maxf(mx); }
        else amax = warp_maxf(amax);
        float (*rb)[4] = red[it & 1];
        if (lane == 0) { rb[warp][0] = amax; rb[warp][1] = mn; rb[warp][2] = mx; }
        __syncthreads();
        float A = 0.0f, MN = 0.0f, MX = 0.0f;
        for (int w = 0; w < nw; ++w) { A = fmaxf(A, rb[w][0]); MN = fminf(MN, rb[w][1]); MX = fmaxf(MX, rb[w][2]); }
        if constexpr (F::asym) A = fmaxf(-MN, MX);

        const PlainScale ps = plain_scale<FMT>(A, MN, MX, fp16);
        const PlainUnit<FMT> u = plain_unit<FMT>(ps);
        if (tid == 0) store_plain_scale<FMT>(a.scales, a.zps, r, ps, fp16);
        const Pow2 pw = pow2_for(A);
        const bool scaled = STATS && !plain_sums_ok(A);      // uniform over the CTA
        const bool exact_res = !HAD && fp16;
        const float p = scaled ? pw.p : 1.0f;
        float2 e2 = splat(0.0f), x2 = splat(0.0f);

        // every lane of a warp quantizes (lanes past the row's end pass zeros and store
        // nothing): the chunk functions are warp-collective
        with_chunk_flags<FMT>(exact_res, unit_general<FMT>(u, scaled), [&](auto ex, auto ge) {
            auto emit = [&](const uint32_t (&wi)[8], uint32_t c, bool valid) {
                float2 v[8];
                uint32_t q[NW];
                widen16x2(wi, v);
                if constexpr (HAD) fwht16x2(v);
                plain_chunk<FMT, STATS, decltype(ex)::value, decltype(ge)::value>(v, u, scaled, p, q, e2, x2);
                if (valid) store_codes<FMT>(a.codes, c_row + c, q);
            };
            if constexpr (K > 0) {
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    const uint32_t c = tid + k * B;
                    emit(cur[k], c, c < a.cpr);
                }
            } else {
                // all lanes run the same trip count (those past the end pass zeros)
                const uint32_t trips = (a.cpr + B - 1) / B;
                for (uint32_t j = 0; j < trips; ++j) {
                    const uint32_t c = tid + j * B;
                    uint32_t w[8];
                    if (c < a.cpr) ld_nc_v8(a.x + (size_t)(c_row + c) * 8, w);
                    else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) w[i] = 0u;
                    }
                    emit(w, c, c < a.cpr);
                }
            }
        });
        if constexpr (K > 0) {
#pragma unroll
            for (int k = 0; k < K; ++k)
#pragma unroll
                for (int i = 0; i < 8; ++i) cur[k][i] = nxt[k][i];
        }

        if constexpr (STATS) {
            add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
            // crest factor of the row: amax / sqrt(mean of squares), on the same scaling
            float ss = __fadd_rn(x2.x, x2.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
            if (lane == 0) rb[warp][3] = ss;
            __syncthreads();
            if (tid == 0) {
                float SS = 0.0f;
                for (int w = 0; w < nw; ++w) SS = __fadd_rn(SS, rb[w][3]);
                kappa_add(acc, __fmul_rn(A, p), SS, a.inv_cols);
            }
        }
    }
    if constexpr (STATS) finish_stats(acc, a.ws, a.stats, false, 0.0f, 0.0, true);
}

namespace {

template <auto KERN, int BLOCK>
int resident_ctas()
{
    static std::atomic<int> cached{-1};
    int v = cached.load(std::memory_order_relaxed);
    if (v < 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, KERN, BLOCK, 0) != cudaSuccess || v < 1) v = 1;
        cached.store(v, std::memory_order_relaxed);
    }
    return v;
}

template <int FMT, bool HAD, bool STATS, int K>
cudaError_t run_row(const RowArgs& a, int block, cudaStream_t st)
{
    constexpr auto kern = k_quant_row<FMT, HAD, STATS, K>;
    int occ;
    switch (block) {
    case 32: occ = resident_ctas<kern, 32>(); break;
    case 64: occ = resident_ctas<kern, 64>(); break;
    case 128: occ = resident_ctas<kern, 128>(); break;
    default: occ = resident_ctas<kern, 256>(); break;
    }
    uint64_t grid = (uint64_t)device_sm_count() * occ;
    if (grid > a.rows) grid = a.rows;
    if (grid > (uint64_t)MAX_GRID) grid = MAX_GRID;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, (unsigned)grid, (unsigned)block, 0, st, a);
}

template <int FMT, bool HAD, bool STATS>
cudaError_t run_row_k(const RowArgs& a, cudaStream_t st)
{
    // two chunks per thread where the row allows it (halves the per-thread scale work),
    // one for short rows, four for long ones; blocks of 32..256 threads.
    const uint32_t cpr = a.cpr;
    auto block_for = [](uint32_t threads) {
        int b = 32;
        while ((uint32_t)b < threads) b <<= 1;
        return b;
    };
    if (cpr <= 32) return run_row<FMT, HAD, STATS, 1>(a, block_for(cpr), st);
    if (cpr <= 512) return run_row<FMT, HAD, STATS, 2>(a, block_for((cpr + 1) / 2), st);
    if (cpr <= 1024) return run_row<FMT, HAD, STATS, 4>(a, block_for((cpr + 3) / 4), st);
    return run_row<FMT, HAD, STATS, 0>(a, 256, st);
}

template <int FMT>
cudaError_t run_row_hs(bool had, bool stats, const RowArgs& a, cudaStream_t st)
{
    if (had) return stats ? run_row_k<FMT, true, true>(a, st) : run_row_k<FMT, true, false>(a, st);
    return stats ? run_row_k<FMT, false, true>(a, st) : run_row_k<FMT, false, false>(a, st);
}

}  // namespace

cudaError_t launch_quant_row(int fmt, bool had, bool stats, const RowArgs& a, cudaStream_t st)
{
    switch (fmt) {
    case BQ_INT8_SYM:   return run_row_hs<BQ_INT8_SYM>(had, stats, a, st);
    case BQ_INT8_ASYM:  return run_row_hs<BQ_INT8_ASYM>(had, stats, a, st);
    case BQ_INT4_SYM:   return run_row_hs<BQ_INT4_SYM>(had, stats, a, st);
    case BQ_UINT4_ASYM: return run_row_hs<BQ_UINT4_ASYM>(had, stats, a, st);
    case BQ_FP8_E4M3:   return run_row_hs<BQ_FP8_E4M3>(had, stats, a, st);
    case BQ_FP8_E5M2:   return run_row_hs<BQ_FP8_E5M2>(had, stats, a, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace bq
