// quant_row.cu -- per-row quantize (one scale per row: an output channel of a weight
// [out, in], or a token of an activation [tokens, hidden]).
//
// Steps (source pages): per-channel weights and per-token dynamic activation scales
// ("FP8 vs INT8" commentary §3.2; 2025 trend article §三, dynamic scales computed at
// run time); AbsMax scale s = max|x_row| / Qmax and q = clamp(round(x/s))
// ("INT vs FP at fine granularity" §2.1); asymmetric rows with a zero point
// ("INT4/INT8/FP8 quantization" §INT8).
//
// A CTA owns a row at a time (persistent over rows). Each thread loads K chunks of 16
// elements (256-bit loads, all issued before any arithmetic), the row range is reduced
// with warp shuffles and one barrier through double-buffered shared memory, and the
// codes are produced from registers: one read of x. Rows longer than K chunks per
// thread are read twice (range pass, then quantize pass; the second read comes from L2).
#include "quant_ops.cuh"
#include "internal.h"

#include <atomic>

namespace bq {

template <int FMT, bool HAD, bool STATS, int K>
__global__ void __launch_bounds__(256) k_quant_row(const RowArgs a)
{
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    __shared__ float red[2][8][4];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const uint32_t B = blockDim.x;
    const bool fp16 = a.scale_fp16 != 0;
    Acc acc;
    int it = 0;
    for (uint32_t r = blockIdx.x; r < a.rows; r += gridDim.x, ++it) {
        const uint32_t c_row = r * a.cpr;   // first chunk of the row (flat index)
        float y[K > 0 ? K : 1][16];
        float amax = 0.0f, mn = 0.0f, mx = 0.0f, ss = 0.0f;

        auto range_of = [&](const float (&v)[16]) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                amax = fmaxf(amax, fabsf(v[i]));
                if constexpr (F::asym) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
                if constexpr (STATS) ss = __fmaf_rn(v[i], v[i], ss);
            }
        };

        if constexpr (K > 0) {
            uint32_t win[K][8];
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const uint32_t c = tid + k * B;
                if (c < a.cpr) ld_nc_v8(a.x + (size_t)(c_row + c) * 8, win[k]);
                else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) win[k][i] = 0u;
                }
            }
#pragma unroll
            for (int k = 0; k < K; ++k) {
                widen16(win[k], y[k]);
                if constexpr (HAD) fwht16(y[k]);
                range_of(y[k]);
            }
        } else {
            for (uint32_t c = tid; c < a.cpr; c += B) {
                float v[16];
                load16(a.x, c_row + c, v);
                if constexpr (HAD) fwht16(v);
                range_of(v);
            }
        }

        amax = warp_maxf(amax);
        if constexpr (F::asym) { mn = warp_minf(mn); mx = warp_maxf(mx); }
        if constexpr (STATS) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
        }
        float (*rb)[4] = red[it & 1];
        if (lane == 0) { rb[warp][0] = amax; rb[warp][1] = mn; rb[warp][2] = mx; rb[warp][3] = ss; }
        __syncthreads();
        float A = 0.0f, MN = 0.0f, MX = 0.0f, SS = 0.0f;
        for (int w = 0; w < nw; ++w) {
            A = fmaxf(A, rb[w][0]); MN = fminf(MN, rb[w][1]); MX = fmaxf(MX, rb[w][2]);
            SS = __fadd_rn(SS, rb[w][3]);
        }

        const PlainScale ps = plain_scale<FMT>(A, MN, MX, fp16);
        const Recip R = make_recip(ps.s, ps.bound);
        if (tid == 0) {
            store_plain_scale<FMT>(a.scales, a.zps, r, ps, fp16);
            if constexpr (STATS) kappa_add(acc, A, SS, a.inv_cols);
        }

        auto emit = [&](const float (&v)[16], uint32_t c) {
            uint32_t w[NW];
            float xh[16];
            quant_plain_chunk<FMT, STATS>(v, ps, R, F::qmin, F::qmax, w, xh);
            store_codes<FMT>(a.codes, c_row + c, w);
            if constexpr (STATS) {
                float e2, x2;
                chunk_sums(v, xh, e2, x2);
                acc.err2 += (double)e2;
                acc.x2 += (double)x2;
            }
        };

        if constexpr (K > 0) {
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const uint32_t c = tid + k * B;
                if (c < a.cpr) emit(y[k], c);
            }
        } else {
            for (uint32_t c = tid; c < a.cpr; c += B) {
                float v[16];
                load16(a.x, c_row + c, v);
                if constexpr (HAD) fwht16(v);
                emit(v, c);
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
    kern<<<(unsigned)grid, block, 0, st>>>(a);
    return cudaGetLastError();
}

template <int FMT, bool HAD, bool STATS>
cudaError_t run_row_k(const RowArgs& a, cudaStream_t st)
{
    // block: the smallest multiple of 32 (<= 256) that covers the row in <= K chunks
    // per thread, K in {1, 2, 4}; longer rows stream twice with 256 threads.
    const uint32_t cpr = a.cpr;
    for (int k : {1, 2, 4}) {
        const uint32_t threads = (cpr + k - 1) / k;
        if (threads <= 256) {
            int block = 32;
            while ((uint32_t)block < threads) block <<= 1;
            if (k == 1) return run_row<FMT, HAD, STATS, 1>(a, block, st);
            if (k == 2) return run_row<FMT, HAD, STATS, 2>(a, block, st);
            return run_row<FMT, HAD, STATS, 4>(a, block, st);
        }
    }
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
