// quant_flat.cu -- one-pass quantize kernels over the tensor seen as a flat run of
// 16-element chunks: per-tensor (after the range pass), per-group, MX block-32 and
// NV block-16 granularities; and the per-tensor range pass itself.
//
// Layout of the work: a warp takes 64 consecutive chunks (1024 elements, 2 KB of
// bf16) per step, lane l the chunks 64t + l and 64t + 32 + l, each loaded with one
// 256-bit load (both loads are issued before either chunk is processed). A scaling
// unit of G elements spans G/16 adjacent lanes and is reduced with xor shuffles. The
// grid is a whole number of waves (SM count x resident CTAs) striding over the steps.
//
// Steps (source pages): AbsMax scale per unit ("INT vs FP at fine granularity" §2.1,
// §3.1); MX block 32 with a power-of-two scale, NV block 16 with an E4M3 block scale
// and an FP32 tensor scale ("Quantization survey" §4.3.1, §4.3.2); optional Hadamard
// rotation of each 16-run ("INT vs FP at fine granularity" §4.2, §7.2); fused QSNR
// and crest-factor sums (same page §4.1).
//
// The fused QSNR of a rotated scheme is summed in the rotated domain: H16/4 is
// orthogonal, so sum (x - xhat)^2 = sum (y - yhat)^2 and sum x^2 = sum y^2 exactly in
// real arithmetic; this saves the inverse transform (bq_qsnr and bq_dequantize
// work in the original domain).
#include "quant_ops.cuh"
#include "internal.h"

#include <atomic>

namespace bq {

// ---------------------------------------------------------------------------
// Per-tensor range pass: amax (and min / max for asymmetric formats) of the
// (rotated) tensor into the workspace header.
// ---------------------------------------------------------------------------

template <bool HAD, bool MINMAX>
__global__ void __launch_bounds__(256) k_range(const uint32_t* __restrict__ x, uint32_t n_chunks, uint8_t* ws)
{
    float amax = 0.0f, mn = 0.0f, mx = 0.0f;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    uint64_t c = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; c + stride < n_chunks; c += 2 * stride) {
        uint32_t w0[8], w1[8];
        ld_nc_v8(x + (size_t)c * 8, w0);
        ld_nc_v8(x + (size_t)(c + stride) * 8, w1);
        float v[16];
        widen16(w0, v);
        if constexpr (HAD) fwht16(v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            amax = fmaxf(amax, fabsf(v[i]));
            if constexpr (MINMAX) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
        }
        widen16(w1, v);
        if constexpr (HAD) fwht16(v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            amax = fmaxf(amax, fabsf(v[i]));
            if constexpr (MINMAX) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
        }
    }
    if (c < n_chunks) {
        float v[16];
        load16(x, (uint32_t)c, v);
        if constexpr (HAD) fwht16(v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            amax = fmaxf(amax, fabsf(v[i]));
            if constexpr (MINMAX) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
        }
    }
    // min / max start from 0: only min(min, 0) and max(max, 0) are ever used.
    amax = warp_maxf(amax);
    if constexpr (MINMAX) { mn = warp_minf(mn); mx = warp_maxf(mx); }
    __shared__ float sh[3][32];
    __shared__ bool is_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (lane == 0) { sh[0][warp] = amax; sh[1][warp] = mn; sh[2][warp] = mx; }
    __syncthreads();
    RangeSlot* slots = ws_range(ws);
    WsHeader* h = ws_header(ws);
    if (threadIdx.x == 0) {
        float a = 0.0f, lo = 0.0f, hi = 0.0f;
        for (int w = 0; w < nw; ++w) { a = fmaxf(a, sh[0][w]); lo = fminf(lo, sh[1][w]); hi = fmaxf(hi, sh[2][w]); }
        slots[blockIdx.x] = RangeSlot{a, lo, hi, 0.0f};
        __threadfence();
        is_last = (atomicAdd(&h->counter_range, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    float a = 0.0f, lo = 0.0f, hi = 0.0f;
    for (unsigned i = threadIdx.x; i < gridDim.x; i += blockDim.x) {
        const float* p = reinterpret_cast<const float*>(&slots[i]);
        a = fmaxf(a, __ldcg(p)); lo = fminf(lo, __ldcg(p + 1)); hi = fmaxf(hi, __ldcg(p + 2));
    }
    a = warp_maxf(a); lo = warp_minf(lo); hi = warp_maxf(hi);
    __syncthreads();
    if (lane == 0) { sh[0][warp] = a; sh[1][warp] = lo; sh[2][warp] = hi; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 0; w < nw; ++w) { a = fmaxf(a, sh[0][w]); lo = fminf(lo, sh[1][w]); hi = fmaxf(hi, sh[2][w]); }
        h->amax = a; h->vmin = lo; h->vmax = hi;
        h->counter_range = 0u;
    }
}

// ---------------------------------------------------------------------------
// One chunk of the flat quantize kernel.
// ---------------------------------------------------------------------------

struct TensorCtx {
    float amax;          // per-tensor / NV: amax of the (rotated) tensor
    PlainScale ps;       // per-tensor plain scale
    Recip rc;            // per-tensor reciprocal bracket
    float S;             // NV tensor scale
};

template <int FMT, int GK, bool HAD, bool STATS>
__device__ __forceinline__ void flat_chunk(const uint32_t (&win)[8], uint32_t c, bool valid, const FlatArgs& a,
                                           const TensorCtx& tc, Acc& acc, int lane)
{
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    float y[16];
    widen16(win, y);
    if constexpr (HAD) fwht16(y);

    uint32_t w[NW];
    float xh[16];

    if constexpr (GK == K_TENSOR) {
        quant_plain_chunk<FMT, STATS>(y, tc.ps, tc.rc, F::qmin, F::qmax, w, xh);
    } else {
        // range of this lane's 16 values, then of its unit
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            amax = fmaxf(amax, fabsf(y[i]));
            if constexpr (F::asym) { mn = fminf(mn, y[i]); mx = fmaxf(mx, y[i]); }
        }
        int T;
        if constexpr (GK == K_NV) T = 1;
        else if constexpr (GK == K_MX) T = 2;
        else T = a.lanes_per_group;
        for (int o = 1; o < T; o <<= 1) {
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            if constexpr (F::asym) {
                mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
            }
        }
        const bool leader = (lane & (T - 1)) == 0;

        if constexpr (GK == K_GROUP) {
            const PlainScale ps = plain_scale<FMT>(amax, mn, mx, a.scale_fp16 != 0);
            const Recip R = make_recip(ps.s, ps.bound);
            quant_plain_chunk<FMT, STATS>(y, ps, R, F::qmin, F::qmax, w, xh);
            if (valid && leader) store_plain_scale<FMT>(a.scales, a.zps, c >> (__ffs(T) - 1), ps, a.scale_fp16 != 0);
        } else if constexpr (GK == K_MX) {
            const int e = ue8m0_exponent<FMT>(amax);
            const float p2 = exp2i(-e), pe = exp2i(e);
            if constexpr (F::is_int) {
                float q[16];
                quant_int8_chunk_pow2(y, p2, *reinterpret_cast<uint32_t(*)[4]>(&w), q);
                if constexpr (STATS) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(q[i], pe);
                }
            } else {
                float val[16];
                quant_fp_chunk_pow2<FMT, STATS>(y, p2, w, val);
                if constexpr (STATS) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(val[i], pe);
                }
            }
            if (valid && leader) reinterpret_cast<uint8_t*>(a.scales)[c >> 1] = (uint8_t)(e + 127);
        } else {  // K_NV
            uint32_t sbc = 0;
            float sbv = 0.0f;
            if (tc.S > 0.0f) {
                const float sb32 = __fdiv_rn(__fdiv_rn(amax, F::qscale), tc.S);
                sbc = e4m3_code(sb32);
                sbv = e4m3_value(sbc);
            }
            const float d = __fmul_rn(sbv, tc.S);
            if (valid) reinterpret_cast<uint8_t*>(a.scales)[c] = (uint8_t)sbc;
            if (d > 0.0f) {
                const Recip R = make_recip(d, amax);
                if constexpr (F::is_int) {
                    float qz[16];
                    quant_int_chunk<FMT, STATS>(y, R, 0.0f, -7, 7, w, qz);
                    if constexpr (STATS) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(__fmul_rn(qz[i], sbv), tc.S);
                    }
                } else {
                    float val[16];
                    quant_fp_chunk<FMT, STATS>(y, R, w, val);
                    if constexpr (STATS) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(__fmul_rn(val[i], sbv), tc.S);
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < NW; ++k) w[k] = 0u;
#pragma unroll
                for (int i = 0; i < 16; ++i) xh[i] = 0.0f;
            }
        }

        if constexpr (STATS) {
            // crest factor of the unit: amax / sqrt(mean y^2)
            float ss = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) ss = __fmaf_rn(y[i], y[i], ss);
            for (int o = 1; o < T; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
            if (valid && leader) kappa_add(acc, amax, ss, a.inv_unit);
        }
    }

    if (valid) {
        store_codes<FMT>(a.codes, c, w);
        if constexpr (STATS) {
            float e2, x2;
            chunk_sums(y, xh, e2, x2);
            acc.err2 += (double)e2;
            acc.x2 += (double)x2;
        }
    }
}

template <int FMT, int GK, bool HAD, bool STATS>
__global__ void __launch_bounds__(256) k_quant_flat(const FlatArgs a)
{
    using F = Fmt<FMT>;
    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;

    TensorCtx tc{};
    if constexpr (GK == K_TENSOR || GK == K_NV) {
        const WsHeader* h = ws_header(a.ws);
        tc.amax = h->amax;
        if constexpr (GK == K_TENSOR) {
            tc.ps = plain_scale<FMT>(h->amax, h->vmin, h->vmax, a.scale_fp16 != 0);
            tc.rc = make_recip(tc.ps.s, tc.ps.bound);
            if (blockIdx.x == 0 && threadIdx.x == 0) store_plain_scale<FMT>(a.scales, a.zps, 0, tc.ps, a.scale_fp16 != 0);
        } else {
            tc.S = __fdiv_rn(h->amax, F::qscale * 448.0f);
            if (blockIdx.x == 0 && threadIdx.x == 0) a.tensor_scale[0] = tc.S;
        }
    }

    Acc acc;
    for (uint32_t t = warp; t < a.n_dtiles; t += nwarps) {
        const uint32_t c0 = t * 64 + lane, c1 = c0 + 32;
        const bool v0 = c0 < a.n_chunks, v1 = c1 < a.n_chunks;
        uint32_t w0[8], w1[8];
        if (v0) ld_nc_v8(a.x + (size_t)c0 * 8, w0);
        else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w0[i] = 0u;
        }
        if (v1) ld_nc_v8(a.x + (size_t)c1 * 8, w1);
        else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w1[i] = 0u;
        }
        flat_chunk<FMT, GK, HAD, STATS>(w0, c0, v0, a, tc, acc, lane);
        flat_chunk<FMT, GK, HAD, STATS>(w1, c1, v1, a, tc, acc, lane);
    }

    if constexpr (STATS) {
        // per-tensor kappa comes from the totals: amax / sqrt(sum y^2 / n)
        acc.ss = acc.x2;
        finish_stats(acc, a.ws, a.stats, GK == K_TENSOR, tc.amax, a.n_elems, true);
    }
}

// ---------------------------------------------------------------------------
// Launchers.
// ---------------------------------------------------------------------------

namespace {

// Resident CTAs per SM of one kernel at one block size (cached per instantiation).
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

// Grid of at most one wave (SM count x resident CTAs), at least enough CTAs to give
// each min_items_per_cta items, capped at the workspace slot count.
template <auto KERN, int BLOCK>
unsigned grid_for(uint64_t min_items_per_cta, uint64_t total_items)
{
    const uint64_t waves = (uint64_t)device_sm_count() * (uint64_t)resident_ctas<KERN, BLOCK>();
    uint64_t need = (total_items + min_items_per_cta - 1) / min_items_per_cta;
    if (need < 1) need = 1;
    uint64_t g = need < waves ? need : waves;
    if (g > (uint64_t)MAX_GRID) g = MAX_GRID;
    return (unsigned)g;
}

template <int FMT, int GK, bool HAD, bool STATS>
cudaError_t run_flat(const FlatArgs& a, cudaStream_t st)
{
    constexpr int block = 256;
    constexpr auto kern = k_quant_flat<FMT, GK, HAD, STATS>;
    // one warp step = 64 chunks; a CTA of 8 warps takes 8 steps per sweep
    const unsigned grid = grid_for<kern, block>(8, a.n_dtiles);
    kern<<<grid, block, 0, st>>>(a);
    return cudaGetLastError();
}

template <int FMT, int GK>
cudaError_t run_flat_hs(bool had, bool stats, const FlatArgs& a, cudaStream_t st)
{
    if (had) return stats ? run_flat<FMT, GK, true, true>(a, st) : run_flat<FMT, GK, true, false>(a, st);
    return stats ? run_flat<FMT, GK, false, true>(a, st) : run_flat<FMT, GK, false, false>(a, st);
}

template <bool HAD, bool MINMAX>
cudaError_t run_range(const uint32_t* x, uint32_t n_chunks, uint8_t* ws, cudaStream_t st)
{
    constexpr int block = 256;
    constexpr auto kern = k_range<HAD, MINMAX>;
    const unsigned grid = grid_for<kern, block>((uint64_t)block * 4, n_chunks);
    kern<<<grid, block, 0, st>>>(x, n_chunks, ws);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_range(const uint32_t* x, uint32_t n_chunks, bool had, bool minmax, uint8_t* ws, cudaStream_t st)
{
    if (had) return minmax ? run_range<true, true>(x, n_chunks, ws, st) : run_range<true, false>(x, n_chunks, ws, st);
    return minmax ? run_range<false, true>(x, n_chunks, ws, st) : run_range<false, false>(x, n_chunks, ws, st);
}

cudaError_t launch_quant_flat(int fmt, int kind, bool had, bool stats, const FlatArgs& a, cudaStream_t st)
{
    switch (kind) {
    case K_TENSOR:
    case K_GROUP:
        switch (fmt) {
        case BQ_INT8_SYM:   return kind == K_TENSOR ? run_flat_hs<BQ_INT8_SYM, K_TENSOR>(had, stats, a, st) : run_flat_hs<BQ_INT8_SYM, K_GROUP>(had, stats, a, st);
        case BQ_INT8_ASYM:  return kind == K_TENSOR ? run_flat_hs<BQ_INT8_ASYM, K_TENSOR>(had, stats, a, st) : run_flat_hs<BQ_INT8_ASYM, K_GROUP>(had, stats, a, st);
        case BQ_INT4_SYM:   return kind == K_TENSOR ? run_flat_hs<BQ_INT4_SYM, K_TENSOR>(had, stats, a, st) : run_flat_hs<BQ_INT4_SYM, K_GROUP>(had, stats, a, st);
        case BQ_UINT4_ASYM: return kind == K_TENSOR ? run_flat_hs<BQ_UINT4_ASYM, K_TENSOR>(had, stats, a, st) : run_flat_hs<BQ_UINT4_ASYM, K_GROUP>(had, stats, a, st);
        case BQ_FP8_E4M3:   return kind == K_TENSOR ? run_flat_hs<BQ_FP8_E4M3, K_TENSOR>(had, stats, a, st) : run_flat_hs<BQ_FP8_E4M3, K_GROUP>(had, stats, a, st);
        case BQ_FP8_E5M2:   return kind == K_TENSOR ? run_flat_hs<BQ_FP8_E5M2, K_TENSOR>(had, stats, a, st) : run_flat_hs<BQ_FP8_E5M2, K_GROUP>(had, stats, a, st);
        default: return cudaErrorInvalidValue;
        }
    case K_MX:
        switch (fmt) {
        case BQ_INT8_SYM: return run_flat_hs<BQ_INT8_SYM, K_MX>(had, stats, a, st);
        case BQ_FP8_E4M3: return run_flat_hs<BQ_FP8_E4M3, K_MX>(had, stats, a, st);
        case BQ_FP8_E5M2: return run_flat_hs<BQ_FP8_E5M2, K_MX>(had, stats, a, st);
        case BQ_FP4_E2M1: return run_flat_hs<BQ_FP4_E2M1, K_MX>(had, stats, a, st);
        default: return cudaErrorInvalidValue;
        }
    case K_NV:
        switch (fmt) {
        case BQ_FP4_E2M1: return run_flat_hs<BQ_FP4_E2M1, K_NV>(had, stats, a, st);
        case BQ_INT4_SYM: return run_flat_hs<BQ_INT4_SYM, K_NV>(had, stats, a, st);
        default: return cudaErrorInvalidValue;
        }
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace bq
