// quant_flat.cu -- one-pass quantize kernels over the tensor seen as a flat run of
// 16-element chunks: per-tensor (after the range pass), per-group, MX block-32 and
// NV block-16 granularities; and the per-tensor range pass itself.
//
// Layout of the work: lane l of a warp owns a span of two consecutive chunks (32
// elements, 64 bytes, two 256-bit loads) of the warp's 1024-element tile; the next
// tile's span is loaded before the current one is processed, so every lane keeps 64
// bytes in flight while it computes. A scaling unit of G >= 32 elements spans G/32
// adjacent lanes and is reduced with xor shuffles; 16-element units (NV blocks,
// groups of 16) are lane-local. The grid is at most one wave (SM count x resident
// CTAs) striding over the tiles.
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
__device__ __forceinline__ void range_chunk(const uint32_t (&w)[8], float& amax, float& mn, float& mx)
{
    float2 v[8];
    widen16x2(w, v);
    if constexpr (HAD) fwht16x2(v);
    amax = chunk_amax(v, amax);
    if constexpr (MINMAX) chunk_minmax(v, mn, mx);
}

template <bool HAD, bool MINMAX>
__global__ void __launch_bounds__(256) k_range(const uint32_t* __restrict__ x, uint32_t n_chunks, uint8_t* ws)
{
    float amax = 0.0f, mn = 0.0f, mx = 0.0f;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    uint64_t c = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; c + 3 * stride < n_chunks; c += 4 * stride) {
        uint32_t w0[8], w1[8], w2[8], w3[8];
        ld_nc_v8(x + c * 8, w0);
        ld_nc_v8(x + (c + stride) * 8, w1);
        ld_nc_v8(x + (c + 2 * stride) * 8, w2);
        ld_nc_v8(x + (c + 3 * stride) * 8, w3);
        range_chunk<HAD, MINMAX>(w0, amax, mn, mx);
        range_chunk<HAD, MINMAX>(w1, amax, mn, mx);
        range_chunk<HAD, MINMAX>(w2, amax, mn, mx);
        range_chunk<HAD, MINMAX>(w3, amax, mn, mx);
    }
    for (; c < n_chunks; c += stride) {
        uint32_t w0[8];
        ld_nc_v8(x + c * 8, w0);
        range_chunk<HAD, MINMAX>(w0, amax, mn, mx);
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
// Quantize kernel.
// ---------------------------------------------------------------------------

struct TensorCtx {
    float amax;          // per-tensor / NV: amax of the (rotated) tensor
    PlainScale ps;       // per-tensor plain scale
    UnitQ u;             // per-tensor unit
    Pow2 p2;             // per-tensor sum scaling
    float S;             // NV tensor scale
};

// Fold a unit's scaled fp32 sums into the lane's doubles.
__device__ __forceinline__ void add_unit_sums(Acc& acc, float2 e2, float2 x2, const Pow2& p)
{
    acc.err2 += (double)__fadd_rn(e2.x, e2.y) * p.inv_p2;
    acc.x2 += (double)__fadd_rn(x2.x, x2.y) * p.inv_p2;
}

// NV block scale: s_b = E4M3((amax / Qmax) / S), d = s_b * S.
template <int FMT>
__device__ __forceinline__ UnitQ nv_unit(float amax, float S, uint32_t& sbc, float& sbv)
{
    using F = Fmt<FMT>;
    sbc = 0;
    sbv = 0.0f;
    if (S > 0.0f) {
        const float sb32 = __fdiv_rn(__fdiv_rn(amax, F::qscale), S);
        sbc = e4m3_code(sb32);
        sbv = e4m3_value(sbc);
    }
    const float d = __fmul_rn(sbv, S);
    if constexpr (F::is_int) return int_unit(d, 0.0f, -amax, amax, -7, 7);
    UnitQ u;
    u.s = d;
    u.zpf = 0.0f;
    u.qmin = u.qmax = 0;
    u.zero = !(d > 0.0f);
    const Recip R = make_recip(d, amax);
    u.rlo = R.rlo;
    u.rhi = R.rhi;
    u.fast = R.fast;
    u.clamp_lo = u.clamp_hi = false;
    return u;
}

// Widen (and rotate) one chunk of a span.
template <bool HAD>
__device__ __forceinline__ void chunk_in(const uint32_t (&w)[8], float2 (&y)[8])
{
    widen16x2(w, y);
    if constexpr (HAD) fwht16x2(y);
}

// Codes of a span (two chunks) stored with one vector store: 32 bytes for 8-bit codes,
// 16 for 4-bit; a half span (the last chunk of an odd count) stores one chunk.
template <int FMT>
__device__ __forceinline__ void store_span(uint8_t* codes, uint32_t span, bool full,
                                           const uint32_t (&q0)[CodeWords<FMT>::n],
                                           const uint32_t (&q1)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) {
        uint8_t* p = codes + (size_t)span * 16;
        if (full) { const uint32_t w[4] = {q0[0], q0[1], q1[0], q1[1]}; st_v4(p, w); }
        else st_v2(p, q0);
    } else {
        uint8_t* p = codes + (size_t)span * 32;
        if (full) { const uint32_t w[8] = {q0[0], q0[1], q0[2], q0[3], q1[0], q1[1], q1[2], q1[3]}; st_v8(p, w); }
        else st_v4(p, q0);
    }
}

// QSNR sums of one chunk under a unit scaled by p (INT codes): d = (y - q s) p with the
// product q (s p) rounded once, e2 += d^2, x2 += (y p)^2.
__device__ __forceinline__ void int_sums(const float2 (&y)[8], const float2 (&qz)[8], float s, float p,
                                         float2& e2, float2& x2)
{
    const float2 P = splat(p), nSP = splat(-__fmul_rn(s, p));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 yp = mul2(y[i], P);
        const float2 d = fma2(qz[i], nSP, yp);
        e2 = fma2(d, d, e2);
        x2 = fma2(yp, yp, x2);
    }
}

// QSNR sums of one chunk from dequantized values xh.
__device__ __forceinline__ void val_sums(const float2 (&y)[8], const float2 (&xh)[8], float p, float2& e2, float2& x2)
{
    chunk_sums2(y, xh, p, e2, x2);
}

// Quantize one chunk under a known unit; codes to q, sums added to e2 / x2.
template <int FMT, bool STATS>
__device__ __forceinline__ void unit_chunk(const float2 (&y)[8], const UnitQ& u, float p,
                                           uint32_t (&q)[CodeWords<FMT>::n], float2& e2, float2& x2)
{
    using F = Fmt<FMT>;
    if constexpr (F::is_int) {
        float2 qz[8];
        int_chunk<FMT, STATS>(y, u, q, qz);
        if constexpr (STATS) int_sums(y, qz, u.s, p, e2, x2);
    } else {
        float2 xh[8];
        quant_unit_chunk<FMT, STATS>(y, u, q, xh);
        if constexpr (STATS) val_sums(y, xh, p, e2, x2);
    }
}

template <int FMT, int GK, bool HAD, bool STATS>
__device__ __forceinline__ void flat_span(const uint32_t (&w0)[8], const uint32_t (&w1)[8], uint32_t span,
                                          const FlatArgs& a, const TensorCtx& tc, Acc& acc, int lane)
{
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    const uint32_t c0 = 2 * span;
    const bool v0 = c0 < a.n_chunks, v1 = c0 + 1 < a.n_chunks;
    uint32_t q0[NW], q1[NW];

    if constexpr (GK == K_TENSOR) {
        float2 e2 = splat(0.0f), x2 = splat(0.0f);
        {
            float2 y[8];
            chunk_in<HAD>(w0, y);
            unit_chunk<FMT, STATS>(y, tc.u, tc.p2.p, q0, e2, x2);
        }
        {
            float2 y[8];
            chunk_in<HAD>(w1, y);
            // a missing second chunk reads as zeros and adds nothing to the sums
            unit_chunk<FMT, STATS>(y, tc.u, tc.p2.p, q1, e2, x2);
        }
        if constexpr (STATS) add_unit_sums(acc, e2, x2, tc.p2);
    } else if (GK == K_NV || (GK == K_GROUP && a.lanes_per_group == 0)) {
        // 16-element units: two per lane, each handled start to finish
        uint32_t scode[2] = {0u, 0u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 y[8];
            chunk_in<HAD>(h ? w1 : w0, y);
            uint32_t (&q)[NW] = h ? q1 : q0;
            const float m = chunk_amax(y, 0.0f);
            const Pow2 pw = pow2_for(m);
            float2 e2 = splat(0.0f), x2 = splat(0.0f);
            if constexpr (GK == K_NV) {
                uint32_t sbc;
                float sbv;
                const UnitQ u = nv_unit<FMT>(m, tc.S, sbc, sbv);
                scode[h] = sbc;
                if constexpr (F::is_int) {
                    float2 qz[8];
                    int_chunk<FMT, STATS>(y, u, q, qz);
                    if constexpr (STATS) {
                        const float2 A = splat(sbv), S2 = splat(tc.S);
                        float2 xh[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) xh[i] = mul2(mul2(qz[i], A), S2);
                        val_sums(y, xh, pw.p, e2, x2);
                    }
                } else {
                    float2 z[8];
                    fp_chunk<FMT, STATS>(y, u, q, z);
                    if constexpr (STATS) {
                        const float2 A = splat(sbv), S2 = splat(tc.S);
                        float2 xh[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) xh[i] = u.zero ? splat(0.0f) : mul2(mul2(z[i], A), S2);
                        val_sums(y, xh, pw.p, e2, x2);
                    }
                }
            } else {
                float mn = 0.0f, mx = 0.0f;
                if constexpr (F::asym) chunk_minmax(y, mn, mx);
                const bool f16 = a.scale_fp16 != 0;
                const PlainScale ps = plain_scale<FMT>(m, mn, mx, f16);
                const UnitQ u = unit_of_plain<FMT>(ps);
                unit_chunk<FMT, STATS>(y, u, pw.p, q, e2, x2);
                if (h ? v1 : v0) store_plain_scale<FMT>(a.scales, a.zps, c0 + h, ps, f16);
            }
            if constexpr (STATS) {
                if (h ? v1 : v0) {
                    add_unit_sums(acc, e2, x2, pw);
                    kappa_add(acc, __fmul_rn(m, pw.p), __fadd_rn(x2.x, x2.y), a.inv_unit);
                }
            }
        }
        if constexpr (GK == K_NV) {
            uint8_t* sc = reinterpret_cast<uint8_t*>(a.scales);
            if (v1) *reinterpret_cast<uint16_t*>(sc + c0) = (uint16_t)(scode[0] | (scode[1] << 8));
            else if (v0) sc[c0] = (uint8_t)scode[0];
        }
    } else {
        // units of 32 elements or more: one per lane (MX, groups of 32) or T lanes per
        // unit. Range first (the chunks are widened again for the quantize step, which
        // keeps register pressure low).
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 y[8];
            chunk_in<HAD>(h ? w1 : w0, y);
            if constexpr (F::asym) chunk_minmax(y, mn, mx);
            else amax = chunk_amax(y, amax);
        }
        const int T = (GK == K_MX) ? 1 : a.lanes_per_group;
        for (int o = 1; o < T; o <<= 1) {
            if constexpr (F::asym) {
                mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
            } else {
                amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            }
        }
        if constexpr (F::asym) amax = fmaxf(-mn, mx);
        const bool leader = (lane & (T - 1)) == 0;
        const Pow2 pw = pow2_for(amax);
        float2 e2 = splat(0.0f), x2 = splat(0.0f);
        if constexpr (GK == K_MX) {
            const int e = ue8m0_exponent<FMT>(amax);
            const float p2 = exp2i(-e);
            const float pe = exp2i(e);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float2 y[8], z[8];
                chunk_in<HAD>(h ? w1 : w0, y);
                uint32_t (&q)[NW] = h ? q1 : q0;
                if constexpr (F::is_int) {
                    int8_chunk_pow2<STATS>(y, p2, false, *reinterpret_cast<uint32_t(*)[4]>(&q), z);
                    if constexpr (STATS) int_sums(y, z, pe, pw.p, e2, x2);
                } else {
                    fp_chunk_pow2<FMT, STATS>(y, p2, q, z);
                    if constexpr (STATS) {
                        float2 xh[8];
                        const float2 PE = splat(pe);
#pragma unroll
                        for (int i = 0; i < 8; ++i) xh[i] = mul2(z[i], PE);
                        val_sums(y, xh, pw.p, e2, x2);
                    }
                }
            }
            if (v0) reinterpret_cast<uint8_t*>(a.scales)[span] = (uint8_t)(e + 127);
        } else {
            const bool f16 = a.scale_fp16 != 0;
            const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
            const UnitQ u = unit_of_plain<FMT>(ps);
            {
                float2 y[8];
                chunk_in<HAD>(w0, y);
                unit_chunk<FMT, STATS>(y, u, pw.p, q0, e2, x2);
            }
            {
                float2 y[8];
                chunk_in<HAD>(w1, y);
                unit_chunk<FMT, STATS>(y, u, pw.p, q1, e2, x2);
            }
            if (v0 && leader) store_plain_scale<FMT>(a.scales, a.zps, span / (uint32_t)T, ps, f16);
        }
        if constexpr (STATS) {
            if (v0) add_unit_sums(acc, e2, x2, pw);
            float ss = __fadd_rn(x2.x, x2.y);
            for (int o = 1; o < T; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
            if (v0 && leader) kappa_add(acc, __fmul_rn(amax, pw.p), ss, a.inv_unit);
        }
    }

    if (v0) store_span<FMT>(a.codes, span, v1, q0, q1);
}

__device__ __forceinline__ void load_span(const uint32_t* x, uint32_t span, uint32_t n_chunks,
                                          uint32_t (&w0)[8], uint32_t (&w1)[8])
{
    const uint32_t c0 = 2 * span;
    if (c0 + 1 < n_chunks) {
        ld_nc_v8(x + (size_t)c0 * 8, w0);
        ld_nc_v8(x + (size_t)c0 * 8 + 8, w1);
    } else {
        if (c0 < n_chunks) ld_nc_v8(x + (size_t)c0 * 8, w0);
        else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w0[i] = 0u;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) w1[i] = 0u;
    }
}

template <int FMT, int GK, bool HAD, bool STATS>
__global__ void __launch_bounds__(256, 2) k_quant_flat(const FlatArgs a)
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
            tc.u = unit_of_plain<FMT>(tc.ps);
            tc.p2 = pow2_for(tc.amax);
            if (blockIdx.x == 0 && threadIdx.x == 0) store_plain_scale<FMT>(a.scales, a.zps, 0, tc.ps, a.scale_fp16 != 0);
        } else {
            tc.S = __fdiv_rn(h->amax, F::qscale * 448.0f);
            if (blockIdx.x == 0 && threadIdx.x == 0) a.tensor_scale[0] = tc.S;
        }
    }

    Acc acc;
    // tile t covers spans 32 t .. 32 t + 31 (chunks 64 t .. 64 t + 63)
    uint32_t t = warp;
    uint32_t c0[8], c1[8];
    if (t < a.n_dtiles) load_span(a.x, t * 32 + lane, a.n_chunks, c0, c1);
    while (t < a.n_dtiles) {
        const uint32_t tn = t + nwarps;
        uint32_t n0[8], n1[8];
        if (tn < a.n_dtiles) load_span(a.x, tn * 32 + lane, a.n_chunks, n0, n1);
        flat_span<FMT, GK, HAD, STATS>(c0, c1, t * 32 + lane, a, tc, acc, lane);
#pragma unroll
        for (int i = 0; i < 8; ++i) { c0[i] = n0[i]; c1[i] = n1[i]; }
        t = tn;
    }

    if constexpr (STATS) {
        // per-tensor kappa comes from the totals: amax / sqrt(sum y^2 / n)
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
    // one tile per warp at least (8 tiles per CTA)
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
