// quant_flat.cu -- one-pass quantize kernels over the tensor seen as a flat run of
// 16-element chunks: per-tensor (after the range pass), per-group, MX block-32 and
// NV block-16 granularities; and the per-tensor range pass itself.
//
// Layout of the work: lane l of a warp owns a span of four consecutive chunks (64
// elements, 128 bytes) of the warp's 2048-element tile. Scaling units of 16, 32 or 64
// elements are lane-local; a unit of G >= 128 elements spans G/64 adjacent lanes and
// is reduced with xor shuffles. The grid is at most one wave (SM count x resident
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
//
// Lane l of a warp owns a span of four consecutive chunks (64 elements, 128 bytes,
// four 256-bit loads, all issued before any arithmetic) of the warp's 2048-element
// tile; two CTAs of eight warps per SM keep 64 KB of loads in flight.
// ---------------------------------------------------------------------------

constexpr int SPAN = 4;   // chunks per lane per tile

struct TensorCtx {
    float amax;          // per-tensor / NV: amax of the (rotated) tensor
    PlainScale ps;       // per-tensor plain scale
    float S;             // NV tensor scale
    float cS;            // ~ 1 / (Qmax * S) for the NV block-scale bracket
};

// Widen (and rotate) one chunk.
template <bool HAD>
__device__ __forceinline__ void chunk_in(const uint32_t (&w)[8], float2 (&y)[8])
{
    widen16x2(w, y);
    if constexpr (HAD) fwht16x2(y);
}

// Range of chunks [c0, c0 + N) of the lane's span: amax, or min and max (asymmetric).
template <bool HAD, bool ASYM, int N>
__device__ __forceinline__ void span_range(const uint32_t (&w)[SPAN][8], int c0, float& amax, float& mn, float& mx)
{
    if constexpr (HAD) {
        amax = 0.0f; mn = 0.0f; mx = 0.0f;
#pragma unroll
        for (int k = 0; k < N; ++k) {
            float2 y[8];
            chunk_in<true>(w[c0 + k], y);
            if constexpr (ASYM) chunk_minmax(y, mn, mx);
            else amax = chunk_amax(y, amax);
        }
        if constexpr (ASYM) amax = fmaxf(-mn, mx);
    } else if constexpr (ASYM) {
        uint32_t lo = 0u, hi = 0u;          // bf16 pair (+0, +0)
#pragma unroll
        for (int k = 0; k < N; ++k) words_minmax(w[c0 + k], lo, hi);
        mn = pair_min(lo);
        mx = pair_max(hi);
        amax = fmaxf(-mn, mx);
    } else {
        uint32_t m = 0u;
#pragma unroll
        for (int k = 0; k < N; ++k) m = words_absmax(w[c0 + k], m);
        amax = pair_absmax(m);
        mn = mx = 0.0f;
    }
}

// NV block scale: s_b = E4M3((amax / Qmax) / S), d = s_b * S. The E4M3 code is taken
// from the bracket amax * c (1 -+ 2^-20), c ~ 1 / (Qmax S) within 2^-23, which holds
// RN(RN(amax / Qmax) / S) strictly inside; where the two codes differ it divides.
template <int FMT>
__device__ __forceinline__ uint32_t nv_scale_code(float amax, float S, float cS)
{
    using F = Fmt<FMT>;
    if (!(S > 0.0f)) return 0u;
    const float a = __fmul_rn(amax, cS);
    const uint32_t pair = cvt_pair<BQ_FP8_E4M3>(__fmul_rn(a, BRACKET_HI), __fmul_rn(a, BRACKET_LO));
    const uint32_t lo = pair & 0xFFu, hi = pair >> 8;
    if (lo == hi && S >= 0x1p-100f && S <= 1.0e30f) return lo;
    return e4m3_code(__fdiv_rn(__fdiv_rn(amax, F::qscale), S));
}

// Codes of chunk k of the lane's span: 4-bit codes are gathered for one 32-byte store
// per span, 8-bit codes are stored right away (16 bytes per chunk).
template <int FMT>
__device__ __forceinline__ void put_codes(uint32_t (&span4)[8], uint8_t* codes, uint32_t c, bool valid, int k,
                                          const uint32_t (&w)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) {
        span4[2 * k] = w[0];
        span4[2 * k + 1] = w[1];
    } else {
        if (valid) st_v4(codes + (size_t)c * 16, w);
    }
}

// One lane's span under the per-tensor unit.
template <int FMT, bool HAD, bool STATS>
__device__ __forceinline__ void span_tensor(const uint32_t (&w)[SPAN][8], uint32_t span, const FlatArgs& a,
                                            const PlainUnit<FMT>& u, float p, double inv_p2, bool scaled,
                                            Acc& acc, uint32_t (&span4)[8])
{
    float2 e2 = splat(0.0f), x2 = splat(0.0f);
    const bool exact_res = !HAD && a.scale_fp16 != 0;
#pragma unroll
    for (int k = 0; k < SPAN; ++k) {
        float2 y[8];
        uint32_t q[CodeWords<FMT>::n];
        chunk_in<HAD>(w[k], y);
        if (scaled) plain_chunk<FMT, STATS, true>(y, u, p, exact_res, q, e2, x2);
        else plain_chunk<FMT, STATS, false>(y, u, p, exact_res, q, e2, x2);
        const uint32_t c = SPAN * span + k;
        put_codes<FMT>(span4, a.codes, c, c < a.n_chunks, k, q);
    }
    if constexpr (STATS) add_unit_sums(acc, e2, x2, scaled ? inv_p2 : 1.0);
}

// Units of N chunks (N = 1, 2 or 4) inside the lane's span; with N = 4 a unit can
// also span T lanes (T = 1, 2, 4, 8: groups of 64 .. 512). A one-chunk unit is widened
// (and rotated) once; larger units take their range from the raw bf16 words (or, when
// rotated, from a first rotation) and widen again to quantize, which keeps register
// pressure low.
template <int FMT, int GK, bool HAD, bool STATS, int N>
__device__ __forceinline__ void span_units(const uint32_t (&w)[SPAN][8], uint32_t span, const FlatArgs& a,
                                           const TensorCtx& tc, Acc& acc, int lane, int T,
                                           uint32_t (&span4)[8], uint8_t (&scode)[SPAN])
{
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    constexpr bool GASYM = F::asym && GK == K_GROUP;
#pragma unroll
    for (int base = 0; base < SPAN; base += N) {
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
        float2 y1[8];                      // the chunk of a one-chunk unit
        if constexpr (N == 1) {
            chunk_in<HAD>(w[base], y1);
            if constexpr (GASYM) { chunk_minmax(y1, mn, mx); amax = fmaxf(-mn, mx); }
            else amax = chunk_amax(y1, 0.0f);
        } else {
            span_range<HAD, GASYM, N>(w, base, amax, mn, mx);
        }
        if (N == SPAN && T > 1) {
            for (int o = 1; o < T; o <<= 1) {
                if constexpr (GASYM) {
                    mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
                    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                } else {
                    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                }
            }
            if constexpr (GASYM) amax = fmaxf(-mn, mx);
        }
        const bool scaled = STATS && __any_sync(0xFFFFFFFFu, !plain_sums_ok(amax));
        const Pow2 pw = pow2_for(amax);
        const float p = scaled ? pw.p : 1.0f;
        float2 e2 = splat(0.0f), x2 = splat(0.0f);

        if constexpr (GK == K_MX) {
            const int e = ue8m0_exponent<FMT>(amax);
            const float p2 = exp2i(-e), pe = exp2i(e);
#pragma unroll
            for (int k = 0; k < N; ++k) {
                float2 y[8], z[8];
                uint32_t q[NW];
                if constexpr (N == 1) { for (int i = 0; i < 8; ++i) y[i] = y1[i]; }
                else chunk_in<HAD>(w[base + k], y);
                if constexpr (F::is_int) {
                    int8_chunk_pow2<STATS>(y, p2, *reinterpret_cast<uint32_t(*)[4]>(&q), z);
                    if constexpr (STATS) {
                        if (scaled) int_sums<true>(y, z, pe, p, e2, x2);
                        else int_sums<false>(y, z, pe, p, e2, x2);
                    }
                } else {
                    fp_chunk_pow2<FMT, STATS>(y, p2, q, z);
                    if constexpr (STATS) {
                        if (scaled) val_sums<true>(y, z, pe, p, e2, x2);
                        else val_sums<false>(y, z, pe, p, e2, x2);
                    }
                }
                const uint32_t c = SPAN * span + base + k;
                put_codes<FMT>(span4, a.codes, c, c < a.n_chunks, base + k, q);
            }
            scode[base] = (uint8_t)(e + 127);
        } else if constexpr (GK == K_NV) {
            // N == 1
            const uint32_t sbc = nv_scale_code<FMT>(amax, tc.S, tc.cS);
            const float sbv = e4m3_value(sbc);
            const float d = __fmul_rn(sbv, tc.S);
            scode[base] = (uint8_t)sbc;
            uint32_t q[NW];
            if constexpr (F::is_int) {
                const IntQ iq = int_unit<FMT>(d, 0.0f, -amax, amax, -7, 7);
                float2 nq[8];
                int_chunk<FMT, STATS>(y1, iq, -7, 7, q, nq);
                if constexpr (STATS) {
                    // x-hat = (q s_b) S: the first product is exact
                    float2 val[8];
                    const float2 nA = splat(-sbv);
#pragma unroll
                    for (int i = 0; i < 8; ++i) val[i] = mul2(nq[i], nA);
                    if (scaled) val_sums<true>(y1, val, tc.S, p, e2, x2);
                    else val_sums<false>(y1, val, tc.S, p, e2, x2);
                }
            } else {
                const FpQ fq = fp_unit(d, amax);
                float2 val[8];
                fp_chunk<FMT, STATS>(y1, fq, q, val);
                if constexpr (STATS) {
                    const float2 A = splat(fq.zero ? 0.0f : sbv);
#pragma unroll
                    for (int i = 0; i < 8; ++i) val[i] = mul2(val[i], A);
                    if (scaled) val_sums<true>(y1, val, tc.S, p, e2, x2);
                    else val_sums<false>(y1, val, tc.S, p, e2, x2);
                }
            }
            {
                const uint32_t c = SPAN * span + base;
                put_codes<FMT>(span4, a.codes, c, c < a.n_chunks, base, q);
            }
        } else {  // K_GROUP
            const bool f16 = a.scale_fp16 != 0;
            const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
            const PlainUnit<FMT> u = plain_unit<FMT>(ps);
            const bool exact_res = !HAD && f16;
#pragma unroll
            for (int k = 0; k < N; ++k) {
                float2 y[8];
                uint32_t q[NW];
                if constexpr (N == 1) { for (int i = 0; i < 8; ++i) y[i] = y1[i]; }
                else chunk_in<HAD>(w[base + k], y);
                if (scaled) plain_chunk<FMT, STATS, true>(y, u, p, exact_res, q, e2, x2);
                else plain_chunk<FMT, STATS, false>(y, u, p, exact_res, q, e2, x2);
                const uint32_t c = SPAN * span + base + k;
                put_codes<FMT>(span4, a.codes, c, c < a.n_chunks, base + k, q);
            }
            // the leader of the unit stores its scale
            const uint32_t c_first = SPAN * span + base;
            const bool leader = (N < SPAN) || ((lane & (T - 1)) == 0);
            if (leader && c_first < a.n_chunks) {
                const uint32_t unit = (N < SPAN) ? c_first / N : span / (uint32_t)T;
                store_plain_scale<FMT>(a.scales, a.zps, unit, ps, f16);
            }
        }

        if constexpr (STATS) {
            const uint32_t c_first = SPAN * span + base;
            const bool valid = c_first < a.n_chunks;
            if (valid) add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
            float ss = __fadd_rn(x2.x, x2.y);
            if (N == SPAN && T > 1)
                for (int o = 1; o < T; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
            const bool leader = (N < SPAN) || ((lane & (T - 1)) == 0);
            if (valid && leader) kappa_add(acc, __fmul_rn(amax, p), ss, a.inv_unit);
        }
    }
}

__device__ __forceinline__ void load_span(const uint32_t* x, uint32_t span, uint32_t n_chunks, uint32_t (&w)[SPAN][8])
{
    const uint32_t c0 = SPAN * span;
    if (c0 + SPAN <= n_chunks) {
#pragma unroll
        for (int k = 0; k < SPAN; ++k) ld_nc_v8(x + (size_t)(c0 + k) * 8, w[k]);
    } else {
#pragma unroll
        for (int k = 0; k < SPAN; ++k) {
            if (c0 + k < n_chunks) ld_nc_v8(x + (size_t)(c0 + k) * 8, w[k]);
            else {
#pragma unroll
                for (int i = 0; i < 8; ++i) w[k][i] = 0u;
            }
        }
    }
}

// Store a span's gathered 4-bit codes: one 32-byte store when the span is whole, chunk
// by chunk at the ragged end.
template <int FMT>
__device__ __forceinline__ void store_span4(uint8_t* codes, uint32_t span, uint32_t n_chunks, const uint32_t (&v)[8])
{
    if constexpr (Fmt<FMT>::four) {
        const uint32_t c0 = SPAN * span;
        if (c0 + SPAN <= n_chunks) {
            st_v8(codes + (size_t)span * 32, v);
        } else {
#pragma unroll
            for (int k = 0; k < SPAN; ++k)
                if (c0 + k < n_chunks) {
                    const uint32_t w2[2] = {v[2 * k], v[2 * k + 1]};
                    st_v2(codes + (size_t)(c0 + k) * 8, w2);
                }
        }
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
    PlainUnit<FMT> tu{};
    Pow2 tp{1.0f, 1.0};
    bool tscaled = false;
    if constexpr (GK == K_TENSOR || GK == K_NV) {
        const WsHeader* h = ws_header(a.ws);
        tc.amax = h->amax;
        if constexpr (GK == K_TENSOR) {
            tc.ps = plain_scale<FMT>(h->amax, h->vmin, h->vmax, a.scale_fp16 != 0);
            tu = plain_unit<FMT>(tc.ps);
            tp = pow2_for(tc.amax);
            tscaled = STATS && !plain_sums_ok(tc.amax);
            if (blockIdx.x == 0 && threadIdx.x == 0) store_plain_scale<FMT>(a.scales, a.zps, 0, tc.ps, a.scale_fp16 != 0);
        } else {
            tc.S = __fdiv_rn(h->amax, F::qscale * 448.0f);
            tc.cS = rcp_approx(__fmul_rn(F::qscale, tc.S));
            if (blockIdx.x == 0 && threadIdx.x == 0) a.tensor_scale[0] = tc.S;
        }
    }
    // per-group units: 16 elements (N = 1), 32 (N = 2), 64 and up (N = 4, T lanes)
    const int T = (GK == K_GROUP && a.lanes_per_group > 0) ? a.lanes_per_group : 1;

    Acc acc;
    for (uint32_t t = warp; t < a.n_dtiles; t += nwarps) {
        const uint32_t span = t * 32 + lane;
        uint32_t cur[SPAN][8];
        load_span(a.x, span, a.n_chunks, cur);
        uint32_t span4[8];
        uint8_t scode[SPAN] = {0, 0, 0, 0};

        if constexpr (GK == K_TENSOR) {
            span_tensor<FMT, HAD, STATS>(cur, span, a, tu, tp.p, tp.inv_p2, tscaled, acc, span4);
        } else if constexpr (GK == K_NV) {
            span_units<FMT, GK, HAD, STATS, 1>(cur, span, a, tc, acc, lane, 1, span4, scode);
        } else if constexpr (GK == K_MX) {
            span_units<FMT, GK, HAD, STATS, 2>(cur, span, a, tc, acc, lane, 1, span4, scode);
        } else {
            if (a.lanes_per_group == 0) span_units<FMT, GK, HAD, STATS, 1>(cur, span, a, tc, acc, lane, 1, span4, scode);
            else if (a.lanes_per_group < 0) span_units<FMT, GK, HAD, STATS, 2>(cur, span, a, tc, acc, lane, 1, span4, scode);
            else span_units<FMT, GK, HAD, STATS, SPAN>(cur, span, a, tc, acc, lane, T, span4, scode);
        }

        store_span4<FMT>(a.codes, span, a.n_chunks, span4);
        const uint32_t c0 = SPAN * span;
        if constexpr (GK == K_NV) {
            // four E4M3 block scales, one per chunk
            uint8_t* sc = reinterpret_cast<uint8_t*>(a.scales);
            if (c0 + SPAN <= a.n_chunks)
                *reinterpret_cast<uint32_t*>(sc + c0) = (uint32_t)scode[0] | ((uint32_t)scode[1] << 8) |
                                                        ((uint32_t)scode[2] << 16) | ((uint32_t)scode[3] << 24);
            else
                for (int k = 0; k < SPAN; ++k)
                    if (c0 + k < a.n_chunks) sc[c0 + k] = scode[k];
        } else if constexpr (GK == K_MX) {
            uint8_t* sc = reinterpret_cast<uint8_t*>(a.scales);
            if (c0 + SPAN <= a.n_chunks)
                *reinterpret_cast<uint16_t*>(sc + c0 / 2) = (uint16_t)(scode[0] | (scode[2] << 8));
            else if (c0 < a.n_chunks)
                sc[c0 / 2] = scode[0];
        }
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
