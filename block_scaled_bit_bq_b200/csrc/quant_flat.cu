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
#include "tma.cuh"
#include "rot.cuh"
#include "rot64.cuh"
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
__global__ void __launch_bounds__(256) k_range(const uint32_t* __restrict__ x, uint32_t n_chunks, uint8_t* ws,
                                               float* out)
{
    pdl_wait();
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
    pdl_release();                   // the CTA's loads are done
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
        if (out) { out[0] = a; out[1] = lo; out[2] = hi; }
        h->counter_range = 0u;
    }
}

// ---------------------------------------------------------------------------
// Quantize kernel.
//
// A warp owns a 2048-element tile at a time (grid-stride over the tiles): 32 rows of
// 64 elements, lane l taking row l, a span of four consecutive 16-element chunks. The
// tiles reach shared memory through the tensor-memory-access unit (a 2-D tensor map
// over x seen as rows of 64 bf16, boxes of 32 rows, 128-byte swizzle), NST tiles ahead
// of the one being quantized, each completed on the warp's own mbarrier; the warps of
// a CTA never wait on each other. The 128-byte swizzle stores 16-byte unit u of row r
// at unit u ^ (r & 7), so the 32 lanes' 16-byte reads hit distinct banks.
// ---------------------------------------------------------------------------

#ifndef BQ_FLAT_WARPS
#define BQ_FLAT_WARPS 8
#endif
#ifndef BQ_FLAT_NST
#define BQ_FLAT_NST 2
#endif
#ifndef BQ_FLAT_MINB
#define BQ_FLAT_MINB 2
#endif

constexpr int SPAN = 4;                                    // chunks per lane per tile
constexpr int FLAT_WARPS = BQ_FLAT_WARPS;                  // warps per CTA
constexpr int NST = BQ_FLAT_NST;                           // tile buffers per warp
constexpr uint32_t ROW_BYTES = SPAN * 32;                  // 128
constexpr uint32_t TILE_BYTES = 32 * ROW_BYTES;            // 4 KiB
constexpr uint32_t FLAT_SMEM = FLAT_WARPS * NST * TILE_BYTES + 1024;

__device__ unsigned int g_flat_wait_timeouts = 0;

// A lane's row of the current tile buffer.
struct Row {
    uint32_t addr;      // shared address of the row
    uint32_t sw;        // row & 7 (the swizzle)
};

__device__ __forceinline__ void row_chunk(const Row& r, int k, uint32_t (&w)[8])
{
    const uint32_t u0 = (uint32_t)(2 * k) ^ r.sw, u1 = (uint32_t)(2 * k + 1) ^ r.sw;
    lds_v4(r.addr + (u0 << 4), w[0], w[1], w[2], w[3]);
    lds_v4(r.addr + (u1 << 4), w[4], w[5], w[6], w[7]);
}

__device__ __forceinline__ void row_put_chunk(const Row& r, int k, const uint32_t (&w)[8])
{
    const uint32_t u0 = (uint32_t)(2 * k) ^ r.sw, u1 = (uint32_t)(2 * k + 1) ^ r.sw;
    sts_v4(r.addr + (u0 << 4), w[0], w[1], w[2], w[3]);
    sts_v4(r.addr + (u1 << 4), w[4], w[5], w[6], w[7]);
}

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
    return e4m3_code(div_rn_call(div_rn_call(amax, F::qscale), S));
}

// Codes of chunk k (0..3, not a compile-time constant) of the lane's span: 4-bit codes
// are gathered for one 32-byte store per span, 8-bit codes are stored right away.
template <int FMT>
__device__ __forceinline__ void put_codes(uint32_t (&span4)[8], uint8_t* codes, size_t c, bool valid, int k,
                                          const uint32_t (&w)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) {
#pragma unroll
        for (int j = 0; j < SPAN; ++j) {
            span4[2 * j] = (j == k) ? w[0] : span4[2 * j];
            span4[2 * j + 1] = (j == k) ? w[1] : span4[2 * j + 1];
        }
    } else {
        if (valid) st_v4(codes + c * 16, w);
    }
}

// The chunks of a lane's span whose bit is set in `mask` through the general chunk path
// (clamping, scaled sums, exact settling of the elements the fast path could not
// decide); their sums are added to o.e2 / o.x2 and their codes stored (8-bit, chunks
// k < n_valid) or gathered into o.span4 (4-bit). Chunk k is chunk c_first + k of the
// tensor. Out of line and called once per span at most: the hot loops stay small.
// Warp-collective (every lane calls it, mask 0 for lanes with nothing to redo).
struct SpanOut {
    float2 e2, x2;
    uint32_t span4[8];
};

template <int FMT, bool HAD, bool STATS, bool EXACT>
__device__ __noinline__ SpanOut general_chunks(uint32_t row_addr, uint32_t sw, PlainUnit<FMT> u, bool scaled, float p,
                                               uint8_t* codes, size_t c_first, uint32_t mask, int n_valid, SpanOut o)
{
    const Row row{row_addr, sw};
    for (int k = 0; k < SPAN; ++k) {
        const bool mine = (mask >> k) & 1u;
        if (!__any_sync(0xFFFFFFFFu, mine)) continue;
        uint32_t w[8], q[CodeWords<FMT>::n];
        float2 y[8];
        float2 ce2 = splat(0.0f), cx2 = splat(0.0f);
        row_chunk(row, k, w);
        chunk_in<HAD>(w, y);
        plain_chunk<FMT, STATS, EXACT, true>(y, u, scaled, p, q, ce2, cx2);
        if (mine) {
            o.e2 = add2(o.e2, ce2);
            o.x2 = add2(o.x2, cx2);
            put_codes<FMT>(o.span4, codes, c_first + k, k < n_valid, k, q);
        }
    }
    return o;
}

// Hand a span's running sums and gathered codes to general_chunks and take them back.
template <int FMT, bool HAD, bool STATS, bool EXACT>
__device__ __forceinline__ void run_general(const Row& row, const PlainUnit<FMT>& u, bool scaled, float p,
                                            uint8_t* codes, size_t c_first, uint32_t mask, int n_valid,
                                            float2& e2, float2& x2, uint32_t (&span4)[8])
{
    SpanOut o;
    o.e2 = e2;
    o.x2 = x2;
#pragma unroll
    for (int i = 0; i < 8; ++i) o.span4[i] = span4[i];
    o = general_chunks<FMT, HAD, STATS, EXACT>(row.addr, row.sw, u, scaled, p, codes, c_first, mask, n_valid, o);
    e2 = o.e2;
    x2 = o.x2;
#pragma unroll
    for (int i = 0; i < 8; ++i) span4[i] = o.span4[i];
}

// Chunks [k0, k0 + n) of the lane's span through the fast path (codes placed, sums
// added; it decides every element). With `general` (the unit needs the general path as
// a whole) it does nothing and returns the mask of all n chunks; else 0.
template <int FMT, bool HAD, bool STATS, bool EXACT>
__device__ __forceinline__ uint32_t fast_chunks(const Row& row, const PlainUnit<FMT>& u, bool general, uint8_t* codes,
                                                size_t c_first, int k0, int n, int n_valid,
                                                float2& e2, float2& x2, uint32_t (&span4)[8])
{
    constexpr int NW = CodeWords<FMT>::n;
    if (general) return ((1u << n) - 1u) << k0;
#pragma unroll
    for (int k = k0; k < k0 + n; ++k) {
        uint32_t w[8], q[NW];
        float2 y[8], ce2, cx2;
        row_chunk(row, k, w);
        chunk_in<HAD>(w, y);
        (void)plain_chunk_fast<FMT, STATS, EXACT>(y, u, q, ce2, cx2);
        if constexpr (STATS) {
            e2 = add2(e2, ce2);
            x2 = add2(x2, cx2);
        }
        put_codes<FMT>(span4, codes, c_first + k, k < n_valid, k, q);
    }
    return 0u;
}

// A plain unit over chunks [k0, k0 + n) of the lane's span: fast path, then the
// general path for whatever it could not do.
template <int FMT, bool HAD, bool STATS, bool EXACT>
__device__ __forceinline__ void plain_unit_chunks(const Row& row, const PlainUnit<FMT>& u, bool scaled, float p,
                                                  uint8_t* codes, size_t c_first, int k0, int n, int n_valid,
                                                  float2& e2, float2& x2, uint32_t (&span4)[8])
{
    const bool general = unit_general_fast<FMT, EXACT>(u, scaled);
    const uint32_t redo = fast_chunks<FMT, HAD, STATS, EXACT>(row, u, general, codes, c_first, k0, n, n_valid,
                                                              e2, x2, span4);
    if (general) run_general<FMT, HAD, STATS, EXACT>(row, u, scaled, p, codes, c_first, redo, n_valid, e2, x2, span4);
}

// Leading chunks of span `span` inside the tensor (0..4).
__device__ __forceinline__ int span_valid(uint32_t span, uint32_t n_chunks)
{
    const uint32_t c0 = SPAN * span;
    return c0 >= n_chunks ? 0 : (n_chunks - c0 >= (uint32_t)SPAN ? SPAN : (int)(n_chunks - c0));
}

// Chunk sums of a unit into the lane's accumulators.
__device__ __forceinline__ void unit_done(Acc& acc, float2 e2, float2 x2, bool scaled, const Pow2& pw)
{
    add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
}

// ---- per-tensor unit -------------------------------------------------------

template <int FMT, bool HAD, bool STATS, bool EXACT>
__device__ __forceinline__ void span_tensor(const Row& row, uint32_t span, const FlatArgs& a,
                                            const PlainUnit<FMT>& u, const Pow2& tp, bool scaled, Acc& acc,
                                            uint32_t (&span4)[8])
{
    float2 e2 = splat(0.0f), x2 = splat(0.0f);
    plain_unit_chunks<FMT, HAD, STATS, EXACT>(row, u, scaled, scaled ? tp.p : 1.0f, a.codes, (size_t)SPAN * span, 0,
                                              SPAN, span_valid(span, a.n_chunks), e2, x2, span4);
    if constexpr (STATS) unit_done(acc, e2, x2, scaled, tp);
}

// ---- one-chunk units: NV block 16, groups of 16 ------------------------------

template <int FMT, int GK, bool HAD, bool STATS, bool EXACT>
__device__ __forceinline__ void span_n1(const Row& row, uint32_t span, const FlatArgs& a, const TensorCtx& tc,
                                        Acc& acc, uint32_t (&span4)[8], uint32_t& scodes)
{
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    constexpr bool GASYM = F::asym && GK == K_GROUP;
    const bool f16 = a.scale_fp16 != 0;
#pragma unroll 1
    for (int k = 0; k < SPAN; ++k) {
        uint32_t w[8], q[NW];
        float2 y[8];
        row_chunk(row, k, w);
        chunk_in<HAD>(w, y);
        float amax, mn = 0.0f, mx = 0.0f;
        if constexpr (GASYM) { chunk_minmax(y, mn, mx); amax = fmaxf(-mn, mx); }
        else amax = chunk_amax(y, 0.0f);
        const bool scaled = STATS && __any_sync(0xFFFFFFFFu, !plain_sums_ok(amax));
        const Pow2 pw = pow2_for(amax);
        const float p = scaled ? pw.p : 1.0f;
        float2 e2 = splat(0.0f), x2 = splat(0.0f);
        const uint32_t c = SPAN * span + k;
        bool valid = c < a.n_chunks;

        if constexpr (GK == K_NV) {
            const uint32_t sbc = nv_scale_code<FMT>(amax, tc.S, tc.cS);
            const float sbv = e4m3_value(sbc);
            const float d = __fmul_rn(sbv, tc.S);
            scodes |= sbc << (8 * k);
            if constexpr (F::is_int) {
                const IntQ iq = int_unit<FMT>(d, rcp_approx(d), false, 0.0f, -amax, amax, -7, 7);
                float2 nq[8];
                int_chunk<FMT, STATS>(y, iq, -7, 7, q, nq);
                if constexpr (STATS) {
                    // x-hat = (q s_b) S: the first product is exact
                    float2 val[8];
                    const float2 nA = splat(-sbv);
#pragma unroll
                    for (int i = 0; i < 8; ++i) val[i] = mul2(nq[i], nA);
                    if (scaled) val_sums<true>(y, val, tc.S, p, e2, x2);
                    else val_sums<false>(y, val, tc.S, p, e2, x2);
                }
            } else {
                const FpQ fq = fp_unit(d, amax);
                float2 val[8];
                fp_chunk<FMT, STATS>(y, fq, q, val);
                if constexpr (STATS) {
                    const float2 A = splat(fq.zero ? 0.0f : sbv);
#pragma unroll
                    for (int i = 0; i < 8; ++i) val[i] = mul2(val[i], A);
                    if (scaled) val_sums<true>(y, val, tc.S, p, e2, x2);
                    else val_sums<false>(y, val, tc.S, p, e2, x2);
                }
            }
        } else {
            const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
            const PlainUnit<FMT> u = plain_unit<FMT>(ps);
            // codes go straight to span4 / memory (valid = false below skips put_codes)
            plain_unit_chunks<FMT, HAD, STATS, EXACT>(row, u, scaled, p, a.codes, (size_t)SPAN * span, k, 1,
                                                      span_valid(span, a.n_chunks), e2, x2, span4);
            if constexpr (Fmt<FMT>::four) { q[0] = span4[2 * k]; q[1] = span4[2 * k + 1]; }
            else { valid = false; }
            if (c < a.n_chunks) store_plain_scale<FMT>(a.scales, a.zps, c, ps, f16);
        }
        put_codes<FMT>(span4, a.codes, c, valid, k, q);
        if constexpr (STATS) {
            if (c < a.n_chunks) {
                unit_done(acc, e2, x2, scaled, pw);
                kappa_add(acc, __fmul_rn(amax, p), __fadd_rn(x2.x, x2.y), a.inv_unit);
            }
        }
    }
}

// ---- NV block 16 ---------------------------------------------------------------

// One NV block through the general path (scaled sums, or a block scale outside the fast
// path's range): the residual-test integer codes with exact settling, or the bracketed
// FP codes with exact division where the bracket is inconclusive. Out of line.
struct NvOut {
    uint32_t w[2];
    float2 e2, x2;
};

template <int FMT, bool STATS>
__device__ __noinline__ NvOut nv_general(float2 y0, float2 y1, float2 y2, float2 y3, float2 y4, float2 y5, float2 y6,
                                         float2 y7, float amax, float sbv, float S, bool scaled, float p)
{
    using F = Fmt<FMT>;
    const float2 y[8] = {y0, y1, y2, y3, y4, y5, y6, y7};
    NvOut o;
    o.e2 = o.x2 = splat(0.0f);
    const float d = __fmul_rn(sbv, S);
    float2 val[8];
    if constexpr (F::is_int) {
        const IntQ iq = int_unit<FMT>(d, rcp_approx(d), false, 0.0f, -amax, amax, -7, 7);
        float2 nq[8];
        int_chunk<FMT, STATS>(y, iq, -7, 7, o.w, nq);
        // x-hat = (q s_b) S: the first product is exact
#pragma unroll
        for (int i = 0; i < 8; ++i) val[i] = mul2(nq[i], splat(-sbv));
    } else {
        const FpQ fq = fp_unit(d, amax);
        fp_chunk<FMT, STATS>(y, fq, o.w, val);
#pragma unroll
        for (int i = 0; i < 8; ++i) val[i] = mul2(val[i], splat(fq.zero ? 0.0f : sbv));
    }
    if constexpr (STATS) {
        if (scaled) val_sums<true>(y, val, S, p, o.e2, o.x2);
        else val_sums<false>(y, val, S, p, o.e2, o.x2);
    }
    return o;
}

// A lane's four NV blocks. Fast path per block: the exact quotient q = RN(x / d),
// d = s_b S, by the reciprocal correction with rn = RN(1/d) (s_b, d and rn from the CTA's
// table over the 127 block-scale codes); FP codes by cvt, INT4 codes rounded half to
// even (no clamp: the table admits only block scales under which no code passes +-7).
// The error of an element is taken as (q - code value) d, the quotient's residual in
// units of d: the sums gather the residuals' squares and scale by d^2 once per block.
// The span's plain sums and crest factors are gathered in fp32 and folded into the
// lane's doubles once per span.
template <int FMT, bool HAD, bool STATS>
__device__ __forceinline__ void span_nv(const Row& row, uint32_t span, const FlatArgs& a, const TensorCtx& tc,
                                        const float4* nvtab, Acc& acc, uint32_t (&span4)[8], uint32_t& scodes)
{
    using F = Fmt<FMT>;
    float se2 = 0.0f;
    float2 sx2 = splat(0.0f);
    float ksum = 0.0f, kmax = 0.0f;
    uint32_t kn = 0u;
    const float S = tc.S;
    const float2 M = splat(MAGIC), M1 = splat(-1.0f);
#pragma unroll 1
    for (int k = 0; k < SPAN; ++k) {
        uint32_t w[8], q[2];
        float2 y[8];
        row_chunk(row, k, w);
        chunk_in<HAD>(w, y);
        const float amax = chunk_amax(y, 0.0f);
        const uint32_t sbc = nv_scale_code<FMT>(amax, S, tc.cS);
        const float4 tb = nvtab[sbc];                  // s_b, d = s_b S, RN(1/d), clamp-free
        const float sbv = tb.x, d = tb.y, rn = tb.z;
        scodes |= sbc << (8 * k);
        // d = 0 codes every element as +0: INT4 gets that from the fast path, FP (where -0
        // would keep its sign) from the general path
        const bool mk = (F::is_int && !(d > 0.0f)) ||
                        (d >= 0x1p-60f && d <= 0x1p100f && __fmul_rn(amax, rn) < 0x1p20f);
        const bool fast = mk && (!F::is_int || tb.w != 0.0f);
        const bool scaled = STATS && !plain_sums_ok(amax);
        if (!__any_sync(0xFFFFFFFFu, !fast || scaled)) {
            const float2 RN = splat(rn), ND = splat(-d);
            float2 r[8];                                   // q - code value
            if constexpr (F::is_int) {
                float2 t[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 q0 = mul2(y[i], RN);
                    const float2 q1 = fma2(fma2(q0, ND, y[i]), RN, q0);      // RN(x / d)
                    const float2 t0 = add2(q1, M);                            // MAGIC + rne(q)
                    if constexpr (STATS) r[i] = add2(q1, fma2(t0, M1, M));    // q1 - rne(q), exact
                    t[i] = add2(t0, splat(8.0f));                             // + bias
                }
                pack_int<FMT>(t, q);
            } else {
                uint32_t pr[8];
                const float2 D = splat(d), NRN = splat(-rn);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    // RN(x / d), the residual taken negated so that -0 keeps its sign
                    const float2 q0 = mul2(y[i], RN);
                    r[i] = fma2(fma2(q0, D, neg2(y[i])), NRN, q0);
                    pr[i] = cvt_pair<FMT>(r[i].y, r[i].x);
                }
                pack_pairs<FMT>(pr, q);
                if constexpr (STATS) {
                    float2 val[8];
                    decode_pairs<FMT>(pr, val);
#pragma unroll
                    for (int i = 0; i < 8; ++i) r[i] = sub2(r[i], val[i]);
                }
            }
            if constexpr (STATS) {
                float2 ea = splat(0.0f), eb = splat(0.0f), xa = splat(0.0f), xb = splat(0.0f);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    ea = fma2(r[i], r[i], ea);
                    eb = fma2(r[i + 1], r[i + 1], eb);
                    xa = fma2(y[i], y[i], xa);
                    xb = fma2(y[i + 1], y[i + 1], xb);
                }
                const float2 ce2 = add2(ea, eb), cx2 = add2(xa, xb);
                se2 = __fmaf_rn(__fadd_rn(ce2.x, ce2.y), __fmul_rn(d, d), se2);
                sx2 = add2(sx2, cx2);
                const float ss = __fadd_rn(cx2.x, cx2.y);
                if (ss > 0.0f) {
                    const float kk = __fmul_rn(amax, rsqrtf(__fmul_rn(ss, a.inv_unit)));
                    ksum = __fadd_rn(ksum, kk);
                    kmax = fmaxf(kmax, kk);
                    ++kn;
                }
            }
        } else {
            const Pow2 pw = pow2_for(amax);
            const float p = scaled ? pw.p : 1.0f;
            const NvOut o = nv_general<FMT, STATS>(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7], amax, sbv, S,
                                                   scaled, p);
            q[0] = o.w[0];
            q[1] = o.w[1];
            if constexpr (STATS) {
                if (SPAN * span + k < a.n_chunks) {
                    unit_done(acc, o.e2, o.x2, scaled, pw);
                    kappa_add(acc, __fmul_rn(amax, p), __fadd_rn(o.x2.x, o.x2.y), a.inv_unit);
                }
            }
        }
        put_codes<FMT>(span4, a.codes, SPAN * span + k, true, k, q);
    }
    if constexpr (STATS) {
        // chunks past the tensor's end are zeros: they add nothing
        acc.err2 += (double)se2;
        acc.x2 += (double)__fadd_rn(sx2.x, sx2.y);
        acc.ksum += (double)ksum;
        acc.kmax = fmaxf(acc.kmax, kmax);
        acc.nunits += kn;
    }
}

// ---- two-chunk units: MX block 32, groups of 32 -------------------------------

template <int FMT, int GK, bool HAD, bool STATS, bool EXACT>
__device__ __forceinline__ void span_n2(const Row& row, uint32_t span, const FlatArgs& a, Acc& acc,
                                        uint32_t (&span4)[8], uint32_t& scodes)
{
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    constexpr bool GASYM = F::asym && GK == K_GROUP;
    const bool f16 = a.scale_fp16 != 0;
#pragma unroll 1
    for (int b = 0; b < SPAN; b += 2) {
        uint32_t w0[8], w1[8], q0[NW], q1[NW];
        float2 y0[8], y1[8];
        row_chunk(row, b, w0);
        row_chunk(row, b + 1, w1);
        chunk_in<HAD>(w0, y0);
        chunk_in<HAD>(w1, y1);
        float amax, mn = 0.0f, mx = 0.0f;
        if constexpr (GASYM) { chunk_minmax(y0, mn, mx); chunk_minmax(y1, mn, mx); amax = fmaxf(-mn, mx); }
        else amax = chunk_amax(y1, chunk_amax(y0, 0.0f));
        const bool scaled = STATS && __any_sync(0xFFFFFFFFu, !plain_sums_ok(amax));
        const Pow2 pw = pow2_for(amax);
        const float p = scaled ? pw.p : 1.0f;
        float2 e2 = splat(0.0f), x2 = splat(0.0f);
        const uint32_t c = SPAN * span + b;
        const bool valid = c < a.n_chunks;
        bool gen = false;                 // codes already placed by the general path

        if constexpr (GK == K_MX) {
            const int e = ue8m0_exponent<FMT>(amax);
            const float p2 = exp2i(-e), pe = exp2i(e);
            mx_chunk<FMT, GK, STATS>(y0, p2, pe, scaled, p, q0, e2, x2);
            mx_chunk<FMT, GK, STATS>(y1, p2, pe, scaled, p, q1, e2, x2);
            scodes |= (uint32_t)(e + 127) << (4 * b);
        } else {
            const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
            const PlainUnit<FMT> u = plain_unit<FMT>(ps);
            plain_unit_chunks<FMT, HAD, STATS, EXACT>(row, u, scaled, p, a.codes, (size_t)SPAN * span, b, 2,
                                                      span_valid(span, a.n_chunks), e2, x2, span4);
            gen = true;
            if (valid) store_plain_scale<FMT>(a.scales, a.zps, c / 2, ps, f16);
        }
        if (!gen) {
            put_codes<FMT>(span4, a.codes, c, valid, b, q0);
            put_codes<FMT>(span4, a.codes, c + 1, c + 1 < a.n_chunks, b + 1, q1);
        }
        if constexpr (STATS) {
            if (valid) {
                unit_done(acc, e2, x2, scaled, pw);
                kappa_add(acc, __fmul_rn(amax, p), __fadd_rn(x2.x, x2.y), a.inv_unit);
            }
        }
    }
}

// ---- groups of 64 .. 512: the span, or T = G / 64 adjacent lanes ---------------

template <int FMT, bool HAD, bool STATS, bool EXACT>
__device__ __forceinline__ void span_n4(const Row& row, uint32_t span, const FlatArgs& a, Acc& acc, int lane, int T,
                                        uint32_t (&span4)[8])
{
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    const bool f16 = a.scale_fp16 != 0;
    float amax = 0.0f, mn = 0.0f, mx = 0.0f;
    // range: from the raw bf16 words, or (rotated) from a first rotation
    if constexpr (HAD) {
#pragma unroll
        for (int k = 0; k < SPAN; ++k) {
            uint32_t w[8];
            float2 y[8];
            row_chunk(row, k, w);
            chunk_in<true>(w, y);
            if constexpr (F::asym) chunk_minmax(y, mn, mx);
            else amax = chunk_amax(y, amax);
        }
    } else if constexpr (F::asym) {
        uint32_t lo = 0u, hi = 0u;          // bf16 pair (+0, +0)
#pragma unroll
        for (int k = 0; k < SPAN; ++k) {
            uint32_t w[8];
            row_chunk(row, k, w);
            words_minmax(w, lo, hi);
        }
        mn = pair_min(lo);
        mx = pair_max(hi);
    } else {
        uint32_t m = 0u;
#pragma unroll
        for (int k = 0; k < SPAN; ++k) {
            uint32_t w[8];
            row_chunk(row, k, w);
            m = words_absmax(w, m);
        }
        amax = pair_absmax(m);
    }
    for (int o = 1; o < T; o <<= 1) {
        if constexpr (F::asym) {
            mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        } else {
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        }
    }
    if constexpr (F::asym) amax = fmaxf(-mn, mx);

    const bool scaled = STATS && __any_sync(0xFFFFFFFFu, !plain_sums_ok(amax));
    const Pow2 pw = scaled ? pow2_for(amax) : Pow2{1.0f, 1.0};
    const float p = pw.p;
    const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
    const PlainUnit<FMT> u = plain_unit<FMT>(ps);
    float2 e2 = splat(0.0f), x2 = splat(0.0f);
    plain_unit_chunks<FMT, HAD, STATS, EXACT>(row, u, scaled, p, a.codes, (size_t)SPAN * span, 0, SPAN,
                                              span_valid(span, a.n_chunks), e2, x2, span4);
    const bool valid = SPAN * span < a.n_chunks;
    const bool leader = (lane & (T - 1)) == 0;
    if (leader && valid) store_plain_scale<FMT>(a.scales, a.zps, span / (uint32_t)T, ps, f16);
    if constexpr (STATS) {
        if (valid) unit_done(acc, e2, x2, scaled, pw);
        float ss = __fadd_rn(x2.x, x2.y);
        for (int o = 1; o < T; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
        if (valid && leader) kappa_add(acc, __fmul_rn(amax, p), ss, a.inv_unit);
    }
}

// Store a span's gathered 4-bit codes: one 32-byte store when the span is whole, chunk
// by chunk at the ragged end.
template <int FMT>
__device__ __forceinline__ void store_span4(uint8_t* codes, uint32_t span, uint32_t n_chunks, const uint32_t (&v)[8])
{
    if constexpr (Fmt<FMT>::four) {
        const uint32_t c0 = SPAN * span;
        if (c0 < n_chunks && n_chunks - c0 >= (uint32_t)SPAN) {
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

// The part of the work a warp owns. The tensor (or each tensor of a batch) is a run of
// spans of 64 elements; spans are grouped into octets of 8 (1 KiB, one tensor-map box),
// and octets into partition units of `unit_oct` octets (a group of more than 8 lanes
// needs its whole tile). A batch gives each tensor its own group of warps (every warp
// sees one tensor); a tensor's units are split evenly over its warps, so the warps of a
// launch finish within one unit of each other.
struct WarpRange {
    uint32_t tensor;        // index in the batch
    uint64_t base;          // global span index of the tensor's first span
    uint32_t oct0, oct1;    // the warp's octets of that tensor, [oct0, oct1)
};

__device__ __forceinline__ WarpRange warp_range(uint32_t w, uint32_t nw, const FlatArgs& a)
{
    WarpRange r;
    const uint64_t B = a.batch, W = nw;
    // tensor b's warps are [floor(W b / B), floor(W (b + 1) / B)) (B <= W)
    const uint32_t b = (uint32_t)(((uint64_t)(w + 1) * B - 1) / W);
    const uint32_t g0 = (uint32_t)(W * b / B), g1 = (uint32_t)(W * (b + 1) / B);
    const uint64_t octs = ((uint64_t)a.spans_per_tensor + 7) / 8;
    const uint64_t units = octs / a.unit_oct, i = w - g0, n = g1 - g0;
    r.tensor = b;
    r.base = (uint64_t)b * a.spans_per_tensor;
    r.oct0 = (uint32_t)(units * i / n * a.unit_oct);
    r.oct1 = (uint32_t)(units * (i + 1) / n * a.unit_oct);
    return r;
}

// Batched stats: every warp's sums go to its own slot; the last CTA sums, for each tensor,
// the slots of that tensor's warps in warp order (a warp of the last CTA per tensor, its
// lanes over the slots, then a fixed xor tree), so the result is bit-reproducible.
__device__ __forceinline__ void finish_stats_batch(Acc mine, uint8_t* ws, bq_stats* out, uint32_t w, uint32_t nw,
                                                   uint32_t batch)
{
    __shared__ bool is_last;
    AccD m;
    m.err2 = mine.err2; m.x2 = mine.x2; m.ksum = mine.ksum; m.kmax = (double)mine.kmax; m.nunits = (double)mine.nunits;
    const AccD t = warp_reduce_acc(m);
    StatSlot* slots = ws_stats(ws);
    WsHeader* h = ws_header(ws);
    if ((threadIdx.x & 31) == 0) {
        slots[w] = StatSlot{t.err2, t.x2, t.ksum, t.kmax, t.nunits, 0.0};
        __threadfence();
    }
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomic_add_acq_rel(&h->counter_stats, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!is_last) return;
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5, nwib = blockDim.x >> 5;
    for (uint32_t b = wib; b < batch; b += nwib) {
        const uint32_t g0 = (uint32_t)((uint64_t)nw * b / batch), g1 = (uint32_t)((uint64_t)nw * (b + 1) / batch);
        AccD a;
        for (uint32_t i = g0 + lane; i < g1; i += 32) {
            const double* p = reinterpret_cast<const double*>(&slots[i]);
            a.err2 += __ldcg(p + 0); a.x2 += __ldcg(p + 1); a.ksum += __ldcg(p + 2);
            a.kmax = fmax(a.kmax, __ldcg(p + 3)); a.nunits += __ldcg(p + 4);
        }
        a = warp_reduce_acc(a);
        if (lane == 0) {
            bq_stats r;
            r.err2 = a.err2; r.x2 = a.x2; r.kappa_sum = a.ksum; r.kappa_max = a.kmax; r.n_units = a.nunits;
            out[b] = r;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) h->counter_stats = 0u;   // ready for the next call on this workspace
}

template <int FMT, int GK, bool HAD, bool STATS, bool EXACT>
__global__ void __launch_bounds__(FLAT_WARPS * 32, BQ_FLAT_MINB) k_quant_flat(const __grid_constant__ CUtensorMap xmap,
                                                                  const __grid_constant__ CUtensorMap xmap32,
                                                                  const FlatArgs a)
{
    pdl_wait();
    using F = Fmt<FMT>;
    extern __shared__ uint8_t flat_smem[];
    __shared__ __align__(8) uint64_t bars[FLAT_WARPS][NST];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    // warps numbered CTA by CTA: a CTA's warps own neighbouring ranges
    const uint32_t warp = blockIdx.x * FLAT_WARPS + wib;
    const uint32_t nwarps = gridDim.x * FLAT_WARPS;
    const uint32_t buf0 = ((smem_addr(flat_smem) + 1023u) & ~1023u) + (uint32_t)wib * NST * TILE_BYTES;
    const uint32_t bar0 = smem_addr(&bars[wib][0]);
    const uint32_t rows_mapped = a.n_chunks / SPAN;     // whole spans the tensor map covers
    const WarpRange wr = warp_range(warp, nwarps, a);
    // the warp's spans, global indices [first_span, end_span) (32-bit: a launch has fewer
    // than 2^30 spans); tile k: spans first_span + 32 k .., octets oct0 + 4 k ..
    const uint32_t first_span = (uint32_t)wr.base + 8u * wr.oct0;
    const uint32_t end_span = (uint32_t)wr.base + min(8u * wr.oct1, a.spans_per_tensor);
    const uint32_t n_oct = wr.oct1 - wr.oct0;
    const uint32_t n_tiles = (n_oct + 3) / 4;

    if (lane == 0) {
        for (int s = 0; s < NST; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();

    uint32_t inflight = 0, parity = 0;                  // per stage bits (warp-uniform)
    // tile k goes in as one 32-span box when it is whole, else as one 8-span box per
    // octet that the map covers (boxes past the map's last span are filled with zeros by
    // the lanes that own them)
    auto issue = [&](uint32_t k, int s) {
        if (k >= n_tiles) return;
        const uint32_t n = min(4u, n_oct - 4 * k), first = first_span + 32 * k;
        if (first >= rows_mapped) return;
        // (the test hook: warp skip_tile issues no copy for its first tile, so its wait runs out)
        if (lane == 0 && !(k == 0 && warp == a.skip_tile)) {
            const uint32_t dst = buf0 + s * TILE_BYTES, bar = bar0 + 8 * s;
            if (n == 4) {
                mbar_arrive_expect_tx(bar, TILE_BYTES);
                tma_load_2d(dst, &xmap32, bar, 0, (int)first);
            } else {
                const uint32_t boxes = min(n, (rows_mapped - first + 7) / 8);
                mbar_arrive_expect_tx(bar, boxes * 1024u);
                for (uint32_t j = 0; j < boxes; ++j) tma_load_2d(dst + j * 1024u, &xmap, bar, 0, (int)(first + 8 * j));
            }
        }
        inflight |= 1u << s;
    };
#pragma unroll
    for (int s = 0; s < NST; ++s) issue((uint32_t)s, s);

    TensorCtx tc{};
    PlainUnit<FMT> tu{};
    Pow2 tp{1.0f, 1.0};
    bool tscaled = false;
    if constexpr (GK == K_TENSOR || GK == K_NV) {
        // {amax, min, max} of the (rotated) tensor: the range pass's result in the
        // workspace header, or the caller's
        const float r_amax = a.range[0], r_min = a.range[1], r_max = a.range[2];
        tc.amax = r_amax;
        if constexpr (GK == K_TENSOR) {
            tc.ps = plain_scale<FMT>(r_amax, r_min, r_max, a.scale_fp16 != 0);
            tu = plain_unit<FMT>(tc.ps);
            tp = pow2_for(tc.amax);
            tscaled = STATS && !plain_sums_ok(tc.amax);
            if (blockIdx.x == 0 && threadIdx.x == 0) store_plain_scale<FMT>(a.scales, a.zps, 0, tc.ps, a.scale_fp16 != 0);
        } else {
            tc.S = div_rn_call(r_amax, F::qscale * 448.0f);
            tc.cS = rcp_approx(__fmul_rn(F::qscale, tc.S));
            if (blockIdx.x == 0 && threadIdx.x == 0) a.tensor_scale[0] = tc.S;
        }
    }
    // NV: per block-scale code c (0..126; satfinite never gives the NaN code 127): s_b,
    // d = s_b S and RN(1/d), computed once per CTA
    __shared__ float4 nvtab[GK == K_NV ? 128 : 1];
    if constexpr (GK == K_NV) {
        for (int c = threadIdx.x; c < 128; c += blockDim.x) {
            const float sb = e4m3_value((uint32_t)c);
            const float d = __fmul_rn(sb, tc.S);
            // w = 1: no integer code can pass +-Qmax (a normal E4M3 s_b is at most 2^-4
            // below (amax / Qmax) / S, so |x / d| < Qmax (1 + 1/15) < Qmax + 0.5; d = 0 codes 0)
            const bool nc = !(d > 0.0f) || (c & 0x78) != 0;
            nvtab[c] = make_float4(sb, d, d > 0.0f ? __frcp_rn(d) : 0.0f, nc ? 1.0f : 0.0f);
        }
        __syncthreads();
    }
    // per-group units: 16 elements (one chunk), 32 (two), 64 and up (the span, T lanes)
    const int T = (GK == K_GROUP && a.lanes_per_group > 0) ? a.lanes_per_group : 1;
    // span index of lanes with nothing to do: its chunks (from 0xFFFFFFF8 on) lie past every
    // tensor's end (at most 2^32 - 128 chunks), and no guard on them wraps around
    constexpr uint32_t NO_SPAN = 0xFFFFFFFFu / SPAN - 1u;

    Acc acc;
    bool ok = true;
    int s = 0;
    for (uint32_t k = 0; k < n_tiles; ++k) {
        const Row row{buf0 + s * TILE_BYTES + lane * ROW_BYTES, (uint32_t)(lane & 7)};
        const uint32_t n = min(4u, n_oct - 4 * k), tspan = first_span + 32 * k;
        const uint32_t gspan = tspan + (uint32_t)lane;            // the lane's span
        const bool mine = gspan < end_span;
        const uint32_t span = mine ? gspan : NO_SPAN;
        if (inflight >> s & 1u) {
            const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(bar0 + 8 * s, parity >> s & 1u));
            // a stage whose wait gave up stays in flight: the drain below waits for it
            if (!got) { ok = false; break; }
            parity ^= 1u << s;
            inflight &= ~(1u << s);
        }
        if ((uint32_t)lane >= 8 * n || (n < 4 && tspan + 8u * ((uint32_t)lane / 8) >= rows_mapped) ||
            tspan >= rows_mapped) {
            // the lane's row is outside this tile, or its box was not issued (past the
            // map's last span): zeros (fast paths sum every lane's values), or for the span
            // holding the ragged end, its chunks from global memory
            const uint32_t c0 = SPAN * gspan;
#pragma unroll 1
            for (int kk = 0; kk < SPAN; ++kk) {
                uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                if (mine && c0 + kk < a.n_chunks) ld_nc_v8(a.x + (size_t)(c0 + kk) * 8, w);
                row_put_chunk(row, kk, w);
            }
        } else if (mine && gspan == rows_mapped && rows_mapped * SPAN < a.n_chunks) {
            // the ragged end inside a mapped box (zero filled there): from global memory
            for (int kk = 0; kk < SPAN; ++kk) {
                uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                const uint32_t c = SPAN * span + kk;
                if (c < a.n_chunks) ld_nc_v8(a.x + (size_t)c * 8, w);
                row_put_chunk(row, kk, w);
            }
        }
        fence_proxy_async();
        __syncwarp();

        uint32_t span4[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        uint32_t scodes = 0u;
        if constexpr (GK == K_TENSOR) {
            span_tensor<FMT, HAD, STATS, EXACT>(row, span, a, tu, tp, tscaled, acc, span4);
        } else if constexpr (GK == K_NV) {
            span_nv<FMT, HAD, STATS>(row, span, a, tc, nvtab, acc, span4, scodes);
        } else if constexpr (GK == K_MX) {
            span_n2<FMT, GK, HAD, STATS, false>(row, span, a, acc, span4, scodes);
        } else {
            if (a.lanes_per_group == 0) span_n1<FMT, GK, HAD, STATS, EXACT>(row, span, a, tc, acc, span4, scodes);
            else if (a.lanes_per_group < 0) span_n2<FMT, GK, HAD, STATS, EXACT>(row, span, a, acc, span4, scodes);
            else span_n4<FMT, HAD, STATS, EXACT>(row, span, a, acc, lane, T, span4);
        }
        __syncwarp();                       // every lane is done with the buffer
        issue(k + NST, s);
        s = (s + 1 == NST) ? 0 : s + 1;

        store_span4<FMT>(a.codes, span, a.n_chunks, span4);
        const uint32_t c0 = SPAN * span;
        if constexpr (GK == K_NV) {
            // four E4M3 block scales, one per chunk (in the GEMM layout: four adjacent
            // bytes, the span's first block being a multiple of 4 in its row)
            uint8_t* sc = reinterpret_cast<uint8_t*>(a.scales);
            if (a.gemm_layout) {
                if (c0 < a.n_chunks) *reinterpret_cast<uint32_t*>(sc + gemm_unit_offset(c0, a.gemm_nb)) = scodes;
            } else if (c0 < a.n_chunks && a.n_chunks - c0 >= (uint32_t)SPAN) {
                *reinterpret_cast<uint32_t*>(sc + c0) = scodes;
            } else {
                for (int kk = 0; kk < SPAN; ++kk)
                    if (c0 + kk < a.n_chunks) sc[c0 + kk] = (uint8_t)(scodes >> (8 * kk));
            }
        } else if constexpr (GK == K_MX) {
            // two UE8M0 block scales (in the GEMM layout: two adjacent bytes)
            uint8_t* sc = reinterpret_cast<uint8_t*>(a.scales);
            if (a.gemm_layout) {
                if (c0 < a.n_chunks) *reinterpret_cast<uint16_t*>(sc + gemm_unit_offset(c0 / 2, a.gemm_nb)) = (uint16_t)scodes;
            } else if (c0 < a.n_chunks && a.n_chunks - c0 >= (uint32_t)SPAN) {
                *reinterpret_cast<uint16_t*>(sc + c0 / 2) = (uint16_t)scodes;
            } else if (c0 < a.n_chunks) {
                sc[c0 / 2] = (uint8_t)scodes;
            }
        }
    }
    if (!ok) {
        // a tile never arrived: record it, give the other loads in flight their chance
        // to land (bounded) and stop; the results of this call are incomplete
        if (lane == 0) atomicAdd(&g_flat_wait_timeouts, 1u);
        for (int kk = 0; kk < NST; ++kk)
            if (inflight >> kk & 1u) (void)mbar_wait(bar0 + 8 * kk, parity >> kk & 1u);
    }

    if constexpr (STATS) {
        if (a.batch > 1) {
            finish_stats_batch(acc, a.ws, a.stats, warp, nwarps, a.batch);
        } else {
            // per-tensor kappa comes from the totals: amax / sqrt(sum y^2 / n)
            finish_stats(acc, a.ws, a.stats, GK == K_TENSOR, tc.amax, a.n_elems, true);
        }
    }
}

// ---------------------------------------------------------------------------
// Per-row quantize, a warp per row (rows of cols % 64 == 0 elements).
//
// The row reaches shared memory as M = ceil(cols / 2048) tiles of a 3-D tensor map (x
// as [rows][cols / 64][64]; a box is 32 segments of 64 elements of one row, zero past
// the row's end), lane l taking segment l of each tile (four chunks, as in the flat
// kernel). A row of at most RN tiles is loaded once and read twice from the ring (range,
// then codes); a longer row passes through the ring twice (the second time from L2), so
// the ring needs no room for a whole row. One scale per row, computed by every lane
// from the warp's reduced range. The ring has RN = 4 stages for rows of 3-4 tiles (6144 to
// 8192 columns: resident, 4.5 % faster at 8192 than reloading them through two stages),
// else 2 (more CTAs per SM: 7.5 % faster on 4096-column rows than four stages).
// ---------------------------------------------------------------------------

// CTAs of 4 warps, 4 per SM (the same 16 warps per SM as the flat kernel): with 1-2
// rows per warp on a 4096-row tensor, warps whose last row ends early wait for fewer
// siblings at the CTA's final reduction (measured 4 % faster than 8-warp CTAs there).
constexpr int ROWS_WARPS = 4;
__host__ __device__ constexpr uint32_t rows_smem(int rn) { return ROWS_WARPS * (uint32_t)rn * TILE_BYTES + 1024u; }

template <int FMT, bool HAD, bool STATS, bool EXACT, int RN>
__global__ void __launch_bounds__(ROWS_WARPS * 32, 4) k_quant_rows(const __grid_constant__ CUtensorMap xmap,
                                                                 const RowsArgs a)
{
    pdl_wait();
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    extern __shared__ uint8_t flat_smem[];
    __shared__ __align__(8) uint64_t bars[ROWS_WARPS][RN];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    // warps numbered across the CTAs first: the last, partly filled round of tiles (rows)
    // spreads over every CTA, and so over every SM, instead of filling the first CTAs
    const uint32_t warp = wib * gridDim.x + blockIdx.x;
    const uint32_t nwarps = gridDim.x * ROWS_WARPS;
    const uint32_t buf0 = ((smem_addr(flat_smem) + 1023u) & ~1023u) + (uint32_t)wib * RN * TILE_BYTES;
    const uint32_t bar0 = smem_addr(&bars[wib][0]);
    // tiles per row; a row of at most RN tiles stays in the ring for both passes
    // (loaded once), a longer one is loaded again (from L2) for the codes
    const uint32_t M = a.tiles;
    const bool resident = M <= (uint32_t)RN;
    const uint32_t L = resident ? M : 2 * M;             // loads per row

    if (lane == 0) {
        for (int s = 0; s < RN; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();

    uint32_t inflight = 0, parity = 0;                   // per stage bits (warp-uniform)
    // load k of this warp: row warp + (k / L) nwarps, tile (k % L) % M
    auto issue = [&](uint32_t k, int s) {
        const uint32_t r = warp + (k / L) * nwarps;
        if (r < a.rows) {
            if (lane == 0) {
                mbar_arrive_expect_tx(bar0 + 8 * s, TILE_BYTES);
                tma_load_3d(buf0 + s * TILE_BYTES, &xmap, bar0 + 8 * s, 0, (int)(((k % L) % M) * 32), (int)r);
            }
            inflight |= 1u << s;
        }
    };
    auto wait_stage = [&](int s) -> bool {
        if (!(inflight >> s & 1u)) return true;
        const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(bar0 + 8 * s, parity >> s & 1u));
        // a stage whose wait gave up stays in flight: the drain at the end waits for it
        if (!got) return false;
        parity ^= 1u << s;
        inflight &= ~(1u << s);
        return true;
    };
#pragma unroll
    for (int s = 0; s < RN; ++s) issue((uint32_t)s, s);

    const bool f16 = a.scale_fp16 != 0;
    Acc acc;
    bool ok = true;
    uint32_t k = 0;
    int s = 0;
    for (uint32_t r = warp; r < a.rows && ok; r += nwarps) {
        const int s_row = s;                              // the row's first stage
        // pass 1: the lane's part of the row's range
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
        uint32_t plo = 0u, phi = 0u, pm = 0u;            // packed bf16 pairs
        for (uint32_t j = 0; j < M; ++j) {
            if (!wait_stage(s)) { ok = false; break; }
            const Row row{buf0 + s * TILE_BYTES + lane * ROW_BYTES, (uint32_t)(lane & 7)};
#pragma unroll
            for (int kk = 0; kk < SPAN; ++kk) {
                uint32_t w[8];
                row_chunk(row, kk, w);
                if constexpr (HAD) {
                    float2 y[8];
                    chunk_in<true>(w, y);
                    if constexpr (F::asym) chunk_minmax(y, mn, mx);
                    else amax = chunk_amax(y, amax);
                } else if constexpr (F::asym) {
                    words_minmax(w, plo, phi);
                } else {
                    pm = words_absmax(w, pm);
                }
            }
            __syncwarp();
            if (!resident) {
                issue(k + RN, s);
                ++k;
            }
            s = (s + 1 == RN) ? 0 : s + 1;
        }
        if (!ok) break;
        if (resident) s = s_row;                          // the codes read the same stages
        if constexpr (!HAD) {
            if constexpr (F::asym) { mn = pair_min(plo); mx = pair_max(phi); }
            else amax = pair_absmax(pm);
        }
        if constexpr (F::asym) { mn = warp_minf(mn); mx = warp_maxf(mx); amax = fmaxf(-mn, mx); }
        else amax = warp_maxf(amax);

        const bool scaled = STATS && !plain_sums_ok(amax);   // uniform over the warp
        const Pow2 pw = pow2_for(amax);
        const float p = scaled ? pw.p : 1.0f;
        const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
        const PlainUnit<FMT> u = plain_unit<FMT>(ps);
        float2 e2 = splat(0.0f), x2 = splat(0.0f);

        // pass 2: codes
        for (uint32_t j = 0; j < M; ++j) {
            if (!resident && !wait_stage(s)) { ok = false; break; }
            const Row row{buf0 + s * TILE_BYTES + lane * ROW_BYTES, (uint32_t)(lane & 7)};
            const uint32_t g = j * 32 + lane;                    // the lane's segment
            const bool seg_ok = g < a.nseg;
            const size_t c0 = (size_t)r * a.cpr + 4u * g;        // its first chunk
            uint32_t span4[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            plain_unit_chunks<FMT, HAD, STATS, EXACT>(row, u, scaled, p, a.codes, c0, 0, SPAN, seg_ok ? SPAN : 0,
                                                      e2, x2, span4);
            if constexpr (F::four) {
                if (seg_ok) st_v8(a.codes + c0 * 8, span4);
            }
            __syncwarp();
            issue(k + RN, s);
            ++k;
            s = (s + 1 == RN) ? 0 : s + 1;
        }
        if (!ok) break;
        if (lane == 0) store_plain_scale<FMT>(a.scales, a.zps, r, ps, f16);
        if constexpr (STATS) {
            add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
            float ss = __fadd_rn(x2.x, x2.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
            if (lane == 0) kappa_add(acc, __fmul_rn(amax, p), ss, a.inv_cols);
        }
    }
    if (!ok) {
        if (lane == 0) atomicAdd(&g_flat_wait_timeouts, 1u);
        for (int kk = 0; kk < RN; ++kk)
            if (inflight >> kk & 1u) (void)mbar_wait(bar0 + 8 * kk, parity >> kk & 1u);
    }
    if constexpr (STATS) finish_stats(acc, a.ws, a.stats, false, 0.0f, 0.0, true);
}

// ---------------------------------------------------------------------------
// 2-D tiles: one scale per 128 x 128 tile (the DeepSeek-V3 weight tiles, "Quantization
// survey" §4.4).
//
// A CTA of 8 warps owns a tile at a time (grid-stride over the tiles in row-major
// order). The tile reaches shared memory as two boxes of a 2-D tensor map over x (128
// rows x 64 columns each, 128-byte swizzle, zero past the last row), TILE_NST tiles
// ahead, completed on one mbarrier per stage. Thread t takes row t & 127 of box t >> 7
// (warps 0-3 the left half, 4-7 the right), a 64-element span as in the flat kernel.
// The warps' partial ranges meet in shared memory at one barrier per tile; passing it
// also means every thread is done with the previous tile, so its stage is refilled
// right there, and that tile's kappa is formed from the warps' sums of squares.
// ---------------------------------------------------------------------------

constexpr int TILE_NST = 2;                                 // tile buffers per CTA
constexpr uint32_t TBOX_BYTES = TILE * ROW_BYTES;           // 128 rows x 64 bf16 = 16 KiB
constexpr uint32_t TSTAGE_BYTES = 2 * TBOX_BYTES;           // a whole tile, 32 KiB
constexpr uint32_t TILE2D_SMEM = TILE_NST * TSTAGE_BYTES + 1024;

template <int FMT, bool HAD, bool STATS, bool EXACT>
__global__ void __launch_bounds__(256, 2) k_quant_tile2d(const __grid_constant__ CUtensorMap xmap,
                                                         const Tile2dArgs a)
{
    pdl_wait();
    using F = Fmt<FMT>;
    extern __shared__ uint8_t tile_smem[];
    __shared__ __align__(8) uint64_t bars[TILE_NST];
    __shared__ float4 red[2][8];          // per warp: amax, min, max (by tile parity)
    __shared__ float red_ss[2][8];        // per warp: sum of squares of the scaled values
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const uint32_t trow = threadIdx.x & (TILE - 1), half = threadIdx.x / TILE;
    const uint32_t buf0 = (smem_addr(tile_smem) + 1023u) & ~1023u;
    const uint32_t bar0 = smem_addr(&bars[0]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < TILE_NST; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncthreads();

    // thread 0: stages with a load in flight, and each stage's next phase
    uint32_t inflight = 0, phase = 0;
    auto issue = [&](uint32_t j, uint32_t s) {           // the CTA's tile j into stage s
        const uint32_t t = blockIdx.x + j * gridDim.x;
        if (t < a.ntiles) {
            const uint32_t tr = t / a.tpr, tc = t - tr * a.tpr;
            const uint32_t dst = buf0 + s * TSTAGE_BYTES, bar = bar0 + 8 * s;
            mbar_arrive_expect_tx(bar, TSTAGE_BYTES);
            tma_load_2d(dst, &xmap, bar, (int)(tc * TILE), (int)(tr * TILE));
            tma_load_2d(dst + TBOX_BYTES, &xmap, bar, (int)(tc * TILE + 64), (int)(tr * TILE));
            inflight |= 1u << s;
        }
    };
    if (threadIdx.x == 0)
        for (uint32_t s = 0; s < (uint32_t)TILE_NST; ++s) issue(s, s);

    const bool f16 = a.scale_fp16 != 0;
    Acc acc;
    float kap_amax = 0.0f, kap_inv_n = 0.0f;              // thread 0: the last tile's kappa inputs
    bool ok = true;
    uint32_t j = 0;
    for (uint32_t t = blockIdx.x; t < a.ntiles; t += gridDim.x, ++j) {
        const uint32_t s = j % TILE_NST;
        const bool got = mbar_wait(bar0 + 8 * s, (j / TILE_NST) & 1u);
        if (threadIdx.x == 0 && got) { inflight &= ~(1u << s); phase ^= 1u << s; }
        const Row row{buf0 + s * TSTAGE_BYTES + half * TBOX_BYTES + trow * ROW_BYTES, trow & 7u};

        // pass 1: the thread's part of the tile's range, then the warp's
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
        if constexpr (HAD) {
#pragma unroll
            for (int k = 0; k < SPAN; ++k) {
                uint32_t w[8];
                float2 y[8];
                row_chunk(row, k, w);
                chunk_in<true>(w, y);
                if constexpr (F::asym) chunk_minmax(y, mn, mx);
                else amax = chunk_amax(y, amax);
            }
        } else {
            uint32_t plo = 0u, phi = 0u, pm = 0u;         // packed bf16 pairs
#pragma unroll
            for (int k = 0; k < SPAN; ++k) {
                uint32_t w[8];
                row_chunk(row, k, w);
                if constexpr (F::asym) words_minmax(w, plo, phi);
                else pm = words_absmax(w, pm);
            }
            if constexpr (F::asym) { mn = pair_min(plo); mx = pair_max(phi); }
            else amax = pair_absmax(pm);
        }
        if constexpr (F::asym) { mn = warp_minf(mn); mx = warp_maxf(mx); }
        else amax = warp_maxf(amax);
        if (lane == 0) red[j & 1][wib] = make_float4(amax, mn, mx, 0.0f);
        if (__syncthreads_or(!got)) { ok = false; break; }

        if (threadIdx.x == 0 && j > 0) {
            const uint32_t jp = j - 1;
            if constexpr (STATS) {
                float ss = red_ss[jp & 1][0];
#pragma unroll
                for (int w = 1; w < 8; ++w) ss = __fadd_rn(ss, red_ss[jp & 1][w]);
                kappa_add(acc, kap_amax, ss, kap_inv_n);
            }
            issue(jp + TILE_NST, jp % TILE_NST);
        }

        // the tile's range and scale (the same in every thread)
        {
            const float4 v0 = red[j & 1][0];
            amax = v0.x; mn = v0.y; mx = v0.z;
#pragma unroll
            for (int w = 1; w < 8; ++w) {
                const float4 v = red[j & 1][w];
                amax = fmaxf(amax, v.x); mn = fminf(mn, v.y); mx = fmaxf(mx, v.z);
            }
            if constexpr (F::asym) amax = fmaxf(-mn, mx);
        }
        const bool scaled = STATS && !plain_sums_ok(amax);
        const Pow2 pw = pow2_for(amax);
        const float p = scaled ? pw.p : 1.0f;
        const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
        const PlainUnit<FMT> u = plain_unit<FMT>(ps);

        // pass 2: codes of the thread's span
        const uint32_t tr = t / a.tpr, tc = t - tr * a.tpr;
        const uint32_t r = tr * TILE + trow;
        const bool row_ok = r < a.rows;
        const size_t c0 = ((size_t)r * a.cols + tc * TILE + half * 64u) / 16u;   // its first chunk
        float2 e2 = splat(0.0f), x2 = splat(0.0f);
        uint32_t span4[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        plain_unit_chunks<FMT, HAD, STATS, EXACT>(row, u, scaled, p, a.codes, c0, 0, SPAN, row_ok ? SPAN : 0,
                                                  e2, x2, span4);
        if constexpr (F::four) {
            if (row_ok) st_v8(a.codes + c0 * 8, span4);
        }
        if (threadIdx.x == 0) store_plain_scale<FMT>(a.scales, a.zps, t, ps, f16);
        if constexpr (STATS) {
            add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
            float ss = __fadd_rn(x2.x, x2.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
            if (lane == 0) red_ss[j & 1][wib] = ss;
            if (threadIdx.x == 0) {
                const uint32_t nr = a.rows - tr * TILE < TILE ? a.rows - tr * TILE : TILE;
                kap_amax = __fmul_rn(amax, p);
                kap_inv_n = 1.0f / (float)(nr * TILE);
            }
        }
    }
    if (ok) {
        __syncthreads();
        if constexpr (STATS) {
            if (threadIdx.x == 0 && j > 0) {
                const uint32_t jp = j - 1;
                float ss = red_ss[jp & 1][0];
#pragma unroll
                for (int w = 1; w < 8; ++w) ss = __fadd_rn(ss, red_ss[jp & 1][w]);
                kappa_add(acc, kap_amax, ss, kap_inv_n);
            }
        }
    } else if (threadIdx.x == 0) {
        atomicAdd(&g_flat_wait_timeouts, 1u);
        for (int k = 0; k < TILE_NST; ++k)
            if (inflight >> k & 1u) (void)mbar_wait(bar0 + 8 * k, phase >> k & 1u);
    }
    if constexpr (STATS) finish_stats(acc, a.ws, a.stats, false, 0.0f, 0.0, true);
}

// ---------------------------------------------------------------------------
// Row transforms, then quantize (per-row, per-group, MX): SmoothQuant's per-column
// factor ("Quantization survey" §3.2, §5.2) and QuaRot's randomized full-row Hadamard
// rotation (same page §5.3).
//
// A CTA of B = min(256, cols / 16) threads owns a row at a time. Thread t loads chunks
// t, t + B, ... of the row, multiplies by the factors, negates the signed columns and
// runs the first four Walsh-Hadamard stages in registers; the row then sits in shared
// memory as fp32 for the remaining stages (wht_smem_stages). The quantize phase reads
// each chunk back times the normalisation and codes it (the fast chunk path when the
// warp's units admit it, else the general one): a scaling unit of L chunks is L
// adjacent threads, reduced with xor shuffles; a per-row unit is reduced over the
// CTA. The fused QSNR sums are taken on the rotated values (an orthogonal rotation
// keeps both sums).
// ---------------------------------------------------------------------------

template <int FMT, bool MX>
__global__ void __launch_bounds__(RT_THREADS, Fmt<FMT>::asym ? 4 : 5) k_quant_rt(const RtArgs a)
{
    pdl_wait();
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    extern __shared__ float4 rt_smem[];
    float* v = reinterpret_cast<float*>(rt_smem);
    __shared__ float4 red[8];
    __shared__ float red_ss[8];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const bool rot = a.sign_bits != nullptr, f16 = a.scale_fp16 != 0;
    const float norm = rot ? a.norm : 1.0f;
    const uint32_t L = a.lanes;
    uint32_t* smask = reinterpret_cast<uint32_t*>(v + rot_row_floats(a.cols));
    if (rot) {
        build_sign_masks(smask, a.sign_bits, a.cols);
        __syncthreads();
    }
    Acc acc;

    for (uint32_t r = blockIdx.x; r < a.rows; r += gridDim.x) {
        // load, factor, signs, stages h = 1 .. 8
        for (uint32_t c = threadIdx.x; c < a.cpr; c += blockDim.x) {
            uint32_t w[8];
            float2 y[8];
            ld_nc_v8(a.x + ((size_t)r * a.cpr + c) * 8, w);
            // the signs flip bf16 sign bits before the factor: the same values as flipping
            // the products' signs (a product's sign is its factors' signs combined)
            if (rot) flip_words(smask, c, w);
            widen16x2(w, y);
            if (a.col_scale) {
                const float4* m = reinterpret_cast<const float4*>(a.col_scale) + 4 * c;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 f = __ldg(m + i);
                    y[2 * i] = mul2(y[2 * i], make_float2(f.x, f.y));
                    y[2 * i + 1] = mul2(y[2 * i + 1], make_float2(f.z, f.w));
                }
            }
            if (rot) wht16x2(y);
            store_chunk_f32(v, c, y);
        }
        if (rot) wht_smem_stages(v, a.cols);
        else __syncthreads();

        if (L == 0) {
            // one unit: the whole row, reduced over the CTA
            float amax = 0.0f, mn = 0.0f, mx = 0.0f;
            for (uint32_t c = threadIdx.x; c < a.cpr; c += blockDim.x) {
                float2 y[8];
                load_chunk_f32(v, c, norm, y);
                if constexpr (F::asym) chunk_minmax(y, mn, mx);
                else amax = chunk_amax(y, amax);
            }
            if constexpr (F::asym) { mn = warp_minf(mn); mx = warp_maxf(mx); }
            else amax = warp_maxf(amax);
            if (lane == 0) red[wib] = make_float4(amax, mn, mx, 0.0f);
            __syncthreads();
            {
                const float4 v0 = red[0];
                amax = v0.x; mn = v0.y; mx = v0.z;
                for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
                    const float4 q = red[w];
                    amax = fmaxf(amax, q.x); mn = fminf(mn, q.y); mx = fmaxf(mx, q.z);
                }
                if constexpr (F::asym) amax = fmaxf(-mn, mx);
            }
            const bool scaled = !plain_sums_ok(amax);
            const Pow2 pw = pow2_for(amax);
            const float p = scaled ? pw.p : 1.0f;
            const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
            const PlainUnit<FMT> u = plain_unit<FMT>(ps);
            float2 e2 = splat(0.0f), x2 = splat(0.0f);
            const bool general = unit_general_fast<FMT, false>(u, scaled);
            for (uint32_t c = threadIdx.x; c < a.cpr; c += blockDim.x) {
                float2 y[8];
                uint32_t q[NW];
                load_chunk_f32(v, c, norm, y);
                rt_chunk<FMT>(y, u, general, scaled, p, q, e2, x2);
                store_codes<FMT>(a.codes, r * a.cpr + c, q);
            }
            if (threadIdx.x == 0) store_plain_scale<FMT>(a.scales, a.zps, r, ps, f16);
            add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
            float ss = __fadd_rn(x2.x, x2.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
            if (lane == 0) red_ss[wib] = ss;
            __syncthreads();
            if (threadIdx.x == 0) {
                float t = red_ss[0];
                for (int w = 1; w < (int)(blockDim.x >> 5); ++w) t = __fadd_rn(t, red_ss[w]);
                kappa_add(acc, __fmul_rn(amax, p), t, a.inv_unit);
            }
        } else {
            // units of L chunks = L adjacent threads (L a power of two dividing 32; cpr is a
            // multiple of 32): unit index and first chunk by shifts
            const uint32_t lgL = (uint32_t)(__ffs((int)L) - 1);
            for (uint32_t c = threadIdx.x; c < a.cpr; c += blockDim.x) {
                float2 y[8];
                uint32_t q[NW];
                load_chunk_f32(v, c, norm, y);
                float amax = 0.0f, mn = 0.0f, mx = 0.0f;
                if constexpr (F::asym && !MX) chunk_minmax(y, mn, mx);
                else amax = chunk_amax(y, 0.0f);
                for (uint32_t o = 1; o < L; o <<= 1) {
                    if constexpr (F::asym && !MX) {
                        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
                        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                    } else {
                        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                    }
                }
                if constexpr (F::asym && !MX) amax = fmaxf(-mn, mx);
                const bool scaled = !plain_sums_ok(amax);
                const Pow2 pw = pow2_for(amax);
                const float p = scaled ? pw.p : 1.0f;
                float2 e2 = splat(0.0f), x2 = splat(0.0f);
                const uint32_t cg = r * a.cpr + c;            // chunk index in the tensor
                const bool first = (c & (L - 1u)) == 0;
                if constexpr (MX) {
                    const int e = ue8m0_exponent<FMT>(amax);
                    mx_chunk<FMT, K_MX, true>(y, exp2i(-e), exp2i(e), scaled, p, q, e2, x2);
                    if (first) {
                        const uint32_t u = cg >> lgL;
                        reinterpret_cast<uint8_t*>(a.scales)[a.gemm_layout ? gemm_unit_offset(u, a.gemm_nb) : u] =
                            (uint8_t)(e + 127);
                    }
                } else {
                    const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
                    const PlainUnit<FMT> u = plain_unit<FMT>(ps);
                    rt_chunk<FMT>(y, u, unit_general_fast<FMT, false>(u, scaled), scaled, p, q, e2, x2);
                    if (first) store_plain_scale<FMT>(a.scales, a.zps, cg >> lgL, ps, f16);
                }
                store_codes<FMT>(a.codes, cg, q);
                add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
                float ss = __fadd_rn(x2.x, x2.y);
                for (uint32_t o = 1; o < L; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
                if (first) kappa_add(acc, __fmul_rn(amax, p), ss, a.inv_unit);
            }
        }
        __syncthreads();             // the row's values are read; the next row may overwrite them
    }
    if (a.stats) finish_stats(acc, a.ws, a.stats, false, 0.0f, 0.0, true);
}

// ---------------------------------------------------------------------------
// Launchers.
// ---------------------------------------------------------------------------

namespace {

// Resident CTAs per SM of one kernel at one block size and dynamic shared memory size
// (cached per instantiation; raises the kernel's dynamic shared memory limit first).
template <auto KERN, int BLOCK, uint32_t SMEM>
int resident_ctas()
{
    static std::atomic<int> cached{-1};
    int v = cached.load(std::memory_order_relaxed);
    if (v < 0) {
        if (SMEM > 48u * 1024u) cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, KERN, BLOCK, SMEM) != cudaSuccess || v < 1) v = 1;
        cached.store(v, std::memory_order_relaxed);
    }
    return v;
}

// Grid of at most one wave (SM count x resident CTAs), at least enough CTAs to give
// each min_items_per_cta items, capped at the workspace slot count.
template <auto KERN, int BLOCK, uint32_t SMEM>
unsigned grid_for(uint64_t min_items_per_cta, uint64_t total_items)
{
    const uint64_t waves = (uint64_t)device_sm_count() * (uint64_t)resident_ctas<KERN, BLOCK, SMEM>();
    uint64_t need = (total_items + min_items_per_cta - 1) / min_items_per_cta;
    if (need < 1) need = 1;
    uint64_t g = need < waves ? need : waves;
    if (g > (uint64_t)MAX_GRID) g = MAX_GRID;
    return (unsigned)g;
}

}  // namespace

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to libcuda).
EncodeTiled encode_tiled()
{
    static std::atomic<void*> fn{nullptr};
    void* f = fn.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn.store(f, std::memory_order_release);
    }
    return reinterpret_cast<EncodeTiled>(f);
}

namespace {

// x seen as rows of 64 bf16 (128 bytes): boxes of box_rows rows (8: one octet, 1 KiB;
// 32: a whole tile), 128-byte swizzle, zero fill past the last row. rows = 0: a zeroed
// map that no launch reads.
cudaError_t x_rows_map(const uint32_t* x, uint32_t rows, uint32_t box_rows, CUtensorMap* map)
{
    *map = CUtensorMap{};
    if (rows == 0) return cudaSuccess;
    const EncodeTiled enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {64, rows};
    const cuuint64_t strides[1] = {ROW_BYTES};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint32_t*>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// x seen as [rows][cols / 64][64]: boxes of 32 segments of one row, 128-byte swizzle,
// zero fill past a row's end.
cudaError_t x_segments_map(const uint32_t* x, uint32_t rows, uint32_t cols, CUtensorMap* map)
{
    *map = CUtensorMap{};
    const EncodeTiled enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {64, cols / 64, rows};
    const cuuint64_t strides[2] = {ROW_BYTES, (cuuint64_t)cols * 2};
    const cuuint32_t box[3] = {64, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint32_t*>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int FMT, bool HAD, bool STATS, bool EXACT>
cudaError_t run_rows(const RowsArgs& a, cudaStream_t st)
{
    constexpr int block = ROWS_WARPS * 32;
    CUtensorMap map;
    const cudaError_t e = x_segments_map(a.x, a.rows, a.cols, &map);
    if (e != cudaSuccess) return e;
    if (a.tiles == 3u || a.tiles == 4u) {
        constexpr auto kern = k_quant_rows<FMT, HAD, STATS, EXACT, 4>;
        constexpr uint32_t smem = rows_smem(4);            // above 48 KiB: resident_ctas opts in
        const unsigned grid = grid_for<kern, block, smem>(ROWS_WARPS, a.rows);
        return launch_pdl(kern, grid, block, smem, st, map, a);
    } else {
        constexpr auto kern = k_quant_rows<FMT, HAD, STATS, EXACT, 2>;
        constexpr uint32_t smem = rows_smem(2);
        const unsigned grid = grid_for<kern, block, smem>(ROWS_WARPS, a.rows);
        return launch_pdl(kern, grid, block, smem, st, map, a);
    }
}

// The exact (value-domain) integer path: integer formats, fp16 scales, unrotated input.
template <int FMT>
constexpr bool can_exact() { return Fmt<FMT>::is_int; }

template <int FMT>
cudaError_t run_rows_hs(bool had, bool stats, const RowsArgs& a, cudaStream_t st)
{
    if (had) return stats ? run_rows<FMT, true, true, false>(a, st) : run_rows<FMT, true, false, false>(a, st);
    if constexpr (can_exact<FMT>()) {
        if (a.scale_fp16)
            return stats ? run_rows<FMT, false, true, true>(a, st) : run_rows<FMT, false, false, true>(a, st);
    }
    return stats ? run_rows<FMT, false, true, false>(a, st) : run_rows<FMT, false, false, false>(a, st);
}

// x seen as [rows][cols]: boxes of 128 rows x 64 columns, 128-byte swizzle, zero fill
// past the last row.
cudaError_t x_tiles_map(const uint32_t* x, uint32_t rows, uint32_t cols, CUtensorMap* map)
{
    *map = CUtensorMap{};
    const EncodeTiled enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, TILE};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint32_t*>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int FMT, bool HAD, bool STATS, bool EXACT>
cudaError_t run_tile2d(const Tile2dArgs& a, cudaStream_t st)
{
    constexpr int block = 256;
    constexpr auto kern = k_quant_tile2d<FMT, HAD, STATS, EXACT>;
    CUtensorMap map;
    const cudaError_t e = x_tiles_map(a.x, a.rows, a.cols, &map);
    if (e != cudaSuccess) return e;
    const unsigned grid = grid_for<kern, block, TILE2D_SMEM>(1, a.ntiles);
    return launch_pdl(kern, grid, block, TILE2D_SMEM, st, map, a);
}

template <int FMT>
cudaError_t run_tile2d_hs(bool had, bool stats, const Tile2dArgs& a, cudaStream_t st)
{
    if (had) return stats ? run_tile2d<FMT, true, true, false>(a, st) : run_tile2d<FMT, true, false, false>(a, st);
    if constexpr (can_exact<FMT>()) {
        if (a.scale_fp16)
            return stats ? run_tile2d<FMT, false, true, true>(a, st) : run_tile2d<FMT, false, false, true>(a, st);
    }
    return stats ? run_tile2d<FMT, false, true, false>(a, st) : run_tile2d<FMT, false, false, false>(a, st);
}

template <int FMT, bool MX>
cudaError_t run_rt(const RtArgs& a, cudaStream_t st)
{
    // a thread per chunk of the row, up to RT_THREADS (narrow rows: more CTAs per SM)
    const int block = a.cpr < (uint32_t)RT_THREADS ? (int)a.cpr : RT_THREADS;
    constexpr auto kern = k_quant_rt<FMT, MX>;
    const size_t smem = rot_smem_bytes(a.cols, a.sign_bits != nullptr);
    if (smem > 48u * 1024u) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, block, smem) != cudaSuccess || occ < 1) occ = 1;
    uint64_t grid = (uint64_t)device_sm_count() * (uint64_t)occ;
    if (grid > a.rows) grid = a.rows;
    if (grid > (uint64_t)MAX_GRID) grid = MAX_GRID;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, (unsigned)grid, (unsigned)block, smem, st, a);
}

template <int FMT, int GK, bool HAD, bool STATS, bool EXACT>
cudaError_t run_flat(const FlatArgs& a, cudaStream_t st)
{
    constexpr int block = FLAT_WARPS * 32;
    constexpr auto kern = k_quant_flat<FMT, GK, HAD, STATS, EXACT>;
    CUtensorMap map, map32;
    cudaError_t e = x_rows_map(a.x, a.n_chunks / SPAN, 8u, &map);
    if (e != cudaSuccess) return e;
    e = x_rows_map(a.x, a.n_chunks / SPAN, 32u, &map32);
    if (e != cudaSuccess) return e;
    // one partition unit per warp at least, and (a batch) a warp per tensor at least;
    // at most one stats slot per warp
    const uint64_t units = (uint64_t)a.batch * ((((uint64_t)a.spans_per_tensor + 7) / 8) / a.unit_oct);
    unsigned grid = grid_for<kern, block, FLAT_SMEM>(FLAT_WARPS, units);
    const unsigned min_grid = (a.batch + FLAT_WARPS - 1) / FLAT_WARPS;
    if (grid < min_grid) grid = min_grid;
    if (grid > MAX_STAT_SLOTS / FLAT_WARPS) grid = MAX_STAT_SLOTS / FLAT_WARPS;
    if (grid * FLAT_WARPS < a.batch) return cudaErrorInvalidValue;
    return launch_pdl(kern, grid, block, FLAT_SMEM, st, map, map32, a);
}

template <int FMT, int GK>
cudaError_t run_flat_hs(bool had, bool stats, const FlatArgs& a, cudaStream_t st)
{
    if (had) return stats ? run_flat<FMT, GK, true, true, false>(a, st) : run_flat<FMT, GK, true, false, false>(a, st);
    if constexpr (can_exact<FMT>() && (GK == K_TENSOR || GK == K_GROUP)) {
        if (a.scale_fp16)
            return stats ? run_flat<FMT, GK, false, true, true>(a, st) : run_flat<FMT, GK, false, false, true>(a, st);
    }
    return stats ? run_flat<FMT, GK, false, true, false>(a, st) : run_flat<FMT, GK, false, false, false>(a, st);
}

template <bool HAD, bool MINMAX>
cudaError_t run_range(const uint32_t* x, uint32_t n_chunks, uint8_t* ws, float* out, cudaStream_t st)
{
    constexpr int block = 256;
    constexpr auto kern = k_range<HAD, MINMAX>;
    const unsigned grid = grid_for<kern, block, 0>((uint64_t)block * 4, n_chunks);
    return launch_pdl(kern, grid, block, 0, st, x, n_chunks, ws, out);
}

}  // namespace

cudaError_t flat_wait_timeouts(unsigned int* count, bool reset)
{
    cudaError_t e = cudaMemcpyFromSymbol(count, g_flat_wait_timeouts, sizeof(unsigned int));
    if (e == cudaSuccess && reset) {
        const unsigned int zero = 0u;
        e = cudaMemcpyToSymbol(g_flat_wait_timeouts, &zero, sizeof(unsigned int));
    }
    return e;
}

cudaError_t launch_range(const uint32_t* x, uint32_t n_chunks, bool had, bool minmax, uint8_t* ws, float* out,
                         cudaStream_t st)
{
    if (had) return minmax ? run_range<true, true>(x, n_chunks, ws, out, st) : run_range<true, false>(x, n_chunks, ws, out, st);
    return minmax ? run_range<false, true>(x, n_chunks, ws, out, st) : run_range<false, false>(x, n_chunks, ws, out, st);
}

cudaError_t launch_quant_rows(int fmt, bool had, bool stats, const RowsArgs& a, cudaStream_t st)
{
    switch (fmt) {
    case BQ_INT8_SYM:   return run_rows_hs<BQ_INT8_SYM>(had, stats, a, st);
    case BQ_INT8_ASYM:  return run_rows_hs<BQ_INT8_ASYM>(had, stats, a, st);
    case BQ_INT4_SYM:   return run_rows_hs<BQ_INT4_SYM>(had, stats, a, st);
    case BQ_UINT4_ASYM: return run_rows_hs<BQ_UINT4_ASYM>(had, stats, a, st);
    case BQ_FP8_E4M3:   return run_rows_hs<BQ_FP8_E4M3>(had, stats, a, st);
    case BQ_FP8_E5M2:   return run_rows_hs<BQ_FP8_E5M2>(had, stats, a, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_quant_tile2d(int fmt, bool had, bool stats, const Tile2dArgs& a, cudaStream_t st)
{
    switch (fmt) {
    case BQ_INT8_SYM:   return run_tile2d_hs<BQ_INT8_SYM>(had, stats, a, st);
    case BQ_INT8_ASYM:  return run_tile2d_hs<BQ_INT8_ASYM>(had, stats, a, st);
    case BQ_INT4_SYM:   return run_tile2d_hs<BQ_INT4_SYM>(had, stats, a, st);
    case BQ_UINT4_ASYM: return run_tile2d_hs<BQ_UINT4_ASYM>(had, stats, a, st);
    case BQ_FP8_E4M3:   return run_tile2d_hs<BQ_FP8_E4M3>(had, stats, a, st);
    case BQ_FP8_E5M2:   return run_tile2d_hs<BQ_FP8_E5M2>(had, stats, a, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_quant_rt(int fmt, bool mx, const RtArgs& a, cudaStream_t st)
{
    // rotated rows of 1024, 2048 or 4096 columns: the two-pass kernels
    if (a.sign_bits && rt64_cols(a.cols) && a.rows > 0) return launch_quant_rt64(fmt, mx, a, st);
    if (mx) {
        switch (fmt) {
        case BQ_INT8_SYM: return run_rt<BQ_INT8_SYM, true>(a, st);
        case BQ_FP8_E4M3: return run_rt<BQ_FP8_E4M3, true>(a, st);
        case BQ_FP8_E5M2: return run_rt<BQ_FP8_E5M2, true>(a, st);
        case BQ_FP4_E2M1: return run_rt<BQ_FP4_E2M1, true>(a, st);
        case BQ_FP6_E2M3: return run_rt<BQ_FP6_E2M3, true>(a, st);
        case BQ_FP6_E3M2: return run_rt<BQ_FP6_E3M2, true>(a, st);
        default: return cudaErrorInvalidValue;
        }
    }
    switch (fmt) {
    case BQ_INT8_SYM:   return run_rt<BQ_INT8_SYM, false>(a, st);
    case BQ_INT8_ASYM:  return run_rt<BQ_INT8_ASYM, false>(a, st);
    case BQ_INT4_SYM:   return run_rt<BQ_INT4_SYM, false>(a, st);
    case BQ_UINT4_ASYM: return run_rt<BQ_UINT4_ASYM, false>(a, st);
    case BQ_FP8_E4M3:   return run_rt<BQ_FP8_E4M3, false>(a, st);
    case BQ_FP8_E5M2:   return run_rt<BQ_FP8_E5M2, false>(a, st);
    default: return cudaErrorInvalidValue;
    }
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
        case BQ_FP6_E2M3: return run_flat_hs<BQ_FP6_E2M3, K_MX>(had, stats, a, st);
        case BQ_FP6_E3M2: return run_flat_hs<BQ_FP6_E3M2, K_MX>(had, stats, a, st);
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
