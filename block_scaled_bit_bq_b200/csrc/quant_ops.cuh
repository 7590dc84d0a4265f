// quant_ops.cuh -- quantize one 16-element chunk given its unit's scale, on fp32 pairs.
//
// Code rules ("INT vs FP at fine granularity" §2.1, "INT4/INT8/FP8 quantization"
// §INT8/§INT4, "Quantization survey" §4.1):
//   INT:  q = clamp(rne(x / s) [+ zp], Qmin, Qmax)
//   FP:   code = cvt.rn.satfinite(x / s)
// with x / s the correctly rounded fp32 quotient.
//
// INT codes come from one fused multiply-add per element with r ~ 1/s (within 2^-23):
// t = RN(x r + M) with M = 1.5 * 2^23 (+ zero point + bias) leaves the integer nearest
// to x r in t's low bits, and the residual f = x r - q (one more FMA) says how far x r
// is from a rounding boundary. Whenever |f| < 1/2 - (|x/s| + 2) 2^-21 the quotient
// RN(x / s) lies strictly inside q's rounding interval, so q is its code. The rest
// (about 1e-3 of the elements for bf16 inputs over fp16 scales, nearly all of them
// exact half-integer quotients) are settled exactly: an exact FMA residual recognises
// x / s == q +- 1/2 (the code is then the even neighbour) and anything else divides.
// FP codes use a reciprocal bracket: cvt of x r_lo and of x r_hi, r_lo < 1/s < r_hi;
// where the two differ the element divides.
//
// The chunk functions are warp-collective: every lane of a warp calls them together
// (lanes with nothing to do pass zeros), because their rare-case branches are taken by
// the whole warp when any lane needs them.
#pragma once

#include <cfloat>
#include <type_traits>

#include "common.cuh"

namespace bq {

template <int FMT> struct CodeWords { static constexpr int n = Fmt<FMT>::four ? 2 : 4; };

// Offset added to signed 4-bit codes so that the nibbles are non-negative while they
// are assembled (undone with one XOR per word).
template <int FMT> struct CodeBias { static constexpr int v = (FMT == BQ_INT4_SYM) ? 8 : 0; };

// ---------------------------------------------------------------------------
// Ranges.
// ---------------------------------------------------------------------------

__device__ __forceinline__ float chunk_amax(const float2 (&y)[8], float m)
{
    // a tree of three-input maxima (depth 3) instead of a chain of eight
    const float a0 = amax3(fabsf(y[0].x), y[0].y, y[1].x);
    const float a1 = amax3(fabsf(y[1].y), y[2].x, y[2].y);
    const float a2 = amax3(fabsf(y[3].x), y[3].y, y[4].x);
    const float a3 = amax3(fabsf(y[4].y), y[5].x, y[5].y);
    const float a4 = amax3(fabsf(y[6].x), y[6].y, y[7].x);
    const float b0 = amax3(a0, a1, a2), b1 = amax3(a3, a4, y[7].y);
    return max3(m, b0, b1);
}

__device__ __forceinline__ void chunk_minmax(const float2 (&y)[8], float& mn, float& mx)
{
    float lo[3], hi[3];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float2 a = y[3 * j], b = y[3 * j + 1], c = y[3 * j + 2];
        lo[j] = min3(min3(a.x, a.y, b.x), b.y, fminf(c.x, c.y));
        hi[j] = max3(max3(a.x, a.y, b.x), b.y, fmaxf(c.x, c.y));
    }
    lo[2] = min3(y[6].x, y[6].y, fminf(y[7].x, y[7].y));
    hi[2] = max3(y[6].x, y[6].y, fmaxf(y[7].x, y[7].y));
    mn = min3(mn, min3(lo[0], lo[1], lo[2]), mn);
    mx = max3(mx, max3(hi[0], hi[1], hi[2]), mx);
}

// on raw bf16 words (no widening); pairwise trees
__device__ __forceinline__ uint32_t words_absmax(const uint32_t (&w)[8], uint32_t m)
{
    uint32_t a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = bf2_absmax(w[2 * i] & 0x7FFF7FFFu, w[2 * i + 1]);
    return bf2_absmax(m, __vmaxu2(__vmaxu2(a[0], a[1]), __vmaxu2(a[2], a[3])));
}

__device__ __forceinline__ void words_minmax(const uint32_t (&w)[8], uint32_t& mn, uint32_t& mx)
{
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lo[i] = bf2_min(w[2 * i], w[2 * i + 1]);
        hi[i] = bf2_max(w[2 * i], w[2 * i + 1]);
    }
    mn = bf2_min(mn, bf2_min(bf2_min(lo[0], lo[1]), bf2_min(lo[2], lo[3])));
    mx = bf2_max(mx, bf2_max(bf2_max(hi[0], hi[1]), bf2_max(hi[2], hi[3])));
}

// ---------------------------------------------------------------------------
// Out-of-line slow paths. They run for a small fraction of the elements (or of the
// units); keeping them out of line keeps the hot loops small for the instruction
// cache.
// ---------------------------------------------------------------------------

// rne(RN(y / s)) as a float, clamped to +-2^22 (far outside every code range).
static __device__ __noinline__ float div_rne_clamped(float y, float s)
{
    const float v = rintf(__fdiv_rn(y, s));
    return fminf(fmaxf(v, -4194304.0f), 4194304.0f);
}

// The correctly rounded quotient a / b.
static __device__ __noinline__ float div_rn_call(float a, float b) { return __fdiv_rn(a, b); }

// FP codes of RN(hi / s) (upper byte) and RN(lo / s) (lower byte).
template <int FMT>
static __device__ __noinline__ uint32_t fp_div_pair(float hi, float lo, float s)
{
    return cvt_pair<FMT>(__fdiv_rn(hi, s), __fdiv_rn(lo, s));
}

// ---------------------------------------------------------------------------
// Integer units.
// ---------------------------------------------------------------------------

struct IntQ {
    float s;        // the scale x is divided by (0: every code is the zero point)
    float r;        // ~ 1/s (0 when s == 0)
    float rlo, rhi; // r (1 -+ 2^-22): strictly below and above 1/s (0 when s == 0)
    float mz;       // MAGIC + zero point + bias (exact)
    float thr;      // |f| below thr: the code is certain
    float xc;       // asymmetric: inputs above xc take the code qmax (+inf: none do)
    float rn;       // RN(1/s), the correctly rounded reciprocal (0 when s == 0)
    bool mk;        // the fast paths' exact quotient holds for every element of the unit
    bool fast;      // s in the range where the residual test is valid
    bool br;        // the bracket decides every code of the unit (fp16 scales, see int_chunk_exact)
    bool clamp;     // codes must be clamped (beyond what xc does)
};

// Unit from its stored scale s, a reciprocal r of it (exact: r = RN(1/s); else within
// an ulp), its zero point zpf and the extreme values lo <= 0 <= hi it holds; qmin / qmax:
// the code range.
template <int FMT>
__device__ __forceinline__ IntQ int_unit(float s, float r, bool r_exact, float zpf, float lo, float hi, int qmin, int qmax)
{
    constexpr float bias = (float)CodeBias<FMT>::v;
    IntQ u;
    u.s = s;
    u.mz = __fadd_rn(__fadd_rn(MAGIC, zpf), bias);
    u.xc = __int_as_float(0x7F800000);
    if (!(s > 0.0f)) {
        u.r = u.rlo = u.rhi = u.rn = 0.0f;
        u.thr = 1.0f;
        u.fast = u.br = u.mk = true;
        u.clamp = false;
        return u;
    }
    u.r = r;
    u.rn = r;
    u.rlo = __fmul_rn(u.r, 0x1.fffff8p-1f);                        // 1 - 2^-22
    u.rhi = __fmul_rn(u.r, 0x1.000004p+0f);                        // 1 + 2^-22
    const float bound = __fmul_rn(fmaxf(-lo, hi), u.r);          // ~ max |x / s|
    u.fast = (s >= 0x1p-100f) && (s <= 1.0e37f) && (bound < 4.0e6f);
    u.br = u.fast && bound < 400.0f;
    u.mk = r_exact && (s >= 0x1p-60f) && (s <= 0x1p100f) && (bound < 0x1p20f);
    u.thr = __fsub_rn(0.5f, __fmul_rn(__fadd_rn(bound, 2.0f), 0x1p-21f));
    if constexpr (Fmt<FMT>::asym) {
        // The code is monotone in x, so the extremes bound every code: rne(hi r_hi) + zp
        // bounds the top one, rne(lo r_hi) + zp the bottom one. With zp = qmin +
        // rne(-lo / s) the bottom code is qmin (round-half-even is odd-symmetric), and the
        // top one can exceed qmax by one, when both -lo/s and hi/s lie near half-integers.
        // Then inputs are capped at xc = (qmax - zp) s, whose quotient is exactly
        // qmax - zp: the capped inputs take the code qmax, the others keep theirs.
        bool under = false;
        if (u.fast) {
            const float qt = __fsub_rn(__fmaf_rn(hi, u.rhi, MAGIC), MAGIC);
            const float qb = __fsub_rn(__fmaf_rn(lo, u.rhi, MAGIC), MAGIC);
            if (__fadd_rn(qt, zpf) > (float)qmax) u.xc = __fmul_rn(__fsub_rn((float)qmax, zpf), s);
            under = __fadd_rn(qb, zpf) < (float)qmin;
        }
        u.clamp = !u.fast || under;
    } else {
        // |x / s| <= Qmax (1 + 2^-10) for an AbsMax scale: a quarter step of slack
        const float top = __fadd_rn(__fmul_rn(hi, u.r), zpf), bot = __fadd_rn(__fmul_rn(lo, u.r), zpf);
        u.clamp = !u.fast || top > (float)qmax + 0.25f || bot < (float)qmin - 0.25f;
    }
    return u;
}

// Exact code (magic form, t = mz + q) of one element whose residual test was
// inconclusive.
static __device__ __noinline__ float settle(float y, float s, float r, float mz, float t)
{
    const float q = __fsub_rn(t, mz);                        // exact
    const float f = __fmaf_rn(y, r, -q);
    const float side = f > 0.0f ? 0.5f : -0.5f;
    const float h = __fadd_rn(q, side);                      // the half-integer next to q
    if (__fmaf_rn(-h, s, y) == 0.0f) {
        // x / s == h exactly: RN(x/s) = h, which rounds half to even
        const bool q_even = (__float_as_uint(__fadd_rn(q, MAGIC)) & 1u) == 0u;
        const float qe = q_even ? q : __fadd_rn(q, __fadd_rn(side, side));
        return __fadd_rn(qe, mz);
    }
    return __fadd_rn(div_rne_clamped(y, s), mz);
}

// Integer chunk: codes into w; nq[i] = -(code - zp) (exact) when NEED_Q. CHECK: test
// for codes outside [qmin, qmax] (a caller passes false only for units whose clamp
// flag is clear in every lane of the warp).
template <int FMT, bool NEED_Q, bool CHECK = true>
__device__ __forceinline__ void int_chunk(const float2 (&y)[8], const IntQ& u, int qmin, int qmax,
                                          uint32_t (&w)[CodeWords<FMT>::n], float2 (&nq)[8])
{
    using F = Fmt<FMT>;
    constexpr float bias = (float)CodeBias<FMT>::v;
    float2 t[8], nqq[8], f[8], yq[8];
    const float2 R = splat(u.r), MZ = splat(u.mz), M1 = splat(-1.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        // asymmetric: inputs capped at xc for the code (the sums use y itself)
        yq[i] = F::asym ? make_float2(fminf(y[i].x, u.xc), fminf(y[i].y, u.xc)) : y[i];
        t[i] = fma2(yq[i], R, MZ);
        nqq[i] = fma2(t[i], M1, MZ);          // -q, exact
        f[i] = fma2(yq[i], R, nqq[i]);
    }
    const float fm = chunk_amax(f, 0.0f);
    const bool rare = !u.fast || !(fm < u.thr);
    if (__any_sync(0xFFFFFFFFu, rare)) {
        if (rare) {
            if (u.fast) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (!(fabsf(f[i].x) < u.thr)) t[i].x = settle(yq[i].x, u.s, u.r, u.mz, t[i].x);
                    if (!(fabsf(f[i].y) < u.thr)) t[i].y = settle(yq[i].y, u.s, u.r, u.mz, t[i].y);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    t[i] = make_float2(__fadd_rn(div_rne_clamped(yq[i].x, u.s), u.mz),
                                       __fadd_rn(div_rne_clamped(yq[i].y, u.s), u.mz));
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) nqq[i] = fma2(t[i], M1, MZ);
    }
    if (CHECK && __any_sync(0xFFFFFFFFu, u.clamp)) {
        // the bounds hold the code + bias whatever the zero point; clamping is the
        // identity for units that never leave the range
        const float cmin = MAGIC + (float)qmin + bias, cmax = MAGIC + (float)qmax + bias;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            t[i] = make_float2(fminf(fmaxf(t[i].x, cmin), cmax), fminf(fmaxf(t[i].y, cmin), cmax));
#pragma unroll
        for (int i = 0; i < 8; ++i) nqq[i] = fma2(t[i], M1, MZ);
    }
    if constexpr (NEED_Q) {
#pragma unroll
        for (int i = 0; i < 8; ++i) nq[i] = nqq[i];
    }
    if constexpr (F::four) {
        // t's low bits hold code + bias in [0, 15]: four codes per multiply-add chain
        // (MAGIC's bits start at bit 22, so they never reach bits 0..15)
        uint32_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t a = __float_as_uint(t[2 * k].x), b = __float_as_uint(t[2 * k].y);
            const uint32_t c = __float_as_uint(t[2 * k + 1].x), d = __float_as_uint(t[2 * k + 1].y);
            h[k] = a + b * 16u + c * 256u + d * 4096u;
        }
        w[0] = __byte_perm(h[0], h[1], 0x5410);
        w[1] = __byte_perm(h[2], h[3], 0x5410);
        if constexpr (CodeBias<FMT>::v == 8) { w[0] ^= 0x88888888u; w[1] ^= 0x88888888u; }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = pack_bytes(__float_as_uint(t[2 * k].x), __float_as_uint(t[2 * k].y),
                              __float_as_uint(t[2 * k + 1].x), __float_as_uint(t[2 * k + 1].y));
    }
}

// Integer chunk for a scale with at most 11 significant bits (an fp16 scale) and
// unrotated bf16 inputs (x has 8 significant bits).
//
// Then x / s is either an exact half-integer (a tie) or at least 2^-12 away from every
// half-integer: 2x - (2k+1) s is a multiple of min(2 ulp(x), ulp(s)), and dividing by 2s
// leaves at least 2^-12 (ulp(s) > s 2^-11; and 2 ulp(x) > |x| 2^-7 >= s 2^-8 whenever
// |x/s| >= 1/2). The codes rne(x r_lo) and rne(x r_hi) of the bracket
// r_lo < 1/s < r_hi are within |x/s| 1.25 2^-21 of it, less than 2^-12 for |x/s| < 400,
// so they agree with rne(x/s) off ties. On a tie they are the two neighbours k, k+1,
// and round-half-even takes the even one. So the code is the bracket code whose q is
// even, and no element divides or branches.
//
// e[i] = x - q_lo s (exact) for the QSNR sums: off ties q_lo is the code, on a tie both
// neighbours are s/2 away, so e^2 is the final code's either way.
// GENERAL: clamp to [qmin, qmax] (e then follows the clamped code).
template <int FMT, bool NEED_E, bool GENERAL>
__device__ __forceinline__ void int_chunk_exact(const float2 (&y)[8], const IntQ& u, int qmin, int qmax,
                                                uint32_t (&w)[CodeWords<FMT>::n], float2 (&e)[8])
{
    using F = Fmt<FMT>;
    constexpr float bias = (float)CodeBias<FMT>::v;
    float2 tl[8], th[8], yq[8];
    const float2 RL = splat(u.rlo), RH = splat(u.rhi), MZ = splat(u.mz), M1 = splat(-1.0f), S = splat(u.s);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        // asymmetric: inputs capped at xc for the code (the residuals use y itself)
        yq[i] = F::asym ? make_float2(fminf(y[i].x, u.xc), fminf(y[i].y, u.xc)) : y[i];
        tl[i] = fma2(yq[i], RL, MZ);
        th[i] = fma2(yq[i], RH, MZ);
    }
    if (GENERAL && __any_sync(0xFFFFFFFFu, !u.br)) {
        // units outside the bracket's range (huge quotients): correctly rounded quotients
        // (without GENERAL the caller guarantees br)
        if (!u.br) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                tl[i] = make_float2(__fadd_rn(div_rne_clamped(yq[i].x, u.s), u.mz),
                                    __fadd_rn(div_rne_clamped(yq[i].y, u.s), u.mz));
                th[i] = tl[i];
            }
        }
    }
    // parity of q = t - mz from t's bits: t = MAGIC + zp + bias + q and MAGIC is even
    const uint32_t zb = (uint32_t)(int)__fsub_rn(u.mz, MAGIC) & 1u;
    if constexpr (!GENERAL) {
        // every code is in range: select per packed code (nibble or byte) with one LOP3
        if constexpr (F::four) {
            uint32_t hl[4], hh[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                hl[k] = __float_as_uint(tl[2 * k].x) + __float_as_uint(tl[2 * k].y) * 16u +
                        __float_as_uint(tl[2 * k + 1].x) * 256u + __float_as_uint(tl[2 * k + 1].y) * 4096u;
                hh[k] = __float_as_uint(th[2 * k].x) + __float_as_uint(th[2 * k].y) * 16u +
                        __float_as_uint(th[2 * k + 1].x) * 256u + __float_as_uint(th[2 * k + 1].y) * 4096u;
                const uint32_t odd = (hl[k] ^ (zb * 0x1111u)) & 0x1111u;
                const uint32_t m = odd * 15u;
                hl[k] = (hl[k] & ~m) | (hh[k] & m);
            }
            w[0] = __byte_perm(hl[0], hl[1], 0x5410);
            w[1] = __byte_perm(hl[2], hl[3], 0x5410);
            if constexpr (CodeBias<FMT>::v == 8) { w[0] ^= 0x88888888u; w[1] ^= 0x88888888u; }
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t bl = pack_bytes(__float_as_uint(tl[2 * k].x), __float_as_uint(tl[2 * k].y),
                                               __float_as_uint(tl[2 * k + 1].x), __float_as_uint(tl[2 * k + 1].y));
                const uint32_t bh = pack_bytes(__float_as_uint(th[2 * k].x), __float_as_uint(th[2 * k].y),
                                               __float_as_uint(th[2 * k + 1].x), __float_as_uint(th[2 * k + 1].y));
                const uint32_t odd = (bl ^ (zb * 0x01010101u)) & 0x01010101u;
                const uint32_t m = odd * 255u;
                w[k] = (bl & ~m) | (bh & m);
            }
        }
        if constexpr (NEED_E) {
#pragma unroll
            for (int i = 0; i < 8; ++i) e[i] = fma2(fma2(tl[i], M1, MZ), S, y[i]);
        }
    } else {
        const float cmin = MAGIC + (float)qmin + bias, cmax = MAGIC + (float)qmax + bias;
        float2 t[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float a = ((__float_as_uint(tl[i].x) ^ zb) & 1u) ? th[i].x : tl[i].x;
            const float b = ((__float_as_uint(tl[i].y) ^ zb) & 1u) ? th[i].y : tl[i].y;
            t[i] = make_float2(fminf(fmaxf(a, cmin), cmax), fminf(fmaxf(b, cmin), cmax));
            if constexpr (NEED_E) e[i] = fma2(fma2(t[i], M1, MZ), S, y[i]);
        }
        if constexpr (F::four) {
            uint32_t h[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                h[k] = __float_as_uint(t[2 * k].x) + __float_as_uint(t[2 * k].y) * 16u +
                       __float_as_uint(t[2 * k + 1].x) * 256u + __float_as_uint(t[2 * k + 1].y) * 4096u;
            w[0] = __byte_perm(h[0], h[1], 0x5410);
            w[1] = __byte_perm(h[2], h[3], 0x5410);
            if constexpr (CodeBias<FMT>::v == 8) { w[0] ^= 0x88888888u; w[1] ^= 0x88888888u; }
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                w[k] = pack_bytes(__float_as_uint(t[2 * k].x), __float_as_uint(t[2 * k].y),
                                  __float_as_uint(t[2 * k + 1].x), __float_as_uint(t[2 * k + 1].y));
        }
    }
}

// ---------------------------------------------------------------------------
// FP element chunks.
// ---------------------------------------------------------------------------

struct FpQ {
    float s;        // the scale x is divided by
    float rlo, rhi; // reciprocal bracket
    float rn;       // RN(1/s) (0 when s == 0)
    bool fast;
    bool zero;      // s == 0: every code is +0
    bool mk;        // the exact reciprocal-correction quotient holds for every element
};

// rn: RN(1/s) (exact), or 0 when the caller has none (then mk is false).
__device__ __forceinline__ FpQ fp_unit(float s, float amax, float rn = 0.0f)
{
    FpQ u;
    u.s = s;
    u.zero = !(s > 0.0f);
    const Recip R = make_recip(s, amax);
    u.rlo = u.zero ? 0.0f : R.rlo;
    u.rhi = u.zero ? 0.0f : R.rhi;
    u.fast = R.fast && !u.zero;
    u.rn = u.zero ? 0.0f : rn;
    u.mk = u.zero || (rn > 0.0f && (s >= 0x1p-60f) && (s <= 0x1p100f) && __fmul_rn(amax, rn) < 0x1p20f);
    return u;
}

template <int FMT>
__device__ __forceinline__ void pack_pairs(const uint32_t (&pr)[8], uint32_t (&w)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) {
        w[0] = pack_bytes(pr[0], pr[1], pr[2], pr[3]);
        w[1] = pack_bytes(pr[4], pr[5], pr[6], pr[7]);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = __byte_perm(pr[2 * k], pr[2 * k + 1], 0x5410);
    }
}

template <int FMT>
__device__ __forceinline__ void decode_pairs(const uint32_t (&pr)[8], float2 (&val)[8])
{
#pragma unroll
    for (int p = 0; p < 8; ++p) val[p] = dec_pair<FMT>(pr[p]);
}

// Codes of x / s (s > 0) or +0 codes (s == 0); val = decoded element values (NEED_V).
template <int FMT, bool NEED_V>
__device__ __forceinline__ void fp_chunk(const float2 (&y)[8], const FpQ& u,
                                         uint32_t (&w)[CodeWords<FMT>::n], float2 (&val)[8])
{
    uint32_t pr[8];
    uint32_t mism = 0;
    const float2 lo = splat(u.rlo), hi = splat(u.rhi);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const float2 a = mul2(y[p], lo), b = mul2(y[p], hi);
        const uint32_t cl = cvt_pair<FMT>(a.y, a.x);
        const uint32_t ch = cvt_pair<FMT>(b.y, b.x);
        mism |= cl ^ ch;
        pr[p] = cl;
    }
    const bool rare = u.zero || !u.fast || mism != 0u;
    if (__any_sync(0xFFFFFFFFu, rare)) {
        if (rare) {
            if (u.zero) {
#pragma unroll
                for (int p = 0; p < 8; ++p) pr[p] = 0u;
            } else {
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const float2 a = mul2(y[p], lo), b = mul2(y[p], hi);
                    const bool bad = !u.fast || (cvt_pair<FMT>(a.y, a.x) != cvt_pair<FMT>(b.y, b.x));
                    if (bad) pr[p] = fp_div_pair<FMT>(y[p].y, y[p].x, u.s);
                }
            }
        }
    }
    pack_pairs<FMT>(pr, w);
    if constexpr (NEED_V) decode_pairs<FMT>(pr, val);
}

// Exact power-of-two scale: code = cvt(x * 2^-e) (the product is exact).
template <int FMT, bool NEED_V>
__device__ __forceinline__ void fp_chunk_pow2(const float2 (&y)[8], float p2,
                                              uint32_t (&w)[CodeWords<FMT>::n], float2 (&val)[8])
{
    uint32_t pr[8];
    const float2 p = splat(p2);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 a = mul2(y[i], p);
        pr[i] = cvt_pair<FMT>(a.y, a.x);
    }
    pack_pairs<FMT>(pr, w);
    if constexpr (NEED_V) decode_pairs<FMT>(pr, val);
}

// MXINT8: q = rne(x * 2^-e) (exact product, |q| <= 127 by the choice of e); nq = -q.
template <bool NEED_Q>
__device__ __forceinline__ void int8_chunk_pow2(const float2 (&y)[8], float p2, uint32_t (&w)[4], float2 (&nq)[8])
{
    float2 t[8];
    const float2 p = splat(p2), m = splat(MAGIC), M1 = splat(-1.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        t[i] = fma2(y[i], p, m);
        if constexpr (NEED_Q) nq[i] = fma2(t[i], M1, m);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
        w[k] = pack_bytes(__float_as_uint(t[2 * k].x), __float_as_uint(t[2 * k].y),
                          __float_as_uint(t[2 * k + 1].x), __float_as_uint(t[2 * k + 1].y));
}

// ---------------------------------------------------------------------------
// Plain (tensor / row / group) scales.
// ---------------------------------------------------------------------------

struct PlainScale {
    float s;        // stored scale (fp16-rounded when the dtype is fp16)
    float rn;       // RN(1/s) (0 when s == 0)
    float zpf;      // zero point as float (0 for symmetric)
    float lo, hi;   // extreme values the unit holds (-amax, amax for symmetric)
};

// RN(a / Qmax) for a >= 0: the reciprocal correction with the compile-time RN(1/Qmax)
// where it is exact (quotients in [2^-40, 2^20]: checked for every fp32 a and every
// Qmax), else a division.
template <int FMT>
__device__ __forceinline__ float div_by_qscale(float a)
{
    constexpr float Q = Fmt<FMT>::qscale;
    constexpr float RQ = 1.0f / Q;
    if (a >= 0x1p-40f * Q && a <= 0x1p20f * Q) {
        const float q0 = __fmul_rn(a, RQ);
        return __fmaf_rn(__fmaf_rn(-q0, Q, a), RQ, q0);
    }
    return a == 0.0f ? 0.0f : div_rn_call(a, Q);
}

template <int FMT>
__device__ __forceinline__ PlainScale plain_scale(float amax, float mn, float mx, bool fp16)
{
    using F = Fmt<FMT>;
    PlainScale p;
    if constexpr (F::asym) {
        const float lo = fminf(mn, 0.0f), hi = fmaxf(mx, 0.0f);
        const float range = __fsub_rn(hi, lo);
        float s32 = range <= FLT_MAX ? div_by_qscale<FMT>(range) : FLT_MAX;   // a range beyond fp32 saturates
        s32 = fminf(s32, FLT_MAX);
        p.s = fp16 ? round_scale_f16(s32) : s32;
        p.rn = p.s > 0.0f ? __frcp_rn(p.s) : 0.0f;
        if (p.s > 0.0f) {
            // zp = Qmin + rne(RN(-lo / s)): the exact quotient by the reciprocal correction
            // where it holds, else a division
            float z;
            if (p.s >= 0x1p-60f && p.s <= 0x1p100f && __fmul_rn(-lo, p.rn) < 0x1p20f) {
                const float q0 = __fmul_rn(-lo, p.rn);
                const float q1 = __fmaf_rn(__fmaf_rn(-q0, p.s, -lo), p.rn, q0);
                z = __fsub_rn(__fadd_rn(q1, MAGIC), MAGIC);
            } else {
                z = div_rne_clamped(-lo, p.s);
            }
            p.zpf = fminf(fmaxf(__fadd_rn((float)F::qmin, z), (float)F::qmin), (float)F::qmax);
        } else {
            p.zpf = (float)F::qmin;
        }
        p.lo = lo;
        p.hi = hi;
    } else {
        const float s32 = div_by_qscale<FMT>(amax);
        p.s = fp16 ? round_scale_f16(s32) : s32;
        p.rn = p.s > 0.0f ? __frcp_rn(p.s) : 0.0f;
        p.zpf = 0.0f;
        p.lo = -amax;
        p.hi = amax;
    }
    return p;
}

template <int FMT>
__device__ __forceinline__ void store_plain_scale(void* scales, void* zps, size_t i, const PlainScale& ps, bool fp16)
{
    if (fp16) {
        reinterpret_cast<__half*>(scales)[i] = __float2half_rn(ps.s);
        if constexpr (Fmt<FMT>::asym) reinterpret_cast<__half*>(zps)[i] = __float2half_rn(ps.zpf);
    } else {
        reinterpret_cast<float*>(scales)[i] = ps.s;
        if constexpr (Fmt<FMT>::asym) reinterpret_cast<float*>(zps)[i] = ps.zpf;
    }
}

// A plain unit, INT or FP.
template <int FMT>
struct PlainUnit {
    IntQ iq;
    FpQ fq;
    float s;
};

template <int FMT>
__device__ __forceinline__ PlainUnit<FMT> plain_unit(const PlainScale& ps)
{
    PlainUnit<FMT> u;
    u.s = ps.s;
    if constexpr (Fmt<FMT>::is_int) u.iq = int_unit<FMT>(ps.s, ps.rn, true, ps.zpf, ps.lo, ps.hi, Fmt<FMT>::qmin, Fmt<FMT>::qmax);
    else u.fq = fp_unit(ps.s, fmaxf(-ps.lo, ps.hi), ps.rn);
    return u;
}

// QSNR sums. Plain form (units whose values lie in [2^-40, 2^40]): e2 += (y - q s)^2
// and x2 += y^2 in fp32. Scaled form (any other unit): x-hat is formed in fp32 first
// (so an x-hat past the fp32 range is inf, as it is for the dequantized tensor), then
// the difference and y are scaled by the power of two p before squaring.
template <bool SCALED>
__device__ __forceinline__ void int_sums(const float2 (&y)[8], const float2 (&nq)[8], float s, float p,
                                         float2& e2, float2& x2)
{
    if constexpr (SCALED) {
        const float2 P = splat(p), nP = splat(-p), nS = splat(-s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 xh = mul2(nq[i], nS);
            const float2 yp = mul2(y[i], P);
            const float2 d = fma2(xh, nP, yp);
            e2 = fma2(d, d, e2);
            x2 = fma2(yp, yp, x2);
        }
    } else {
        const float2 S = splat(s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 d = fma2(nq[i], S, y[i]);
            e2 = fma2(d, d, e2);
            x2 = fma2(y[i], y[i], x2);
        }
    }
}

// Sums from exact residuals e = x - x-hat.
template <bool SCALED>
__device__ __forceinline__ void res_sums(const float2 (&y)[8], const float2 (&e)[8], float p, float2& e2, float2& x2)
{
    if constexpr (SCALED) {
        const float2 P = splat(p);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 d = mul2(e[i], P), yp = mul2(y[i], P);
            e2 = fma2(d, d, e2);
            x2 = fma2(yp, yp, x2);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            e2 = fma2(e[i], e[i], e2);
            x2 = fma2(y[i], y[i], x2);
        }
    }
}

// Sums from element values val with x-hat = val * s.
template <bool SCALED>
__device__ __forceinline__ void val_sums(const float2 (&y)[8], const float2 (&val)[8], float s, float p,
                                         float2& e2, float2& x2)
{
    if constexpr (SCALED) {
        const float2 P = splat(p), nP = splat(-p), S = splat(s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 xh = mul2(val[i], S);
            const float2 yp = mul2(y[i], P);
            const float2 d = fma2(xh, nP, yp);
            e2 = fma2(d, d, e2);
            x2 = fma2(yp, yp, x2);
        }
    } else {
        const float2 nS = splat(-s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 d = fma2(val[i], nS, y[i]);
            e2 = fma2(d, d, e2);
            x2 = fma2(y[i], y[i], x2);
        }
    }
}

// Quantize one chunk of a plain unit; STATS adds its sums. EXACT: the unit's scale has
// at most 11 significant bits (fp16) and y is unrotated bf16 (the value-domain residual
// decides the codes). GENERAL: clamping is tested and the sums take the scaled form when
// `scaled`; without it (a unit whose clamp flag is clear in every lane of the warp and
// whose sums are plain) neither is looked at.
template <int FMT, bool STATS, bool EXACT, bool GENERAL>
__device__ __forceinline__ void plain_chunk(const float2 (&y)[8], const PlainUnit<FMT>& u, bool scaled, float p,
                                            uint32_t (&w)[CodeWords<FMT>::n], float2& e2, float2& x2)
{
    using F = Fmt<FMT>;
    if constexpr (F::is_int) {
        if constexpr (EXACT) {
            float2 e[8];
            int_chunk_exact<FMT, STATS, GENERAL>(y, u.iq, F::qmin, F::qmax, w, e);
            if constexpr (STATS) {
                if (GENERAL && scaled) res_sums<true>(y, e, p, e2, x2);
                else res_sums<false>(y, e, p, e2, x2);
            }
        } else {
            float2 nq[8];
            int_chunk<FMT, STATS, GENERAL>(y, u.iq, F::qmin, F::qmax, w, nq);
            if constexpr (STATS) {
                if (GENERAL && scaled) int_sums<true>(y, nq, u.s, p, e2, x2);
                else int_sums<false>(y, nq, u.s, p, e2, x2);
            }
        }
    } else {
        float2 val[8];
        fp_chunk<FMT, STATS>(y, u.fq, w, val);
        if constexpr (STATS) {
            if (GENERAL && scaled) val_sums<true>(y, val, u.s, p, e2, x2);
            else val_sums<false>(y, val, u.s, p, e2, x2);
        }
    }
}

// Whether a plain unit needs the general chunk path (warp-uniform: clamping in some lane,
// or scaled sums).
template <int FMT>
__device__ __forceinline__ bool unit_general(const PlainUnit<FMT>& u, bool scaled)
{
    if constexpr (Fmt<FMT>::is_int) return __any_sync(0xFFFFFFFFu, scaled || u.iq.clamp);
    else return __any_sync(0xFFFFFFFFu, scaled);
}

// Call f(std::integral_constant<bool, EXACT>, std::integral_constant<bool, GENERAL>) with
// the runtime flags as compile-time constants (the integer formats only use EXACT).
template <int FMT, typename Fn>
__device__ __forceinline__ void with_chunk_flags(bool exact, bool general, Fn&& f)
{
    using T = std::true_type;
    using N = std::false_type;
    if constexpr (Fmt<FMT>::is_int) {
        if (exact) { if (general) f(T{}, T{}); else f(T{}, N{}); }
        else { if (general) f(N{}, T{}); else f(N{}, N{}); }
    } else {
        if (general) f(N{}, T{}); else f(N{}, N{});
    }
}

// ---------------------------------------------------------------------------
// Fast chunk paths, for units that need neither clamping (beyond the asymmetric cap at
// xc) nor scaled sums nor a divide. No branches, no votes, no calls: the hot loops stay
// small. They decide every element of a unit whose flags admit them; ce2 / cx2 are the
// chunk's plain sums. (The bool result, always false, is kept for the callers' shape.)
// ---------------------------------------------------------------------------

// Integer codes from the magic form t = MAGIC + zero point + bias + q.
template <int FMT>
__device__ __forceinline__ void pack_int(const float2 (&t)[8], uint32_t (&w)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) {
        uint32_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            h[k] = __float_as_uint(t[2 * k].x) + __float_as_uint(t[2 * k].y) * 16u +
                   __float_as_uint(t[2 * k + 1].x) * 256u + __float_as_uint(t[2 * k + 1].y) * 4096u;
        w[0] = __byte_perm(h[0], h[1], 0x5410);
        w[1] = __byte_perm(h[2], h[3], 0x5410);
        if constexpr (CodeBias<FMT>::v == 8) { w[0] ^= 0x88888888u; w[1] ^= 0x88888888u; }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = pack_bytes(__float_as_uint(t[2 * k].x), __float_as_uint(t[2 * k].y),
                              __float_as_uint(t[2 * k + 1].x), __float_as_uint(t[2 * k + 1].y));
    }
}

// The fast paths take the correctly rounded quotient RN(x / s) without a divide: with
// rn = RN(1/s), q0 = RN(x rn) is within an ulp of x / s, the remainder x - q0 s is
// exact (one FMA), and RN(q0 + rem rn) = RN(x / s) (Markstein's theorem on division
// with a correctly rounded reciprocal). It holds for every element a unit's mk flag
// admits: s in [2^-60, 2^100] and |x / s| < 2^20; a quotient below 2^-40 (where the
// remainder may underflow) can be off by a few of its ulps, but every format codes it
// as zero. (Checked against IEEE division for every bf16 x and every scale
// RN(amax / Q) of a bf16 amax, Q each format's Qmax, and on 10^9 random fp32 pairs.)

// Integer codes, any scale (unit flags fast, mk and no clamp): t = RN(q + 2^23 1.5)
// rounds the exact quotient half to even, then zero point and bias are added exactly.
// Decides every element.
template <int FMT, bool STATS>
__device__ __forceinline__ bool int_chunk_fast(const float2 (&y)[8], const IntQ& u, uint32_t (&w)[CodeWords<FMT>::n],
                                               float2& ce2, float2& cx2)
{
    using F = Fmt<FMT>;
    float2 t[8], nq[8];
    const float2 RN = splat(u.rn), S = splat(u.s), NS = splat(-u.s), M = splat(MAGIC), M1 = splat(-1.0f);
    const float2 ZB = splat(__fsub_rn(u.mz, MAGIC));           // zero point + bias (exact)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 yq = F::asym ? make_float2(fminf(y[i].x, u.xc), fminf(y[i].y, u.xc)) : y[i];
        const float2 q0 = mul2(yq, RN);
        const float2 q1 = fma2(fma2(q0, NS, yq), RN, q0);       // RN(x / s)
        const float2 t0 = add2(q1, M);                          // MAGIC + rne(q)
        nq[i] = fma2(t0, M1, M);                                // -q, exact
        t[i] = add2(t0, ZB);
    }
    pack_int<FMT>(t, w);
    if constexpr (STATS) {
        // two accumulators each: shorter dependency chains
        float2 ea = splat(0.0f), eb = splat(0.0f), xa = splat(0.0f), xb = splat(0.0f);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float2 d0 = fma2(nq[i], S, y[i]), d1 = fma2(nq[i + 1], S, y[i + 1]);
            ea = fma2(d0, d0, ea);
            eb = fma2(d1, d1, eb);
            xa = fma2(y[i], y[i], xa);
            xb = fma2(y[i + 1], y[i + 1], xb);
        }
        ce2 = add2(ea, eb);
        cx2 = add2(xa, xb);
    }
    return false;
}

// Integer codes, fp16 scale, unrotated bf16 input: the bracket select of
// int_chunk_exact (its unit must have br set). Decides every element.
template <int FMT, bool STATS>
__device__ __forceinline__ bool int_chunk_exact_fast(const float2 (&y)[8], const IntQ& u,
                                                     uint32_t (&w)[CodeWords<FMT>::n], float2& ce2, float2& cx2)
{
    float2 e[8];
    int_chunk_exact<FMT, STATS, false>(y, u, 0, 0, w, e);
    if constexpr (STATS) {
        float2 ea = splat(0.0f), eb = splat(0.0f), xa = splat(0.0f), xb = splat(0.0f);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            ea = fma2(e[i], e[i], ea);
            eb = fma2(e[i + 1], e[i + 1], eb);
            xa = fma2(y[i], y[i], xa);
            xb = fma2(y[i + 1], y[i + 1], xb);
        }
        ce2 = add2(ea, eb);
        cx2 = add2(xa, xb);
    }
    return false;
}

// FP codes (unit flag mk): cvt of the exact quotient. Decides every element.
template <int FMT, bool STATS>
__device__ __forceinline__ bool fp_chunk_fast(const float2 (&y)[8], const FpQ& u, uint32_t (&w)[CodeWords<FMT>::n],
                                              float2& ce2, float2& cx2)
{
    uint32_t pr[8];
    const float2 RN = splat(u.rn), NS = splat(-u.s), S = splat(u.s), NRN = splat(-u.rn);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        // RN(x / s) = RN(q0 - (q0 s - x) rn): the residual is taken negated so that a -0
        // input keeps its sign (-0 + -0); every nonzero result is the same either way
        const float2 q0 = mul2(y[p], RN);
        const float2 q1 = fma2(fma2(q0, S, neg2(y[p])), NRN, q0);
        pr[p] = cvt_pair<FMT>(q1.y, q1.x);
    }
    pack_pairs<FMT>(pr, w);
    if constexpr (STATS) {
        float2 val[8];
        decode_pairs<FMT>(pr, val);
        float2 ea = splat(0.0f), eb = splat(0.0f), xa = splat(0.0f), xb = splat(0.0f);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float2 d0 = fma2(val[i], NS, y[i]), d1 = fma2(val[i + 1], NS, y[i + 1]);
            ea = fma2(d0, d0, ea);
            eb = fma2(d1, d1, eb);
            xa = fma2(y[i], y[i], xa);
            xb = fma2(y[i + 1], y[i + 1], xb);
        }
        ce2 = add2(ea, eb);
        cx2 = add2(xa, xb);
    }
    return false;
}

template <int FMT, bool STATS, bool EXACT>
__device__ __forceinline__ bool plain_chunk_fast(const float2 (&y)[8], const PlainUnit<FMT>& u,
                                                 uint32_t (&w)[CodeWords<FMT>::n], float2& ce2, float2& cx2)
{
    if constexpr (!Fmt<FMT>::is_int) return fp_chunk_fast<FMT, STATS>(y, u.fq, w, ce2, cx2);
    else if constexpr (EXACT) return int_chunk_exact_fast<FMT, STATS>(y, u.iq, w, ce2, cx2);
    else return int_chunk_fast<FMT, STATS>(y, u.iq, w, ce2, cx2);
}

// Whether a plain unit must take the general path as a whole (warp-uniform: any lane
// with scaled sums, clamping, or a scale outside the fast paths' range).
template <int FMT, bool EXACT>
__device__ __forceinline__ bool unit_general_fast(const PlainUnit<FMT>& u, bool scaled)
{
    // every lane votes (scaled may differ between the lanes' units): the general chunk
    // path is itself warp-collective, so all lanes must take the same path
    if constexpr (Fmt<FMT>::is_int) {
        const bool g = u.iq.clamp || !u.iq.fast || (EXACT ? !u.iq.br : !u.iq.mk);
        return __any_sync(0xFFFFFFFFu, scaled || g);
    } else {
        return __any_sync(0xFFFFFFFFu, scaled || !u.fq.mk);
    }
}

// One chunk of an MX block (power-of-two scale 2^e: p2 = 2^-e, pe = 2^e); STATS adds
// its sums (scaled form when `scaled`).
template <int FMT, int GK, bool STATS>
__device__ __forceinline__ void mx_chunk(const float2 (&y)[8], float p2, float pe, bool scaled, float p,
                                         uint32_t (&q)[CodeWords<FMT>::n], float2& e2, float2& x2)
{
    using F = Fmt<FMT>;
    float2 z[8];
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
}

// One chunk of a plain unit: the fast path when the warp's units admit it, else the
// general one (sums added to e2 / x2).
template <int FMT>
__device__ __forceinline__ void rt_chunk(const float2 (&y)[8], const PlainUnit<FMT>& u, bool general, bool scaled,
                                         float p, uint32_t (&q)[CodeWords<FMT>::n], float2& e2, float2& x2)
{
    if (!general) {
        float2 ce2, cx2;
        (void)plain_chunk_fast<FMT, true, false>(y, u, q, ce2, cx2);
        e2 = add2(e2, ce2);
        x2 = add2(x2, cx2);
    } else {
        plain_chunk<FMT, true, false, true>(y, u, scaled, p, q, e2, x2);
    }
}

// Fold a unit's fp32 sums into the lane's doubles (inv_p2 = 1 / p^2).
__device__ __forceinline__ void add_unit_sums(Acc& acc, float2 e2, float2 x2, double inv_p2)
{
    acc.err2 += (double)__fadd_rn(e2.x, e2.y) * inv_p2;
    acc.x2 += (double)__fadd_rn(x2.x, x2.y) * inv_p2;
}

template <int FMT>
__device__ __forceinline__ void store_codes(uint8_t* codes, uint32_t c, const uint32_t (&w)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) st_v2(codes + (size_t)c * 8, w);
    else st_v4(codes + (size_t)c * 16, w);
}

__device__ __forceinline__ float pair_absmax(uint32_t m) { return fmaxf(bf_lo(m), bf_hi(m)); }
__device__ __forceinline__ float pair_min(uint32_t m) { return fminf(bf_lo(m), bf_hi(m)); }
__device__ __forceinline__ float pair_max(uint32_t m) { return fmaxf(bf_lo(m), bf_hi(m)); }

// Plain fp32 QSNR sums are safe (no overflow, no underflow that matters) for units whose
// largest magnitude lies in [2^-40, 2^40] (or is zero).
__device__ __forceinline__ bool plain_sums_ok(float amax) { return amax <= 0x1p40f && (amax >= 0x1p-40f || amax == 0.0f); }

}  // namespace bq
