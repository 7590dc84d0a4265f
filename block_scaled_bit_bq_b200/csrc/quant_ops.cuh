// quant_ops.cuh -- quantize one 16-element chunk given its scale, on fp32 pairs.
//
// Code rules ("INT vs FP at fine granularity" §2.1, "INT4/INT8/FP8 quantization"
// §INT8/§INT4, "Quantization survey" §4.1):
//   INT:  q = clamp(rne(x / s) [+ zp], Qmin, Qmax)
//   FP:   code = cvt.rn.satfinite(x / s)
// with x / s the correctly rounded fp32 quotient, decided through the reciprocal
// bracket of common.cuh (a correctly rounded division only where the bracket is
// inconclusive, about one element in 10^4).
#pragma once

#include <cfloat>

#include "common.cuh"

namespace bq {

template <int FMT> struct CodeWords { static constexpr int n = Fmt<FMT>::four ? 2 : 4; };

// Everything a chunk needs to know about its unit's scale.
struct UnitQ {
    float s;        // scale the codes divide by (stored plain scale, d for NV)
    float rlo, rhi; // reciprocal bracket (both 0 for an INT unit with s == 0)
    float zpf;      // zero point (exact float; 0 for symmetric)
    int qmin, qmax; // integer code range
    bool fast;      // bracket usable for this unit
    bool clamp_lo;  // some element can fall below qmin
    bool clamp_hi;  // some element can rise above qmax
    bool zero;      // s == 0 (or d == 0): every code is the zero code
};

// Clamping flags. q is monotone in x, so the unit's extreme values bound it.
__device__ __forceinline__ void clamp_flags(float lo, float hi, const Recip& R, float zpf, int qmin, int qmax,
                                            bool& clo, bool& chi)
{
    if (!R.fast) { clo = chi = true; return; }
    const float top = __fadd_rn(__fmaf_rn(hi, R.rhi, MAGIC), zpf);   // >= MAGIC + q for every x <= hi
    const float bot = __fadd_rn(__fmaf_rn(lo, R.rhi, MAGIC), zpf);   // <= MAGIC + q for every x >= lo (lo <= 0)
    chi = top > MAGIC + (float)qmax;
    clo = bot < MAGIC + (float)qmin;
}

// Integer unit from a scale: a unit with s == 0 maps every element to the zero code
// through the fast path itself (r_lo = r_hi = 0 gives q = 0, plus the zero point).
__device__ __forceinline__ UnitQ int_unit(float s, float zpf, float lo, float hi, int qmin, int qmax)
{
    UnitQ u;
    u.s = s;
    u.zpf = zpf;
    u.qmin = qmin;
    u.qmax = qmax;
    u.zero = !(s > 0.0f);
    if (u.zero) {
        u.rlo = u.rhi = 0.0f;
        u.fast = true;
        u.clamp_lo = u.clamp_hi = false;
        return u;
    }
    const Recip R = make_recip(s, fmaxf(-lo, hi));
    u.rlo = R.rlo;
    u.rhi = R.rhi;
    u.fast = R.fast;
    clamp_flags(lo, hi, R, zpf, qmin, qmax, u.clamp_lo, u.clamp_hi);
    return u;
}

// Settle elements whose bracket ends disagree. The two candidates are adjacent
// integers; h is the half-integer between them. fma(-h, s, x) is the exactly rounded
// x - h s, which is zero only when x / s == h exactly: then RN(x/s) = h and the code is
// the even candidate (the magic sum's low bit is the integer's parity). Any other
// disagreement returns false and the caller divides.
__device__ __forceinline__ bool settle_ties(float y, float s, float rhi, float& t)
{
    const float a = t;
    const float b = __fmaf_rn(y, rhi, MAGIC);
    if (__float_as_uint(a) == __float_as_uint(b)) return true;
    const float qa = __fsub_rn(a, MAGIC), qb = __fsub_rn(b, MAGIC);   // exact
    const float h = __fmul_rn(0.5f, __fadd_rn(qa, qb));                // exact: an odd integer / 2
    if (__fmaf_rn(-h, s, y) != 0.0f) return false;
    t = (__float_as_uint(a) & 1u) == 0u ? a : b;
    return true;
}

// ---------------------------------------------------------------------------
// Integer chunk. On return: w = packed codes; qz[i] = q - zp (exact floats) when NEED_Q.
// ---------------------------------------------------------------------------

template <int FMT, bool NEED_Q>
__device__ __forceinline__ void int_chunk(const float2 (&y)[8], const UnitQ& u,
                                          uint32_t (&w)[CodeWords<FMT>::n], float2 (&qz)[8])
{
    using F = Fmt<FMT>;
    float2 t[8];
    bool ok = u.fast;
    if (ok) {
        uint32_t mism = 0;
        const float2 lo = splat(u.rlo), hi = splat(u.rhi), m = splat(MAGIC);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 a = fma2(y[i], lo, m);
            const float2 b = fma2(y[i], hi, m);
            mism |= (__float_as_uint(a.x) ^ __float_as_uint(b.x)) | (__float_as_uint(a.y) ^ __float_as_uint(b.y));
            t[i] = a;
        }
        if (mism) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ok &= settle_ties(y[i].x, u.s, u.rhi, t[i].x);
                ok &= settle_ties(y[i].y, u.s, u.rhi, t[i].y);
            }
        }
    }
    if (!ok) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float qa = rintf(__fdiv_rn(y[i].x, u.s));
            float qb = rintf(__fdiv_rn(y[i].y, u.s));
            qa = fminf(fmaxf(qa, -4194304.0f), 4194304.0f);
            qb = fminf(fmaxf(qb, -4194304.0f), 4194304.0f);
            t[i] = make_float2(__fadd_rn(qa, MAGIC), __fadd_rn(qb, MAGIC));
        }
    }
    if constexpr (F::asym) {
        const float2 z = splat(u.zpf);
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = add2(t[i], z);
    }
    if (u.clamp_hi || !ok) {
        const float cmax = MAGIC + (float)u.qmax;
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = make_float2(fminf(t[i].x, cmax), fminf(t[i].y, cmax));
    }
    if (u.clamp_lo || !ok) {
        const float cmin = MAGIC + (float)u.qmin;
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = make_float2(fmaxf(t[i].x, cmin), fmaxf(t[i].y, cmin));
    }
    if constexpr (NEED_Q) {
        const float2 z = splat(-__fadd_rn(MAGIC, u.zpf));
#pragma unroll
        for (int i = 0; i < 8; ++i) qz[i] = add2(t[i], z);
    }
    // the low bits of t are the two's complement code
    if constexpr (F::four) {
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = pack_nibbles(__float_as_uint(t[i].x), __float_as_uint(t[i].y));
        w[0] = pack_bytes(b[0], b[1], b[2], b[3]);
        w[1] = pack_bytes(b[4], b[5], b[6], b[7]);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = pack_bytes(__float_as_uint(t[2 * k].x), __float_as_uint(t[2 * k].y),
                              __float_as_uint(t[2 * k + 1].x), __float_as_uint(t[2 * k + 1].y));
    }
}

// ---------------------------------------------------------------------------
// FP element chunks.
// ---------------------------------------------------------------------------

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

// General scale s > 0: codes of x / s. val = decoded element values when NEED_V.
template <int FMT, bool NEED_V>
__device__ __forceinline__ void fp_chunk(const float2 (&y)[8], const UnitQ& u,
                                         uint32_t (&w)[CodeWords<FMT>::n], float2 (&val)[8])
{
    uint32_t pr[8];
    if (u.zero) {
#pragma unroll
        for (int p = 0; p < 8; ++p) pr[p] = 0u;
    } else {
        bool ok = u.fast;
        if (ok) {
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
            ok = (mism == 0);
        }
        if (!ok) {
#pragma unroll
            for (int p = 0; p < 8; ++p)
                pr[p] = cvt_pair<FMT>(__fdiv_rn(y[p].y, u.s), __fdiv_rn(y[p].x, u.s));
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

// MXINT8: q = clamp(rne(x * 2^-e), -127, 127); the clamp never binds (amax <= 127 * 2^e)
// except for the clamped exponent range, which the caller flags.
template <bool NEED_Q>
__device__ __forceinline__ void int8_chunk_pow2(const float2 (&y)[8], float p2, bool clamp, uint32_t (&w)[4],
                                                float2 (&q)[8])
{
    float2 t[8];
    const float2 p = splat(p2), m = splat(MAGIC);
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = fma2(y[i], p, m);
    if (clamp) {
        const float cmin = MAGIC - 127.0f, cmax = MAGIC + 127.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            t[i] = make_float2(fminf(fmaxf(t[i].x, cmin), cmax), fminf(fmaxf(t[i].y, cmin), cmax));
    }
    if constexpr (NEED_Q) {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = add2(t[i], splat(-MAGIC));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
        w[k] = pack_bytes(__float_as_uint(t[2 * k].x), __float_as_uint(t[2 * k].y),
                          __float_as_uint(t[2 * k + 1].x), __float_as_uint(t[2 * k + 1].y));
}

template <int FMT>
__device__ __forceinline__ void store_codes(uint8_t* codes, uint32_t c, const uint32_t (&w)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) st_v2(codes + (size_t)c * 8, w);
    else st_v4(codes + (size_t)c * 16, w);
}

// ---------------------------------------------------------------------------
// Plain (tensor / row / group) scales.
// ---------------------------------------------------------------------------

struct PlainScale {
    float s;        // stored scale (fp16-rounded when the dtype is fp16)
    float zpf;      // zero point as float (0 for symmetric)
    float lo, hi;   // extreme values the unit holds (-amax, amax for symmetric)
};

template <int FMT>
__device__ __forceinline__ PlainScale plain_scale(float amax, float mn, float mx, bool fp16)
{
    using F = Fmt<FMT>;
    PlainScale p;
    if constexpr (F::asym) {
        const float lo = fminf(mn, 0.0f), hi = fmaxf(mx, 0.0f);
        float s32 = __fdiv_rn(__fsub_rn(hi, lo), F::qscale);
        s32 = fminf(s32, FLT_MAX);                  // a range beyond fp32 saturates
        p.s = fp16 ? round_scale_f16(s32) : s32;
        if (p.s > 0.0f) {
            float z = rintf(__fdiv_rn(-lo, p.s));
            z = fminf(fmaxf(z, -1.0e9f), 1.0e9f);
            p.zpf = fminf(fmaxf(__fadd_rn((float)F::qmin, z), (float)F::qmin), (float)F::qmax);
        } else {
            p.zpf = (float)F::qmin;
        }
        p.lo = lo;
        p.hi = hi;
    } else {
        const float s32 = __fdiv_rn(amax, F::qscale);
        p.s = fp16 ? round_scale_f16(s32) : s32;
        p.zpf = 0.0f;
        p.lo = -amax;
        p.hi = amax;
    }
    return p;
}

template <int FMT>
__device__ __forceinline__ UnitQ unit_of_plain(const PlainScale& ps)
{
    using F = Fmt<FMT>;
    if constexpr (F::is_int) return int_unit(ps.s, ps.zpf, ps.lo, ps.hi, F::qmin, F::qmax);
    UnitQ u;
    u.s = ps.s;
    u.zpf = 0.0f;
    u.qmin = u.qmax = 0;
    u.zero = !(ps.s > 0.0f);
    const Recip R = make_recip(ps.s, fmaxf(-ps.lo, ps.hi));
    u.rlo = R.rlo;
    u.rhi = R.rhi;
    u.fast = R.fast;
    u.clamp_lo = u.clamp_hi = false;
    return u;
}

// Quantize a chunk under a unit; xh = dequantized value (rotated domain) when NEED_X.
template <int FMT, bool NEED_X>
__device__ __forceinline__ void quant_unit_chunk(const float2 (&y)[8], const UnitQ& u,
                                                 uint32_t (&w)[CodeWords<FMT>::n], float2 (&xh)[8])
{
    using F = Fmt<FMT>;
    if constexpr (F::is_int) {
        float2 qz[8];
        int_chunk<FMT, NEED_X>(y, u, w, qz);
        if constexpr (NEED_X) {
            const float2 s = splat(u.s);
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = mul2(qz[i], s);   // s == 0 gives 0: qz is 0 there
        }
    } else {
        float2 val[8];
        fp_chunk<FMT, NEED_X>(y, u, w, val);
        if constexpr (NEED_X) {
            const float2 s = splat(u.s);
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = u.zero ? splat(0.0f) : mul2(val[i], s);
        }
    }
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

// ---------------------------------------------------------------------------
// QSNR sums of one chunk on values scaled by a power of two p:
// e2 += sum ((y - xh) p)^2, x2 += sum (y p)^2 (pairs accumulate separately).
// ---------------------------------------------------------------------------

__device__ __forceinline__ void chunk_sums2(const float2 (&y)[8], const float2 (&xh)[8], float p,
                                            float2& e2, float2& x2)
{
    const float2 P = splat(p), nP = splat(-p);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 yp = mul2(y[i], P);
        const float2 d = fma2(xh[i], nP, yp);    // (y - xh) p: xh * p is exact
        e2 = fma2(d, d, e2);
        x2 = fma2(yp, yp, x2);
    }
}

// range of a chunk
__device__ __forceinline__ float chunk_amax(const float2 (&y)[8], float m)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) m = amax3(m, y[i].x, y[i].y);
    return m;
}

__device__ __forceinline__ void chunk_minmax(const float2 (&y)[8], float& mn, float& mx)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        mn = min3(mn, y[i].x, y[i].y);
        mx = max3(mx, y[i].x, y[i].y);
    }
}

}  // namespace bq
