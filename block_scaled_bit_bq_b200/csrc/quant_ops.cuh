// quant_ops.cuh -- quantize one 16-element chunk given its scale.
//
// Code rules ("INT vs FP at fine granularity" §2.1, "INT4/INT8/FP8 quantization"
// §INT8/§INT4, "Quantization survey" §4.1):
//   INT:  q = clamp(rne(x / s) [+ zp], Qmin, Qmax)
//   FP:   code = cvt.rn.satfinite(x / s)
// with x / s the correctly rounded fp32 quotient, decided through the reciprocal
// bracket of common.cuh (a correctly rounded division only where the bracket is
// inconclusive).
#pragma once

#include "common.cuh"

namespace bq {

template <int FMT> struct CodeWords { static constexpr int n = Fmt<FMT>::four ? 2 : 4; };

// Integer chunk. zpf = zero point as an exact float (0 for symmetric formats);
// qmin / qmax the code range. On return: w holds the packed codes, qz[i] = q - zp.
template <int FMT, bool NEED_Q>
__device__ __forceinline__ void quant_int_chunk(const float (&y)[16], const Recip& R, float zpf,
                                                int qmin, int qmax,
                                                uint32_t (&w)[CodeWords<FMT>::n], float (&qz)[16])
{
    using F = Fmt<FMT>;
    float t[16];
    bool ok = R.fast;
    if (ok) {
        uint32_t mism = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = __fmaf_rn(y[i], R.rlo, MAGIC);
            const float b = __fmaf_rn(y[i], R.rhi, MAGIC);
            mism |= __float_as_uint(a) ^ __float_as_uint(b);
            t[i] = a;
        }
        ok = (mism == 0);
    }
    if (!ok) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float q = rintf(__fdiv_rn(y[i], R.s));
            q = fminf(fmaxf(q, -4194304.0f), 4194304.0f);
            t[i] = __fadd_rn(q, MAGIC);
        }
    }
    const float cmin = MAGIC + (float)qmin, cmax = MAGIC + (float)qmax;
    const float zero_at = __fadd_rn(MAGIC, zpf);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float u = t[i];
        if constexpr (F::asym) u = __fadd_rn(u, zpf);
        u = fminf(fmaxf(u, cmin), cmax);
        t[i] = u;
        if constexpr (NEED_Q) qz[i] = __fsub_rn(u, zero_at);
    }
    if constexpr (F::four) {
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = pack_nibbles(__float_as_uint(t[2 * i]), __float_as_uint(t[2 * i + 1]));
        w[0] = pack_bytes(b[0], b[1], b[2], b[3]);
        w[1] = pack_bytes(b[4], b[5], b[6], b[7]);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = pack_bytes(__float_as_uint(t[4 * k]), __float_as_uint(t[4 * k + 1]),
                              __float_as_uint(t[4 * k + 2]), __float_as_uint(t[4 * k + 3]));
    }
}

// Pack eight pair-codes (cvt_pair results, element 2p in the low part) into words.
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
__device__ __forceinline__ void decode_pairs(const uint32_t (&pr)[8], float (&val)[16])
{
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const float2 f = dec_pair<FMT>(pr[p]);
        val[2 * p] = f.x;
        val[2 * p + 1] = f.y;
    }
}

// FP element chunk (E4M3 / E5M2 / E2M1) with a general scale s > 0. On return w holds
// the packed codes and (NEED_V) val[i] the decoded element values.
template <int FMT, bool NEED_V>
__device__ __forceinline__ void quant_fp_chunk(const float (&y)[16], const Recip& R,
                                               uint32_t (&w)[CodeWords<FMT>::n], float (&val)[16])
{
    uint32_t pr[8];
    bool ok = R.fast;
    if (ok) {
        uint32_t mism = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const uint32_t lo = cvt_pair<FMT>(__fmul_rn(y[2 * p + 1], R.rlo), __fmul_rn(y[2 * p], R.rlo));
            const uint32_t hi = cvt_pair<FMT>(__fmul_rn(y[2 * p + 1], R.rhi), __fmul_rn(y[2 * p], R.rhi));
            mism |= lo ^ hi;
            pr[p] = lo;
        }
        ok = (mism == 0);
    }
    if (!ok) {
#pragma unroll
        for (int p = 0; p < 8; ++p)
            pr[p] = cvt_pair<FMT>(__fdiv_rn(y[2 * p + 1], R.s), __fdiv_rn(y[2 * p], R.s));
    }
    pack_pairs<FMT>(pr, w);
    if constexpr (NEED_V) decode_pairs<FMT>(pr, val);
}

// FP element chunk with an exact power-of-two scale: code = cvt(x * 2^-e).
template <int FMT, bool NEED_V>
__device__ __forceinline__ void quant_fp_chunk_pow2(const float (&y)[16], float p2,
                                                    uint32_t (&w)[CodeWords<FMT>::n], float (&val)[16])
{
    uint32_t pr[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) pr[p] = cvt_pair<FMT>(__fmul_rn(y[2 * p + 1], p2), __fmul_rn(y[2 * p], p2));
    pack_pairs<FMT>(pr, w);
    if constexpr (NEED_V) decode_pairs<FMT>(pr, val);
}

// MXINT8 chunk with an exact power-of-two scale: q = clamp(rne(x * 2^-e), -127, 127).
__device__ __forceinline__ void quant_int8_chunk_pow2(const float (&y)[16], float p2, uint32_t (&w)[4],
                                                      float (&q)[16])
{
    const float cmin = MAGIC - 127.0f, cmax = MAGIC + 127.0f;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float u = fminf(fmaxf(__fmaf_rn(y[i], p2, MAGIC), cmin), cmax);
        t[i] = u;
        q[i] = __fsub_rn(u, MAGIC);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
        w[k] = pack_bytes(__float_as_uint(t[4 * k]), __float_as_uint(t[4 * k + 1]),
                          __float_as_uint(t[4 * k + 2]), __float_as_uint(t[4 * k + 3]));
}

// Store one chunk's codes (chunk c of the flat code array).
template <int FMT>
__device__ __forceinline__ void store_codes(uint8_t* codes, uint32_t c, const uint32_t (&w)[CodeWords<FMT>::n])
{
    if constexpr (Fmt<FMT>::four) st_v2(codes + (size_t)c * 8, w);
    else st_v4(codes + (size_t)c * 16, w);
}

// Scale of a plain (tensor / row / group) unit from its range.
struct PlainScale {
    float s;        // stored scale (fp16-rounded when the dtype is fp16)
    float zpf;      // zero point as float (0 for symmetric)
    float bound;    // max |y| the unit can hold (for the integer magic range)
};

template <int FMT>
__device__ __forceinline__ PlainScale plain_scale(float amax, float mn, float mx, bool fp16)
{
    using F = Fmt<FMT>;
    PlainScale p;
    if constexpr (F::asym) {
        const float lo = fminf(mn, 0.0f), hi = fmaxf(mx, 0.0f);
        const float s32 = __fdiv_rn(__fsub_rn(hi, lo), F::qscale);
        p.s = fp16 ? round_scale_f16(s32) : s32;
        if (p.s > 0.0f) {
            float z = __fadd_rn((float)F::qmin, rintf(__fdiv_rn(-lo, p.s)));
            p.zpf = fminf(fmaxf(z, (float)F::qmin), (float)F::qmax);
        } else {
            p.zpf = (float)F::qmin;
        }
        p.bound = fmaxf(-lo, hi);
    } else {
        const float s32 = __fdiv_rn(amax, F::qscale);
        p.s = fp16 ? round_scale_f16(s32) : s32;
        p.zpf = 0.0f;
        p.bound = amax;
    }
    return p;
}

// Quantize a chunk under a plain scale; returns codes and, when NEED_X, the dequantized
// value of each element in xh (rotated domain). A unit with s == 0 gets code "zero"
// (q = zp for INT, +0 for FP) and xhat = 0.
template <int FMT, bool NEED_X>
__device__ __forceinline__ void quant_plain_chunk(const float (&y)[16], const PlainScale& ps, const Recip& R,
                                                  int qmin, int qmax,
                                                  uint32_t (&w)[CodeWords<FMT>::n], float (&xh)[16])
{
    using F = Fmt<FMT>;
    if (!(ps.s > 0.0f)) {
        if constexpr (F::is_int) {
            const uint32_t z = ((uint32_t)(int)ps.zpf) & (F::four ? 0xFu : 0xFFu);
            const uint32_t b = F::four ? (z | (z << 4)) : z;
            const uint32_t word = b * 0x01010101u;
#pragma unroll
            for (int k = 0; k < CodeWords<FMT>::n; ++k) w[k] = word;
        } else {
#pragma unroll
            for (int k = 0; k < CodeWords<FMT>::n; ++k) w[k] = 0u;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) xh[i] = 0.0f;
        return;
    }
    if constexpr (F::is_int) {
        float qz[16];
        quant_int_chunk<FMT, NEED_X>(y, R, ps.zpf, qmin, qmax, w, qz);
        if constexpr (NEED_X) {
#pragma unroll
            for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(qz[i], ps.s);
        }
    } else {
        float val[16];
        quant_fp_chunk<FMT, NEED_X>(y, R, w, val);
        if constexpr (NEED_X) {
#pragma unroll
            for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(val[i], ps.s);
        }
    }
}

// Store a plain scale (and zero point) at index i.
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

// Sums for QSNR over one chunk: err2 = sum (y - yhat)^2, x2 = sum y^2.
__device__ __forceinline__ void chunk_sums(const float (&y)[16], const float (&xh)[16], float& e2, float& x2)
{
    float e = 0.0f, s = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float d = __fsub_rn(y[i], xh[i]);
        e = __fmaf_rn(d, d, e);
        s = __fmaf_rn(y[i], y[i], s);
    }
    e2 = e;
    x2 = s;
}

}  // namespace bq
