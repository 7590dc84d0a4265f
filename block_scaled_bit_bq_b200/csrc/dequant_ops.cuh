// dequant_ops.cuh -- code decoding and scale application shared by the dequantize
// kernels: w = scale * (q - zero_point) ("INT4/INT8/FP8 quantization" §INT8), x = x_q *
// s_block * S_tensor ("Quantization survey" §4.3.2), and the FP element decode (-1)^s
// (1.m) 2^(e - bias) ("INT vs FP at fine granularity" §2.2).
#pragma once

#include "quant_ops.cuh"
#include "internal.h"

namespace bq {

// Codes of a lane's span of CPL consecutive chunks (CPL = 2 or 4), as 32-bit words.
template <int FMT, int CPL = 2>
struct SpanCodes {
    static constexpr int n = (Fmt<FMT>::four ? 2 : 4) * CPL;
};

template <int FMT, int CPL = 2>
__device__ __forceinline__ void load_codes(const uint8_t* codes, uint32_t span, uint32_t n_chunks,
                                           uint32_t (&w)[SpanCodes<FMT, CPL>::n])
{
    constexpr int CB = Fmt<FMT>::four ? 8 : 16;     // code bytes per chunk
    constexpr int NB = CB * CPL;                    // per span
    const uint32_t c0 = CPL * span;
    const uint8_t* p = codes + (size_t)span * NB;
    if (c0 + CPL <= n_chunks) {
        if constexpr (NB == 8) ld_nc_v2(p, *reinterpret_cast<uint32_t(*)[2]>(&w));
        else if constexpr (NB == 16) ld_nc_v4(p, *reinterpret_cast<uint32_t(*)[4]>(&w));
        else if constexpr (NB == 32) ld_nc_v8(p, *reinterpret_cast<uint32_t(*)[8]>(&w));
        else {
            ld_nc_v8(p, *reinterpret_cast<uint32_t(*)[8]>(&w));
            ld_nc_v8(p + 32, *reinterpret_cast<uint32_t(*)[8]>(&w[8]));
        }
    } else {
#pragma unroll
        for (int i = 0; i < SpanCodes<FMT, CPL>::n; ++i) w[i] = 0u;
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            if (c0 + k < n_chunks) {
                // one chunk's codes
                if constexpr (CB == 8) ld_nc_v2(p + k * CB, *reinterpret_cast<uint32_t(*)[2]>(&w[2 * k]));
                else ld_nc_v4(p + k * CB, *reinterpret_cast<uint32_t(*)[4]>(&w[4 * k]));
            }
        }
    }
}

// Element values of chunk h (0 or 1) of a span: FP codes decoded; integer codes as
// exact floats offset by MAGIC + bias (the caller subtracts MAGIC + bias + zero point in
// the same exact addition). An integer code's float is assembled by one byte permute:
// the (biased, non-negative) code byte becomes the low byte of MAGIC's bit pattern.
template <int FMT> struct DecodeBias { static constexpr int v = (FMT == BQ_INT8_SYM || FMT == BQ_INT8_ASYM) ? 128 : (FMT == BQ_INT4_SYM ? 8 : 0); };

template <int FMT, int CPL = 2>
__device__ __forceinline__ void chunk_values(const uint32_t (&w)[SpanCodes<FMT, CPL>::n], int h, float2 (&val)[8])
{
    using F = Fmt<FMT>;
    if constexpr (F::four) {
        const uint32_t w0 = w[2 * h], w1 = w[2 * h + 1];
        if constexpr (F::is_int) {
            constexpr uint32_t flip = DecodeBias<FMT>::v == 8 ? 0x08080808u : 0u;
            // byte k of lo* holds element 2k, byte k of hi* element 2k + 1
            const uint32_t lo0 = (w0 & 0x0F0F0F0Fu) ^ flip, hi0 = ((w0 >> 4) & 0x0F0F0F0Fu) ^ flip;
            const uint32_t lo1 = (w1 & 0x0F0F0F0Fu) ^ flip, hi1 = ((w1 >> 4) & 0x0F0F0F0Fu) ^ flip;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const uint32_t lo = p < 4 ? lo0 : lo1, hi = p < 4 ? hi0 : hi1;
                const uint32_t sel = 0x7650u | (uint32_t)(p & 3);
                val[p] = make_float2(__uint_as_float(__byte_perm(lo, MAGIC_BITS, sel)),
                                     __uint_as_float(__byte_perm(hi, MAGIC_BITS, sel)));
            }
        } else {
#pragma unroll
            for (int p = 0; p < 8; ++p) val[p] = dec_pair<FMT>(((p < 4 ? w0 : w1) >> (8 * (p & 3))) & 0xFFu);
        }
    } else {
        if constexpr (F::is_int) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t word = w[4 * h + k] ^ 0x80808080u;     // two's complement byte + 128
                val[2 * k] = make_float2(__uint_as_float(__byte_perm(word, MAGIC_BITS, 0x7650u)),
                                         __uint_as_float(__byte_perm(word, MAGIC_BITS, 0x7651u)));
                val[2 * k + 1] = make_float2(__uint_as_float(__byte_perm(word, MAGIC_BITS, 0x7652u)),
                                             __uint_as_float(__byte_perm(word, MAGIC_BITS, 0x7653u)));
            }
        } else {
#pragma unroll
            for (int p = 0; p < 8; ++p) val[p] = dec_pair<FMT>((w[4 * h + (p >> 1)] >> (16 * (p & 1))) & 0xFFFFu);
        }
    }
}

// The scale factors of chunk c's unit, as loaded (a, b): plain scales (s, zero point),
// MX (2^e, unused), NV (s_b, the tensor scale). Loaded ahead of the chunk's codes' use.
struct UnitScale {
    float a, b;
};

template <int FMT, int SK>
__device__ __forceinline__ UnitScale load_unit_scale(const DequantArgs& d, uint32_t c)
{
    uint32_t u = d.chunks_per_unit == 0 ? 0u : (uint32_t)(((uint64_t)__umulhi(c, d.fd_m) + c) >> d.fd_s);
    if constexpr (SK == SK_UE8M0 || SK == SK_NV) {
        if (d.gemm_layout) u = gemm_unit_offset(u, d.gemm_nb);
    }
    if constexpr (SK == SK_F32 || SK == SK_F16) {
        if (d.tile_cols) {
            // u is the chunk's row: tile (row / 128, column / 128), 8 chunks per tile column
            const uint32_t cc = c - u * d.chunks_per_unit;
            u = (u / TILE) * d.tile_cols + cc / (TILE / 16);
        }
    }
    UnitScale r{0.0f, 0.0f};
    if constexpr (SK == SK_UE8M0) {
        r.a = exp2i((int)__ldg(reinterpret_cast<const uint8_t*>(d.scales) + u) - 127);
    } else if constexpr (SK == SK_NV) {
        r.a = e4m3_value(__ldg(reinterpret_cast<const uint8_t*>(d.scales) + u));
        r.b = __ldg(d.tensor_scale);
    } else {
        if (d.scale_fp16) {
            r.a = __half2float(__ldg(reinterpret_cast<const __half*>(d.scales) + u));
            if constexpr (Fmt<FMT>::asym) r.b = __half2float(__ldg(reinterpret_cast<const __half*>(d.zps) + u));
        } else {
            r.a = __ldg(reinterpret_cast<const float*>(d.scales) + u);
            if constexpr (Fmt<FMT>::asym) r.b = __ldg(reinterpret_cast<const float*>(d.zps) + u);
        }
    }
    return r;
}

// Dequantized fp32 values of a chunk (before any inverse rotation) from its element
// values and its unit's scale factors.
template <int FMT, int SK>
__device__ __forceinline__ void dequant_chunk(const UnitScale& us, const float2 (&val)[8], float2 (&xh)[8])
{
    using F = Fmt<FMT>;
    constexpr float off = MAGIC + (float)DecodeBias<FMT>::v;     // integer codes arrive as off + q
    if constexpr (SK == SK_UE8M0) {
        const float2 pe = splat(us.a);
        if constexpr (F::is_int) {
            const float2 nz = splat(-off);
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = mul2(add2(val[i], nz), pe);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = mul2(val[i], pe);
        }
    } else if constexpr (SK == SK_NV) {
        const float2 sbv = splat(us.a), S = splat(us.b);
        if constexpr (F::is_int) {
            const float2 nz = splat(-off);
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = mul2(mul2(add2(val[i], nz), sbv), S);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = mul2(mul2(val[i], sbv), S);
        }
    } else {
        const float2 S = splat(us.a);
        if constexpr (F::is_int) {
            // (off + q) - (off + zp) = q - zp, exact
            const float2 nz = splat(-__fadd_rn(off, us.b));
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = mul2(add2(val[i], nz), S);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) xh[i] = mul2(val[i], S);
        }
    }
}

}  // namespace bq
