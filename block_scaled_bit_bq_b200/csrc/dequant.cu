// dequant.cu -- dequantize and standalone QSNR kernels.
//
// Steps (source pages): w = scale * (q - zero_point) ("INT4/INT8/FP8 quantization"
// §INT8), q * scale (same page §INT4), x = x_q * s_block * S_tensor ("Quantization
// survey" §4.3.2), the FP element decode (-1)^s (1.m) 2^(e - bias) ("INT vs FP at fine
// granularity" §2.2), the inverse Hadamard rotation (H16/4 is its own inverse), and
// QSNR = -10 log10(||X - Xq||^2 / ||X||^2) (same page §4.1).
//
// Work layout as in the quantize kernels: lane l of a warp owns two consecutive
// 16-element chunks of the warp's 1024-element tile, reads their codes with one
// vector load (32 bytes for 8-bit codes, 16 for 4-bit), and loads the next tile's
// codes before decoding the current ones. A chunk's scale index is its chunk index
// divided (multiply-high) by the chunks per scaling unit.
#include "quant_ops.cuh"
#include "rot.cuh"
#include "internal.h"

#include <atomic>

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

// Dequantize: lane l of a warp owns a span of DQ_CPL consecutive chunks of the warp's
// tile; the next tile's codes and unit scales are loaded before the current tile is
// decoded. (Two chunks per lane measured faster than four.) A 2-D tile's scale is found
// from the chunk's row and column.
constexpr int DQ_CPL = 2;

template <int FMT, int SK, bool HAD, int OUT>
__global__ void __launch_bounds__(256) k_dequant(const DequantArgs a)
{
    constexpr int NC = SpanCodes<FMT, DQ_CPL>::n;
    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t ntiles = (a.n_chunks + 32u * DQ_CPL - 1u) / (32u * DQ_CPL);
    // a chunk index past the end reads the last unit's scale (in bounds, unused)
    auto clampc = [&](uint32_t c) { return c < a.n_chunks ? c : a.n_chunks - 1; };
    uint32_t t = warp;
    uint32_t cur[NC];
    UnitScale cs[DQ_CPL];
    if (t < ntiles) {
        load_codes<FMT, DQ_CPL>(a.codes, t * 32 + lane, a.n_chunks, cur);
#pragma unroll
        for (int h = 0; h < DQ_CPL; ++h) cs[h] = load_unit_scale<FMT, SK>(a, clampc(DQ_CPL * (t * 32 + lane) + h));
    }
    while (t < ntiles) {
        const uint32_t tn = t + nwarps;
        uint32_t nxt[NC];
        UnitScale ns[DQ_CPL];
        if (tn < ntiles) {
            load_codes<FMT, DQ_CPL>(a.codes, tn * 32 + lane, a.n_chunks, nxt);
#pragma unroll
            for (int h = 0; h < DQ_CPL; ++h) ns[h] = load_unit_scale<FMT, SK>(a, clampc(DQ_CPL * (tn * 32 + lane) + h));
        } else {
#pragma unroll
            for (int h = 0; h < DQ_CPL; ++h) ns[h] = UnitScale{0.0f, 0.0f};
        }
        const uint32_t span = t * 32 + lane;
#pragma unroll
        for (int h = 0; h < DQ_CPL; ++h) {
            const uint32_t c = DQ_CPL * span + h;
            if (c >= a.n_chunks) break;
            float2 val[8], xh[8];
            chunk_values<FMT, DQ_CPL>(cur, h, val);
            dequant_chunk<FMT, SK>(cs[h], val, xh);
            if constexpr (HAD) fwht16x2(xh);
            if constexpr (OUT == BQ_DT_BF16) {
                uint32_t o[8];
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const __nv_bfloat162 b = __floats2bfloat162_rn(xh[p].x, xh[p].y);
                    o[p] = *reinterpret_cast<const uint32_t*>(&b);
                }
                st_v8(reinterpret_cast<uint8_t*>(a.out) + (size_t)c * 32, o);
            } else {
                uint32_t o0[8], o1[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o0[2 * i] = __float_as_uint(xh[i].x); o0[2 * i + 1] = __float_as_uint(xh[i].y);
                    o1[2 * i] = __float_as_uint(xh[4 + i].x); o1[2 * i + 1] = __float_as_uint(xh[4 + i].y);
                }
                uint8_t* p = reinterpret_cast<uint8_t*>(a.out) + (size_t)c * 64;
                st_v8(p, o0);
                st_v8(p + 32, o1);
            }
        }
#pragma unroll
        for (int i = 0; i < NC; ++i) cur[i] = nxt[i];
#pragma unroll
        for (int h = 0; h < DQ_CPL; ++h) cs[h] = ns[h];
        t = tn;
    }
}

template <int FMT, int SK, bool HAD>
__global__ void __launch_bounds__(256) k_qsnr(const DequantArgs a)
{
    constexpr int NC = SpanCodes<FMT>::n;
    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    Acc acc;
    for (uint32_t t = warp; t < a.n_dtiles; t += nwarps) {
        const uint32_t span = t * 32 + lane;
        uint32_t w[NC];
        load_codes<FMT>(a.codes, span, a.n_chunks, w);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t c = 2 * span + h;
            if (c >= a.n_chunks) break;
            uint32_t xw[8];
            ld_nc_v8(a.x + (size_t)c * 8, xw);
            float2 x[8], val[8], xh[8];
            widen16x2(xw, x);
            chunk_values<FMT>(w, h, val);
            dequant_chunk<FMT, SK>(load_unit_scale<FMT, SK>(a, c), val, xh);
            if constexpr (HAD) fwht16x2(xh);
            // sums on values scaled by a power of two fitted to the chunk (no overflow
            // or underflow in fp32), brought back in double
            const Pow2 pw = pow2_for(chunk_amax(x, chunk_amax(xh, 0.0f)));
            float2 e2 = splat(0.0f), x2 = splat(0.0f);
            const float2 P = splat(pw.p);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 d = mul2(sub2(x[i], xh[i]), P);
                const float2 xp = mul2(x[i], P);
                e2 = fma2(d, d, e2);
                x2 = fma2(xp, xp, x2);
            }
            acc.err2 += (double)__fadd_rn(e2.x, e2.y) * pw.inv_p2;
            acc.x2 += (double)__fadd_rn(x2.x, x2.y) * pw.inv_p2;
        }
    }
    finish_stats(acc, a.ws, a.stats, false, 0.0f, 0.0, false);
}

// Dequantize with the inverse full-row rotation: a CTA per row at a time. Each chunk
// is decoded, scaled and run through the first four Walsh-Hadamard stages in
// registers; the row sits in shared memory (fp32) for the remaining stages; then each
// value is multiplied by the normalisation, the signed columns negated and the result
// written. The per-column factor is not undone (the codes stand for x times it).
template <int FMT, int SK, int OUT>
__global__ void __launch_bounds__(RT_THREADS, 8) k_dequant_rt(const DequantArgs a, const uint32_t* sign_bits, uint32_t rows,
                                                    uint32_t cols, float norm)
{
    constexpr int NC = SpanCodes<FMT, 1>::n;
    extern __shared__ float4 rt_smem[];
    float* v = reinterpret_cast<float*>(rt_smem);
    const uint32_t cpr = cols / 16;
    uint32_t* smask = reinterpret_cast<uint32_t*>(v + rot_row_floats(cols));
    build_sign_masks(smask, sign_bits, cols);
    __syncthreads();
    for (uint32_t r = blockIdx.x; r < rows; r += gridDim.x) {
        for (uint32_t c = threadIdx.x; c < cpr; c += blockDim.x) {
            const uint32_t cg = r * cpr + c;
            uint32_t w[NC];
            float2 val[8], xh[8];
            load_codes<FMT, 1>(a.codes, cg, a.n_chunks, w);
            chunk_values<FMT, 1>(w, 0, val);
            dequant_chunk<FMT, SK>(load_unit_scale<FMT, SK>(a, cg), val, xh);
            wht16x2(xh);
            store_chunk_f32(v, c, xh);
        }
        wht_smem_stages(v, cols);
        for (uint32_t c = threadIdx.x; c < cpr; c += blockDim.x) {
            float2 xh[8];
            load_chunk_f32(v, c, norm, xh);
            const size_t cg = (size_t)r * cpr + c;
            // the signs last: a flip of the sign bit (rounding to bf16 is odd-symmetric, so
            // flipping after the rounding gives the same bits as before it)
            uint32_t m[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            flip_words(smask, c, m);
            if constexpr (OUT == BQ_DT_BF16) {
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const __nv_bfloat162 b = __floats2bfloat162_rn(xh[i].x, xh[i].y);
                    o[i] = *reinterpret_cast<const uint32_t*>(&b) ^ m[i];
                }
                st_v8(reinterpret_cast<uint8_t*>(a.out) + cg * 32, o);
            } else {
                uint32_t o0[8], o1[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o0[2 * i] = __float_as_uint(xh[i].x) ^ (m[i] << 16);
                    o0[2 * i + 1] = __float_as_uint(xh[i].y) ^ (m[i] & 0x80000000u);
                    o1[2 * i] = __float_as_uint(xh[4 + i].x) ^ (m[4 + i] << 16);
                    o1[2 * i + 1] = __float_as_uint(xh[4 + i].y) ^ (m[4 + i] & 0x80000000u);
                }
                uint8_t* p = reinterpret_cast<uint8_t*>(a.out) + cg * 64;
                st_v8(p, o0);
                st_v8(p + 32, o1);
            }
        }
        __syncthreads();             // the row is written out; the next row may overwrite it
    }
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

template <auto KERN>
cudaError_t launch_flat_kernel(const DequantArgs& a, cudaStream_t st)
{
    constexpr int block = 256;
    const uint64_t waves = (uint64_t)device_sm_count() * (uint64_t)resident_ctas<KERN, block>();
    uint64_t need = (a.n_dtiles + 7) / 8;
    if (need < 1) need = 1;
    uint64_t grid = need < waves ? need : waves;
    if (grid > (uint64_t)MAX_GRID) grid = MAX_GRID;
    KERN<<<(unsigned)grid, block, 0, st>>>(a);
    return cudaGetLastError();
}

template <int FMT, int SK>
cudaError_t run_dq(bool had, int out, const DequantArgs& a0, cudaStream_t st)
{
    DequantArgs a = a0;                 // the dequantize tile is 32 lanes x DQ_CPL chunks
    a.n_dtiles = (a0.n_chunks + 32u * DQ_CPL - 1u) / (32u * DQ_CPL);
    if (had) {
        return out == BQ_DT_BF16 ? launch_flat_kernel<k_dequant<FMT, SK, true, BQ_DT_BF16>>(a, st)
                                 : launch_flat_kernel<k_dequant<FMT, SK, true, BQ_DT_FP32>>(a, st);
    }
    return out == BQ_DT_BF16 ? launch_flat_kernel<k_dequant<FMT, SK, false, BQ_DT_BF16>>(a, st)
                             : launch_flat_kernel<k_dequant<FMT, SK, false, BQ_DT_FP32>>(a, st);
}

template <int FMT, int SK>
cudaError_t run_qs(bool had, const DequantArgs& a, cudaStream_t st)
{
    return had ? launch_flat_kernel<k_qsnr<FMT, SK, true>>(a, st)
               : launch_flat_kernel<k_qsnr<FMT, SK, false>>(a, st);
}

// Dispatch over (format, scale kind) pairs the library offers. Plain fp32 and fp16
// scales share one instantiation (the dtype is a runtime flag).
template <typename Fn>
cudaError_t dispatch(int fmt, int sk, Fn&& fn)
{
    if (sk == SK_F32 || sk == SK_F16) {
        switch (fmt) {
        case BQ_INT8_SYM:   return fn.template operator()<BQ_INT8_SYM, SK_F32>();
        case BQ_INT8_ASYM:  return fn.template operator()<BQ_INT8_ASYM, SK_F32>();
        case BQ_INT4_SYM:   return fn.template operator()<BQ_INT4_SYM, SK_F32>();
        case BQ_UINT4_ASYM: return fn.template operator()<BQ_UINT4_ASYM, SK_F32>();
        case BQ_FP8_E4M3:   return fn.template operator()<BQ_FP8_E4M3, SK_F32>();
        case BQ_FP8_E5M2:   return fn.template operator()<BQ_FP8_E5M2, SK_F32>();
        default: return cudaErrorInvalidValue;
        }
    }
    if (sk == SK_UE8M0) {
        switch (fmt) {
        case BQ_INT8_SYM: return fn.template operator()<BQ_INT8_SYM, SK_UE8M0>();
        case BQ_FP8_E4M3: return fn.template operator()<BQ_FP8_E4M3, SK_UE8M0>();
        case BQ_FP8_E5M2: return fn.template operator()<BQ_FP8_E5M2, SK_UE8M0>();
        case BQ_FP4_E2M1: return fn.template operator()<BQ_FP4_E2M1, SK_UE8M0>();
        case BQ_FP6_E2M3: return fn.template operator()<BQ_FP6_E2M3, SK_UE8M0>();
        case BQ_FP6_E3M2: return fn.template operator()<BQ_FP6_E3M2, SK_UE8M0>();
        default: return cudaErrorInvalidValue;
        }
    }
    if (sk == SK_NV) {
        switch (fmt) {
        case BQ_FP4_E2M1: return fn.template operator()<BQ_FP4_E2M1, SK_NV>();
        case BQ_INT4_SYM: return fn.template operator()<BQ_INT4_SYM, SK_NV>();
        default: return cudaErrorInvalidValue;
        }
    }
    return cudaErrorInvalidValue;
}

template <auto KERN>
cudaError_t launch_row_kernel(const DequantArgs& a, const uint32_t* sign_bits, uint32_t rows, uint32_t cols,
                              float norm, cudaStream_t st)
{
    const int block = cols / 16 < (uint32_t)RT_THREADS ? (int)(cols / 16) : RT_THREADS;   // a thread per chunk, up to RT_THREADS
    const size_t smem = rot_smem_bytes(cols, true);
    if (smem > 48u * 1024u) {
        const cudaError_t e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, KERN, block, smem) != cudaSuccess || occ < 1) occ = 1;
    uint64_t grid = (uint64_t)device_sm_count() * (uint64_t)occ;
    if (grid > rows) grid = rows;
    if (grid > (uint64_t)MAX_GRID) grid = MAX_GRID;
    if (grid < 1) grid = 1;
    KERN<<<(unsigned)grid, block, smem, st>>>(a, sign_bits, rows, cols, norm);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequant(int fmt, int sk, bool had, int out_dtype, const DequantArgs& a, cudaStream_t st)
{
    return dispatch(fmt, sk, [&]<int FMT, int SK>() { return run_dq<FMT, SK>(had, out_dtype, a, st); });
}

cudaError_t launch_dequant_rt(int fmt, int sk, int out_dtype, const DequantArgs& a, const uint32_t* sign_bits,
                              uint32_t rows, uint32_t cols, float norm, cudaStream_t st)
{
    return dispatch(fmt, sk, [&]<int FMT, int SK>() {
        return out_dtype == BQ_DT_BF16
                   ? launch_row_kernel<k_dequant_rt<FMT, SK, BQ_DT_BF16>>(a, sign_bits, rows, cols, norm, st)
                   : launch_row_kernel<k_dequant_rt<FMT, SK, BQ_DT_FP32>>(a, sign_bits, rows, cols, norm, st);
    });
}

cudaError_t launch_qsnr(int fmt, int sk, bool had, const DequantArgs& a, cudaStream_t st)
{
    return dispatch(fmt, sk, [&]<int FMT, int SK>() { return run_qs<FMT, SK>(had, a, st); });
}

}  // namespace bq
