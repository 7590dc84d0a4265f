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
#include "dequant_ops.cuh"
#include "rot.cuh"
#include "internal.h"

#include <atomic>

namespace bq {

// Dequantize: lane l of a warp owns a span of DQ_CPL consecutive chunks of the warp's
// tile; the next tile's codes and unit scales are loaded before the current tile is
// decoded. (Two chunks per lane measured faster than four.) A 2-D tile's scale is found
// from the chunk's row and column.
constexpr int DQ_CPL = 2;

template <int FMT, int SK, bool HAD, int OUT>
__global__ void __launch_bounds__(256) k_dequant(const DequantArgs a)
{
    pdl_wait();
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
    pdl_wait();
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
    pdl_wait();
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
    return launch_pdl(KERN, (unsigned)grid, (unsigned)block, 0, st, a);
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
    return launch_pdl(KERN, (unsigned)grid, (unsigned)block, smem, st, a, sign_bits, rows, cols, norm);
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
