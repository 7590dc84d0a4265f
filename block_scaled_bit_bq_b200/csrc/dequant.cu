// dequant.cu -- dequantize and standalone QSNR kernels.
//
// Steps (source pages): w = scale * (q - zero_point) ("INT4/INT8/FP8 quantization"
// §INT8), q * scale (same page §INT4), x = x_q * s_block * S_tensor ("Quantization
// survey" §4.3.2), the FP element decode (-1)^s (1.m) 2^(e - bias) ("INT vs FP at fine
// granularity" §2.2), the inverse Hadamard rotation (H16/4 is its own inverse), and
// QSNR = -10 log10(||X - Xq||^2 / ||X||^2) (same page §4.1).
//
// Work layout as in the quantize kernels: a warp takes 64 consecutive 16-element
// chunks per step, two per lane, codes read with one vector load per chunk, the
// chunk's scale found by a multiply-high division of the chunk index.
#include "common.cuh"
#include "internal.h"

#include <atomic>

namespace bq {

// Dequantized fp32 values of chunk c (before any inverse rotation).
template <int FMT, int SK>
__device__ __forceinline__ void dequant_chunk(const DequantArgs& a, uint32_t c, float (&xh)[16])
{
    using F = Fmt<FMT>;
    const uint32_t u = a.chunks_per_unit == 0 ? 0u : (uint32_t)(((uint64_t)__umulhi(c, a.fd_m) + c) >> a.fd_s);

    // element values (integers as exact floats, FP codes decoded)
    float val[16];
    if constexpr (F::four) {
        uint32_t w[2];
        ld_nc_v2(a.codes + (size_t)c * 8, w);
        if constexpr (F::is_int) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t nib = (w[i >> 3] >> (4 * (i & 7))) & 0xFu;
                int q = (int)nib;
                if constexpr (FMT != BQ_UINT4_ASYM) q = (q ^ 8) - 8;   // sign-extend
                val[i] = (float)q;
            }
        } else {
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const float2 f = dec_pair<FMT>((w[p >> 2] >> (8 * (p & 3))) & 0xFFu);
                val[2 * p] = f.x;
                val[2 * p + 1] = f.y;
            }
        }
    } else {
        uint32_t w[4];
        ld_nc_v4(a.codes + (size_t)c * 16, w);
        if constexpr (F::is_int) {
#pragma unroll
            for (int i = 0; i < 16; ++i) val[i] = (float)(int)(int8_t)(w[i >> 2] >> (8 * (i & 3)));
        } else {
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const float2 f = dec_pair<FMT>((w[p >> 1] >> (16 * (p & 1))) & 0xFFFFu);
                val[2 * p] = f.x;
                val[2 * p + 1] = f.y;
            }
        }
    }

    if constexpr (SK == SK_UE8M0) {
        const int e = (int)reinterpret_cast<const uint8_t*>(a.scales)[u] - 127;
        const float pe = exp2i(e);
#pragma unroll
        for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(val[i], pe);
    } else if constexpr (SK == SK_NV) {
        const float sbv = e4m3_value(reinterpret_cast<const uint8_t*>(a.scales)[u]);
        const float S = a.tensor_scale[0];
#pragma unroll
        for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(__fmul_rn(val[i], sbv), S);
    } else {
        float s, zp = 0.0f;
        if (a.scale_fp16) {
            s = __half2float(reinterpret_cast<const __half*>(a.scales)[u]);
            if constexpr (F::asym) zp = __half2float(reinterpret_cast<const __half*>(a.zps)[u]);
        } else {
            s = reinterpret_cast<const float*>(a.scales)[u];
            if constexpr (F::asym) zp = reinterpret_cast<const float*>(a.zps)[u];
        }
        if constexpr (F::asym) {
#pragma unroll
            for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(s, __fsub_rn(val[i], zp));
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) xh[i] = __fmul_rn(val[i], s);
        }
    }
}

template <int FMT, int SK, bool HAD, int OUT>
__global__ void __launch_bounds__(256) k_dequant(const DequantArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t t = warp; t < a.n_dtiles; t += nwarps) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t c = t * 64 + lane + 32 * h;
            if (c >= a.n_chunks) continue;
            float xh[16];
            dequant_chunk<FMT, SK>(a, c, xh);
            if constexpr (HAD) fwht16(xh);
            if constexpr (OUT == BQ_DT_BF16) {
                uint32_t o[8];
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const __nv_bfloat162 b = __floats2bfloat162_rn(xh[2 * p], xh[2 * p + 1]);
                    o[p] = *reinterpret_cast<const uint32_t*>(&b);
                }
                st_v8(reinterpret_cast<uint8_t*>(a.out) + (size_t)c * 32, o);
            } else {
                uint32_t o0[8], o1[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) { o0[i] = __float_as_uint(xh[i]); o1[i] = __float_as_uint(xh[8 + i]); }
                uint8_t* p = reinterpret_cast<uint8_t*>(a.out) + (size_t)c * 64;
                st_v8(p, o0);
                st_v8(p + 32, o1);
            }
        }
    }
}

template <int FMT, int SK, bool HAD>
__global__ void __launch_bounds__(256) k_qsnr(const DequantArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    Acc acc;
    for (uint32_t t = warp; t < a.n_dtiles; t += nwarps) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t c = t * 64 + lane + 32 * h;
            if (c >= a.n_chunks) continue;
            float x[16];
            load16(a.x, c, x);
            float xh[16];
            dequant_chunk<FMT, SK>(a, c, xh);
            if constexpr (HAD) fwht16(xh);
            float e = 0.0f, s = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float d = __fsub_rn(x[i], xh[i]);
                e = __fmaf_rn(d, d, e);
                s = __fmaf_rn(x[i], x[i], s);
            }
            acc.err2 += (double)e;
            acc.x2 += (double)s;
        }
    }
    finish_stats(acc, a.ws, a.stats, false, 0.0f, 0.0, false);
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
cudaError_t run_dq(bool had, int out, const DequantArgs& a, cudaStream_t st)
{
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

}  // namespace

cudaError_t launch_dequant(int fmt, int sk, bool had, int out_dtype, const DequantArgs& a, cudaStream_t st)
{
    return dispatch(fmt, sk, [&]<int FMT, int SK>() { return run_dq<FMT, SK>(had, out_dtype, a, st); });
}

cudaError_t launch_qsnr(int fmt, int sk, bool had, const DequantArgs& a, cudaStream_t st)
{
    return dispatch(fmt, sk, [&]<int FMT, int SK>() { return run_qs<FMT, SK>(had, a, st); });
}

}  // namespace bq
