// rot_dequant.cu -- dequantize with the inverse of the full-row randomized Hadamard
// rotation (QuaRot, "Quantization survey" §5.3: the rotation is orthogonal, R^T R = I,
// and H_n is symmetric, so the inverse is the same stages, the normalisation, then the
// signs), for rows of 1024, 2048 or 4096 columns.
//
// The same two-pass transform as the quantize side (rot64.cuh): thread m of a row decodes
// the row's values 64 m .. 64 m + 63 (four 16-element chunks, their codes in one or two
// 32-byte loads, the next row's codes and scales loaded right after), scales them, runs
// stages 1 .. 32 in registers; after a barrier, the stages along the matrix columns and
// the normalisation; after a barrier, it reads its 64 values back, rounds them to the
// output type, flips the signed columns' sign bits and stores them.
#include "dequant_ops.cuh"
#include "rot64.cuh"
#include "internal.h"

namespace bq {
namespace {

template <int FMT, int SK, int OUT, int MB>
__global__ void __launch_bounds__(RT64_THREADS, 8) k_dequant_rt64(const DequantArgs a, const uint32_t* sign_bits,
                                                                  uint32_t rows, float norm)
{
    constexpr int NC = SpanCodes<FMT, 4>::n;
    constexpr uint32_t T = 1u << MB, N = 64u * T, RS = 64u / T, CPR = N / 16u;
    extern __shared__ float4 rt64_smem[];
    const uint32_t slot = threadIdx.x >> MB, tau = threadIdx.x & (T - 1u);
    float* const vbase = reinterpret_cast<float*>(rt64_smem);
    float* const v = vbase + slot * rt64_row_floats(N);
    uint32_t* const msk = reinterpret_cast<uint32_t*>(vbase + RS * rt64_row_floats(N));
    build_sign_masks64(msk, sign_bits, N);
    __syncthreads();

    // row groups (RS rows each) split evenly over the CTAs: [g0, g1) for this one
    const uint32_t groups = (rows + RS - 1u) / RS;
    const uint32_t g0 = (uint32_t)((uint64_t)blockIdx.x * groups / gridDim.x);
    const uint32_t g1 = (uint32_t)((uint64_t)(blockIdx.x + 1u) * groups / gridDim.x);
    const uint32_t iters = (groups + gridDim.x - 1u) / gridDim.x;
    auto row_of = [&](uint32_t it) { return (g0 + it) * RS + slot; };
    auto row_ok = [&](uint32_t it) { return g0 + it < g1 && row_of(it) < rows; };
    uint32_t cw[NC];
    UnitScale us[4];
    auto load = [&](uint32_t r, bool ok) {
        if (ok) {
            const uint32_t span = r * T + tau;         // chunks 4 span .. 4 span + 3
            load_codes<FMT, 4>(a.codes, span, a.n_chunks, cw);
#pragma unroll
            for (int k = 0; k < 4; ++k) us[k] = load_unit_scale<FMT, SK>(a, 4u * span + (uint32_t)k);
        } else {
#pragma unroll
            for (int i = 0; i < NC; ++i) cw[i] = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) us[k] = UnitScale{0.0f, 0.0f};
        }
    };
    load(row_of(0), row_ok(0));

    for (uint32_t it = 0; it < iters; ++it) {
        const uint32_t r = row_of(it);
        const bool ok = row_ok(it);
        {
            float2 P[32];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 val[8], xh[8];
                chunk_values<FMT, 4>(cw, k, val);
                dequant_chunk<FMT, SK>(us[k], val, xh);
#pragma unroll
                for (int j = 0; j < 8; ++j) P[8 * k + j] = xh[j];
            }
            load(row_of(it + 1u), row_ok(it + 1u));
            wht64_rows(P);
            store_row64(v, tau, P);
        }
        __syncthreads();
        wht64_columns<MB>(v, tau, norm);
        __syncthreads();
        if (ok) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 xh[8];
                uint32_t m[8];
                load_piece64(v, tau, k, xh);
                piece_masks64(msk, tau, k, m);
                const size_t cg = (size_t)r * CPR + 4u * tau + (uint32_t)k;
                // the signs last: a flip of the sign bit (rounding to bf16 is odd-symmetric,
                // so flipping after the rounding gives the same bits as before it)
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
        }
        __syncthreads();             // the rows are read; the next rows may overwrite them
    }
}

template <int FMT, int SK, int OUT, int MB>
cudaError_t run_dq_rt64(const DequantArgs& a, const uint32_t* sign_bits, uint32_t rows, float norm, cudaStream_t st)
{
    constexpr auto kern = k_dequant_rt64<FMT, SK, OUT, MB>;
    constexpr uint32_t RS = 64u >> MB;
    const size_t smem = rt64_smem_bytes(64u << MB);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, RT64_THREADS, smem) != cudaSuccess || occ < 1) occ = 1;
    uint64_t slots = (uint64_t)device_sm_count() * (uint64_t)occ;
    if (slots > (uint64_t)MAX_GRID) slots = MAX_GRID;
    // every CTA slot busy, the row groups split evenly over them
    const uint64_t groups = ((uint64_t)rows + RS - 1) / RS;
    const uint64_t grid = groups < slots ? groups : slots;
    kern<<<(unsigned)grid, RT64_THREADS, smem, st>>>(a, sign_bits, rows, norm);
    return cudaGetLastError();
}

template <int FMT, int SK>
cudaError_t run_dq_rt64_n(int out_dtype, const DequantArgs& a, const uint32_t* sign_bits, uint32_t rows,
                          uint32_t cols, float norm, cudaStream_t st)
{
    const bool bf = out_dtype == BQ_DT_BF16;
    switch (cols) {
    case 1024: return bf ? run_dq_rt64<FMT, SK, BQ_DT_BF16, 4>(a, sign_bits, rows, norm, st)
                         : run_dq_rt64<FMT, SK, BQ_DT_FP32, 4>(a, sign_bits, rows, norm, st);
    case 2048: return bf ? run_dq_rt64<FMT, SK, BQ_DT_BF16, 5>(a, sign_bits, rows, norm, st)
                         : run_dq_rt64<FMT, SK, BQ_DT_FP32, 5>(a, sign_bits, rows, norm, st);
    case 4096: return bf ? run_dq_rt64<FMT, SK, BQ_DT_BF16, 6>(a, sign_bits, rows, norm, st)
                         : run_dq_rt64<FMT, SK, BQ_DT_FP32, 6>(a, sign_bits, rows, norm, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_dequant_rt64(int fmt, int sk, int out_dtype, const DequantArgs& a, const uint32_t* sign_bits,
                                uint32_t rows, uint32_t cols, float norm, cudaStream_t st)
{
    if (!sign_bits || !rt64_cols(cols) || rows == 0) return cudaErrorInvalidValue;
    if (sk == SK_UE8M0) {
        switch (fmt) {
        case BQ_INT8_SYM: return run_dq_rt64_n<BQ_INT8_SYM, SK_UE8M0>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_FP8_E4M3: return run_dq_rt64_n<BQ_FP8_E4M3, SK_UE8M0>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_FP8_E5M2: return run_dq_rt64_n<BQ_FP8_E5M2, SK_UE8M0>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_FP4_E2M1: return run_dq_rt64_n<BQ_FP4_E2M1, SK_UE8M0>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_FP6_E2M3: return run_dq_rt64_n<BQ_FP6_E2M3, SK_UE8M0>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_FP6_E3M2: return run_dq_rt64_n<BQ_FP6_E3M2, SK_UE8M0>(out_dtype, a, sign_bits, rows, cols, norm, st);
        default: return cudaErrorInvalidValue;
        }
    }
    if (sk == SK_F32 || sk == SK_F16) {            // fp16 scales: a runtime flag of the loads
        switch (fmt) {
        case BQ_INT8_SYM:   return run_dq_rt64_n<BQ_INT8_SYM, SK_F32>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_INT8_ASYM:  return run_dq_rt64_n<BQ_INT8_ASYM, SK_F32>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_INT4_SYM:   return run_dq_rt64_n<BQ_INT4_SYM, SK_F32>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_UINT4_ASYM: return run_dq_rt64_n<BQ_UINT4_ASYM, SK_F32>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_FP8_E4M3:   return run_dq_rt64_n<BQ_FP8_E4M3, SK_F32>(out_dtype, a, sign_bits, rows, cols, norm, st);
        case BQ_FP8_E5M2:   return run_dq_rt64_n<BQ_FP8_E5M2, SK_F32>(out_dtype, a, sign_bits, rows, cols, norm, st);
        default: return cudaErrorInvalidValue;
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace bq
