// rot_quant.cu -- quantize after the randomized full-row Hadamard rotation (QuaRot,
// "Quantization survey" §5.3) and the optional per-column factor (SmoothQuant, same page
// §3.2 and §5.2), for rows of n = 1024, 2048 or 4096 columns: per-row, per-group and MX
// scales.
//
// A CTA of 64 threads owns 64 / T rows at a time (T = n / 64 threads per row) and a
// contiguous range of rows. Thread m of a row:
//   - loads the row's columns 64 m .. 64 m + 63 (bf16) with four 32-byte loads, flips the
//     signed columns' sign bits, widens, multiplies by the factors, and runs the rotation's
//     stages 1 .. 32 in registers (rot64.cuh, pass A); the next row's loads are issued
//     right after the widening, so they are in flight during the rest of this row;
//   - after a barrier, runs the stages along the matrix columns it owns (pass B), times the
//     normalisation;
//   - after a barrier, quantizes the row's values 64 m .. 64 m + 63 (four 16-element
//     pieces): an MX block or a group of 32 is two of its pieces, a group of 16 one, a group
//     of 64 .. 512 spans L / 4 adjacent threads (xor-shuffle reductions), a per-row unit the
//     row's T threads.
// The QSNR sums are taken on the rotated values (the rotation is orthogonal: both sums
// are kept).
// Six CTAs per SM (up to 170 registers a thread): the 64 values, the next row's prefetched
// words and the quantize phase fit without spilling, which measured faster than eight
// CTAs with spills or than dropping the prefetch.
#include "quant_ops.cuh"
#include "rot64.cuh"
#include "internal.h"

namespace bq {
namespace {

// Max (amax, max) and min over the T threads of a row: xor shuffles inside the warp, and
// (T = 64) the two warps' values through shared memory.
template <int MB>
__device__ __forceinline__ void row_range(float& amax, float& mn, float& mx, float4 (&red)[2])
{
    constexpr int T = 1 << MB;
    constexpr int W = T < 32 ? T : 32;
#pragma unroll
    for (int o = 1; o < W; o <<= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    }
    if constexpr (T == 64) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = make_float4(amax, mn, mx, 0.0f);
        __syncthreads();
        const float4 a = red[0], b = red[1];
        amax = fmaxf(a.x, b.x);
        mn = fminf(a.y, b.y);
        mx = fmaxf(a.z, b.z);
    }
}

// Sum over the T threads of a row, in a fixed order (the xor tree, then warp 0 + warp 1).
template <int MB>
__device__ __forceinline__ float row_sum(float s, float (&red)[2])
{
    constexpr int T = 1 << MB;
    constexpr int W = T < 32 ? T : 32;
#pragma unroll
    for (int o = 1; o < W; o <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xFFFFFFFFu, s, o));
    if constexpr (T == 64) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
        __syncthreads();
        s = __fadd_rn(red[0], red[1]);
    }
    return s;
}

template <int FMT, bool MX, int MB>
__global__ void __launch_bounds__(RT64_THREADS, 6) k_quant_rt64(const RtArgs a)
{
    pdl_wait();
    using F = Fmt<FMT>;
    constexpr int NW = CodeWords<FMT>::n;
    constexpr uint32_t T = 1u << MB, N = 64u * T, RS = 64u / T, CPR = N / 16u;
    extern __shared__ float4 rt64_smem[];
    __shared__ float4 red[2];
    __shared__ float red_ss[2];
    const uint32_t slot = threadIdx.x >> MB, tau = threadIdx.x & (T - 1u);
    float* const vbase = reinterpret_cast<float*>(rt64_smem);
    float* const v = vbase + slot * rt64_row_floats(N);
    uint32_t* const msk = reinterpret_cast<uint32_t*>(vbase + RS * rt64_row_floats(N));
    const bool f16 = a.scale_fp16 != 0;
    const uint32_t L = a.lanes;
    build_sign_masks64(msk, a.sign_bits, N);
    __syncthreads();

    // row groups (RS rows each) split evenly over the CTAs: [g0, g1) for this one
    const uint32_t groups = (a.rows + RS - 1u) / RS;
    const uint32_t g0 = (uint32_t)((uint64_t)blockIdx.x * groups / gridDim.x);
    const uint32_t g1 = (uint32_t)((uint64_t)(blockIdx.x + 1u) * groups / gridDim.x);
    const uint32_t iters = (groups + gridDim.x - 1u) / gridDim.x;
    auto row_of = [&](uint32_t it) { return (g0 + it) * RS + slot; };
    auto row_ok = [&](uint32_t it) { return g0 + it < g1 && row_of(it) < a.rows; };
    Acc acc;
    uint32_t w[32];
    auto load_words = [&](uint32_t r, bool ok) {
        if (ok) {
            const uint32_t* src = a.x + (size_t)r * (N / 2) + 32u * tau;
#pragma unroll
            for (int i = 0; i < 4; ++i) ld_nc_v8(src + 8 * i, *reinterpret_cast<uint32_t(*)[8]>(&w[8 * i]));
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = 0u;
        }
    };
    load_words(row_of(0), row_ok(0));

    for (uint32_t it = 0; it < iters; ++it) {
        const uint32_t r = row_of(it);
        const bool ok = row_ok(it);
        {
            float2 P[32];
            // the signs flip bf16 sign bits before the factor: the same values as flipping
            // the products' signs
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 m4 = *reinterpret_cast<const uint4*>(msk + mask64(tau, 4u * i));
                P[4 * i] = make_float2(__uint_as_float((w[4 * i] ^ m4.x) << 16), __uint_as_float((w[4 * i] ^ m4.x) & 0xFFFF0000u));
                P[4 * i + 1] = make_float2(__uint_as_float((w[4 * i + 1] ^ m4.y) << 16), __uint_as_float((w[4 * i + 1] ^ m4.y) & 0xFFFF0000u));
                P[4 * i + 2] = make_float2(__uint_as_float((w[4 * i + 2] ^ m4.z) << 16), __uint_as_float((w[4 * i + 2] ^ m4.z) & 0xFFFF0000u));
                P[4 * i + 3] = make_float2(__uint_as_float((w[4 * i + 3] ^ m4.w) << 16), __uint_as_float((w[4 * i + 3] ^ m4.w) & 0xFFFF0000u));
            }
            load_words(row_of(it + 1u), row_ok(it + 1u));
            if (a.col_scale) {
                const float4* cs = reinterpret_cast<const float4*>(a.col_scale) + 16u * tau;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float4 f = __ldg(cs + i);
                    P[2 * i] = mul2(P[2 * i], make_float2(f.x, f.y));
                    P[2 * i + 1] = mul2(P[2 * i + 1], make_float2(f.z, f.w));
                }
            }
            wht64_rows(P);
            store_row64(v, tau, P);
        }
        __syncthreads();
        wht64_columns<MB>(v, tau, a.norm);
        __syncthreads();

        const uint32_t cg0 = r * CPR + 4u * tau;        // the thread's first chunk
        if constexpr (MX) {
            // two MX blocks per thread
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                float2 y0[8], y1[8];
                uint32_t q0[NW], q1[NW];
                load_piece64(v, tau, 2 * b, y0);
                load_piece64(v, tau, 2 * b + 1, y1);
                const float amax = chunk_amax(y1, chunk_amax(y0, 0.0f));
                const bool scaled = !plain_sums_ok(amax);
                const Pow2 pw = pow2_for(amax);
                const float p = scaled ? pw.p : 1.0f;
                const int e = ue8m0_exponent<FMT>(amax);
                const float p2 = exp2i(-e), pe = exp2i(e);
                float2 e2 = splat(0.0f), x2 = splat(0.0f);
                mx_chunk<FMT, K_MX, true>(y0, p2, pe, scaled, p, q0, e2, x2);
                mx_chunk<FMT, K_MX, true>(y1, p2, pe, scaled, p, q1, e2, x2);
                if (ok) {
                    const uint32_t c = cg0 + 2u * b;
                    store_codes<FMT>(a.codes, c, q0);
                    store_codes<FMT>(a.codes, c + 1u, q1);
                    const uint32_t u = c >> 1;
                    reinterpret_cast<uint8_t*>(a.scales)[a.gemm_layout ? gemm_unit_offset(u, a.gemm_nb) : u] =
                        (uint8_t)(e + 127);
                    add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
                    kappa_add(acc, __fmul_rn(amax, p), __fadd_rn(x2.x, x2.y), a.inv_unit);
                }
            }
        } else if (L == 1u || L == 2u) {
            // groups of 16 or 32: 4 / L units per thread
            const uint32_t lgL = L >> 1;
#pragma unroll 1
            for (uint32_t b = 0; b < 4u; b += L) {
                float2 y0[8], y1[8];
                uint32_t q[NW];
                load_piece64(v, tau, (int)b, y0);
                if (L == 2u) load_piece64(v, tau, (int)b + 1, y1);
                float amax = 0.0f, mn = 0.0f, mx = 0.0f;
                if constexpr (F::asym) {
                    chunk_minmax(y0, mn, mx);
                    if (L == 2u) chunk_minmax(y1, mn, mx);
                    amax = fmaxf(-mn, mx);
                } else {
                    amax = chunk_amax(y0, 0.0f);
                    if (L == 2u) amax = chunk_amax(y1, amax);
                }
                const bool scaled = !plain_sums_ok(amax);
                const Pow2 pw = pow2_for(amax);
                const float p = scaled ? pw.p : 1.0f;
                const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
                const PlainUnit<FMT> u = plain_unit<FMT>(ps);
                const bool general = unit_general_fast<FMT, false>(u, scaled);
                float2 e2 = splat(0.0f), x2 = splat(0.0f);
                const uint32_t c = cg0 + b;
                rt_chunk<FMT>(y0, u, general, scaled, p, q, e2, x2);
                if (ok) store_codes<FMT>(a.codes, c, q);
                if (L == 2u) {
                    rt_chunk<FMT>(y1, u, general, scaled, p, q, e2, x2);
                    if (ok) store_codes<FMT>(a.codes, c + 1u, q);
                }
                if (ok) {
                    store_plain_scale<FMT>(a.scales, a.zps, c >> lgL, ps, f16);
                    add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
                    kappa_add(acc, __fmul_rn(amax, p), __fadd_rn(x2.x, x2.y), a.inv_unit);
                }
            }
        } else {
            // a group of 64 .. 512 (L / 4 adjacent threads) or the whole row (L = 0)
            float amax = 0.0f, mn = 0.0f, mx = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 y[8];
                load_piece64(v, tau, k, y);
                if constexpr (F::asym) chunk_minmax(y, mn, mx);
                else amax = chunk_amax(y, amax);
            }
            const uint32_t tpu = L >> 2;                  // threads per unit (0: the row)
            if (L == 0u) {
                row_range<MB>(amax, mn, mx, red);
            } else {
                for (uint32_t o = 1; o < tpu; o <<= 1) {
                    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                    mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
                    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                }
            }
            if constexpr (F::asym) amax = fmaxf(-mn, mx);
            const bool scaled = !plain_sums_ok(amax);
            const Pow2 pw = pow2_for(amax);
            const float p = scaled ? pw.p : 1.0f;
            const PlainScale ps = plain_scale<FMT>(amax, mn, mx, f16);
            const PlainUnit<FMT> u = plain_unit<FMT>(ps);
            const bool general = unit_general_fast<FMT, false>(u, scaled);
            float2 e2 = splat(0.0f), x2 = splat(0.0f);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 y[8];
                uint32_t q[NW];
                load_piece64(v, tau, k, y);
                rt_chunk<FMT>(y, u, general, scaled, p, q, e2, x2);
                if (ok) store_codes<FMT>(a.codes, cg0 + (uint32_t)k, q);
            }
            if (ok) add_unit_sums(acc, e2, x2, scaled ? pw.inv_p2 : 1.0);
            float ss = __fadd_rn(x2.x, x2.y);
            bool first;
            uint32_t unit;
            if (L == 0u) {
                ss = row_sum<MB>(ss, red_ss);
                first = tau == 0u;
                unit = r;
            } else {
                for (uint32_t o = 1; o < tpu; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
                first = (tau & (tpu - 1u)) == 0u;
                unit = cg0 / L;
            }
            if (ok && first) {
                store_plain_scale<FMT>(a.scales, a.zps, unit, ps, f16);
                kappa_add(acc, __fmul_rn(amax, p), ss, a.inv_unit);
            }
        }
        __syncthreads();             // the rows are read; the next rows may overwrite them
    }
    if (a.stats) finish_stats(acc, a.ws, a.stats, false, 0.0f, 0.0, true);
}

template <int FMT, bool MX, int MB>
cudaError_t run_rt64(const RtArgs& a, cudaStream_t st)
{
    constexpr auto kern = k_quant_rt64<FMT, MX, MB>;
    constexpr uint32_t RS = 64u >> MB;
    const size_t smem = rt64_smem_bytes(64u << MB);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, RT64_THREADS, smem) != cudaSuccess || occ < 1) occ = 1;
    uint64_t slots = (uint64_t)device_sm_count() * (uint64_t)occ;
    if (slots > (uint64_t)MAX_GRID) slots = MAX_GRID;
    // every CTA slot busy, the row groups split evenly over them
    const uint64_t groups = ((uint64_t)a.rows + RS - 1) / RS;
    const uint64_t grid = groups < slots ? groups : slots;
    return launch_pdl(kern, (unsigned)grid, (unsigned)RT64_THREADS, smem, st, a);
}

template <int FMT, bool MX>
cudaError_t run_rt64_n(const RtArgs& a, cudaStream_t st)
{
    switch (a.cols) {
    case 1024: return run_rt64<FMT, MX, 4>(a, st);
    case 2048: return run_rt64<FMT, MX, 5>(a, st);
    case 4096: return run_rt64<FMT, MX, 6>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_quant_rt64(int fmt, bool mx, const RtArgs& a, cudaStream_t st)
{
    if (!a.sign_bits || !rt64_cols(a.cols) || a.rows == 0) return cudaErrorInvalidValue;
    if (mx) {
        switch (fmt) {
        case BQ_INT8_SYM: return run_rt64_n<BQ_INT8_SYM, true>(a, st);
        case BQ_FP8_E4M3: return run_rt64_n<BQ_FP8_E4M3, true>(a, st);
        case BQ_FP8_E5M2: return run_rt64_n<BQ_FP8_E5M2, true>(a, st);
        case BQ_FP4_E2M1: return run_rt64_n<BQ_FP4_E2M1, true>(a, st);
        case BQ_FP6_E2M3: return run_rt64_n<BQ_FP6_E2M3, true>(a, st);
        case BQ_FP6_E3M2: return run_rt64_n<BQ_FP6_E3M2, true>(a, st);
        default: return cudaErrorInvalidValue;
        }
    }
    switch (fmt) {
    case BQ_INT8_SYM:   return run_rt64_n<BQ_INT8_SYM, false>(a, st);
    case BQ_INT8_ASYM:  return run_rt64_n<BQ_INT8_ASYM, false>(a, st);
    case BQ_INT4_SYM:   return run_rt64_n<BQ_INT4_SYM, false>(a, st);
    case BQ_UINT4_ASYM: return run_rt64_n<BQ_UINT4_ASYM, false>(a, st);
    case BQ_FP8_E4M3:   return run_rt64_n<BQ_FP8_E4M3, false>(a, st);
    case BQ_FP8_E5M2:   return run_rt64_n<BQ_FP8_E5M2, false>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace bq
