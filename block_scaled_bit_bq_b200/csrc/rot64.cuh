// rot64.cuh -- the full-row Walsh-Hadamard transform (QuaRot's randomized rotation,
// "Quantization survey" §5.3) of rows of n = 64 T values, T = 16, 32 or 64 threads per row.
//
// The row is seen as a T x 64 matrix: element (m, p) is the value at position 64 m + p.
// Stages h = 1 .. 32 act along p, stages h = 64 .. n / 2 along m. Two passes:
//   pass A: thread m holds row m of the matrix (64 consecutive values, as 32 pairs of
//           neighbours) and runs stages 1 .. 32 in registers: stage 1 inside each pair,
//           stages 2 .. 32 on whole pairs (packed f32x2 adds);
//   pass B: thread p holds column(s) p of the matrix from shared memory and runs the
//           stages along m in registers, then multiplies by the normalisation.
// Each output of each stage is a + b or a - b of the same two values as in the
// sequential stage order h = 1, 2, ..., n / 2, so the result is the one of that order.
//
// Shared-memory layout (one row): element (m, p) at
//     64 m + 4 ((p >> 2) ^ (m & 7)) + (p & 3),
// the 16-byte granules of matrix row m permuted by m & 7. Row-wise 16-byte accesses by
// consecutive threads (pass A stores, the quantize phase's reads) and
// column-wise 4-byte accesses (pass B) both touch 32 distinct banks per 32 accesses.
// Rows of one CTA sit n + 16 floats apart (the 16-float shift keeps two rows read by
// one warp, T = 16, on different banks). A pass-B thread reads and writes back the same
// addresses, so no barrier separates its reads from its writes.
#pragma once

#include "common.cuh"

namespace bq {

// Threads per CTA of the two-pass row kernel: 64 / T rows at a time.
constexpr int RT64_THREADS = 64;

__host__ __device__ constexpr uint32_t rt64_row_floats(uint32_t n) { return n + 16u; }

// Dynamic shared memory of a CTA: its rows, then the sign masks (n / 2 words).
__host__ __device__ constexpr uint32_t rt64_smem_bytes(uint32_t n)
{
    return (RT64_THREADS / (n / 64u)) * rt64_row_floats(n) * 4u + n / 2u * 4u;
}

// Whether a row length takes the two-pass kernel.
__host__ __device__ constexpr bool rt64_cols(uint32_t n) { return n == 1024u || n == 2048u || n == 4096u; }

__device__ __forceinline__ uint32_t la64(uint32_t m, uint32_t p)
{
    return 64u * m + 4u * ((p >> 2) ^ (m & 7u)) + (p & 3u);
}

// Pass A on a thread's 64 consecutive values, P[i] = (value 2i, value 2i + 1).
__device__ __forceinline__ void wht64_rows(float2 (&P)[32])
{
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float a = P[i].x, b = P[i].y;
        P[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {          // stage 2h on pairs h apart
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((i & h) == 0) {
                const float2 a = P[i], b = P[i + h];
                P[i] = add2(a, b);
                P[i + h] = sub2(a, b);
            }
        }
    }
}

// Matrix row m (the thread's 64 values) into shared memory.
__device__ __forceinline__ void store_row64(float* v, uint32_t m, const float2 (&P)[32])
{
#pragma unroll
    for (int g = 0; g < 16; ++g)
        *reinterpret_cast<float4*>(v + la64(m, 4u * g)) = make_float4(P[2 * g].x, P[2 * g].y, P[2 * g + 1].x, P[2 * g + 1].y);
}

// Piece k (values 16 k .. 16 k + 15) of matrix row m.
__device__ __forceinline__ void load_piece64(const float* v, uint32_t m, int k, float2 (&y)[8])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 q = *reinterpret_cast<const float4*>(v + la64(m, 16u * k + 4u * j));
        y[2 * j] = make_float2(q.x, q.y);
        y[2 * j + 1] = make_float2(q.z, q.w);
    }
}

// Pass B: the stages along m (h = 64 .. n / 2) of the columns owned by thread p (p,
// p + T, ..., 64 / T of them), then * norm, written back in place. T = 2^MB.
template <int MB>
__device__ __forceinline__ void wht64_columns(float* v, uint32_t p, float norm)
{
    constexpr int T = 1 << MB;
    const float2 NR = splat(norm);
    if constexpr (MB == 6) {
        // one column of 64: pairs (m, m + 32); stages along m bits 0..4 on pairs, bit 5
        // inside each pair
        uint32_t off[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) off[k] = 4u * ((p >> 2) ^ (uint32_t)k) + (p & 3u);
        float2 Q[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) Q[i] = make_float2(v[64 * i + off[i & 7]], v[64 * (i + 32) + off[i & 7]]);
#pragma unroll
        for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if ((i & h) == 0) {
                    const float2 a = Q[i], b = Q[i + h];
                    Q[i] = add2(a, b);
                    Q[i + h] = sub2(a, b);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float a = Q[i].x, b = Q[i].y;
            Q[i] = mul2(make_float2(__fadd_rn(a, b), __fsub_rn(a, b)), NR);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[64 * i + off[i & 7]] = Q[i].x;
            v[64 * (i + 32) + off[i & 7]] = Q[i].y;
        }
    } else {
        // 64 / T columns of T: pairs (column c, column c + 32 / T); every stage on pairs
        constexpr int NC = 64 / T, H = NC / 2;
        float2 Q[H][T];
#pragma unroll
        for (int c = 0; c < H; ++c)
#pragma unroll
            for (int m = 0; m < T; ++m)
                Q[c][m] = make_float2(v[la64(m, p + T * c)], v[la64(m, p + T * (c + H))]);
#pragma unroll
        for (int h = 1; h < T; h <<= 1) {
#pragma unroll
            for (int c = 0; c < H; ++c) {
#pragma unroll
                for (int m = 0; m < T; ++m) {
                    if ((m & h) == 0) {
                        const float2 a = Q[c][m], b = Q[c][m + h];
                        Q[c][m] = add2(a, b);
                        Q[c][m + h] = sub2(a, b);
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < H; ++c)
#pragma unroll
            for (int m = 0; m < T; ++m) {
                const float2 q = mul2(Q[c][m], NR);
                v[la64(m, p + T * c)] = q.x;
                v[la64(m, p + T * (c + H))] = q.y;
            }
    }
}

// The random signs as XOR masks of bf16 pairs (bit 15: the even column, bit 31: the odd
// one), one word per two columns. Thread m's 32 words (columns 64 m .. 64 m + 63) sit at
// 32 m + 4 ((j >> 2) ^ (m & 7)) + (j & 3), so its 16-byte loads by consecutive threads
// touch distinct banks.
__device__ __forceinline__ uint32_t mask64(uint32_t m, uint32_t j)
{
    return 32u * m + 4u * ((j >> 2) ^ (m & 7u)) + (j & 3u);
}

__device__ __forceinline__ void build_sign_masks64(uint32_t* msk, const uint32_t* sign_bits, uint32_t n)
{
    for (uint32_t j = threadIdx.x; j < n / 2; j += blockDim.x) {
        const uint32_t b = (__ldg(sign_bits + (j >> 4)) >> ((2u * j) & 31u)) & 3u;
        msk[mask64(j >> 5, j & 31u)] = ((b & 1u) << 15) | ((b & 2u) << 30);
    }
}

}  // namespace bq
