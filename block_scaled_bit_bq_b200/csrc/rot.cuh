// rot.cuh -- Walsh-Hadamard stages over a row held in shared memory, for the full-row
// randomized rotation (QuaRot, "Quantization survey" §5.3).
//
// The row's n = 2^m fp32 values sit in shared memory after each thread has run the
// first four stages (h = 1, 2, 4, 8) on its own 16-element chunks in registers
// (wht16x2). The remaining stages h = 16, 32, ..., n/2 run in passes of up to four:
// a pass with stride S takes groups of R values S apart (R = 16, fewer in the last
// pass) and runs stages S, 2S, ..., S R / 2 on each group in registers. Every output
// is a + b or a - b of the same two values as in the sequential stage order, so the
// result does not depend on how the threads split the work.
#pragma once

#include "common.cuh"

namespace bq {

template <int R>
__device__ __forceinline__ void wht_pass(float* v, uint32_t n, uint32_t S)
{
    const uint32_t ngroups = n / R;
    for (uint32_t g = threadIdx.x; g < ngroups; g += blockDim.x) {
        const uint32_t base = (g % S) + (g / S) * S * R;
        float t[R];
#pragma unroll
        for (int k = 0; k < R; ++k) t[k] = v[base + S * k];
#pragma unroll
        for (int h = 1; h < R; h <<= 1) {
#pragma unroll
            for (int i = 0; i < R; i += 2 * h) {
#pragma unroll
                for (int j = i; j < i + h; ++j) {
                    const float a = t[j], b = t[j + h];
                    t[j] = __fadd_rn(a, b);
                    t[j + h] = __fsub_rn(a, b);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < R; ++k) v[base + S * k] = t[k];
    }
}

// Stages h = 16 .. n / 2 of v[0, n) (16 <= n <= 65536, a power of two). Called by every
// thread of the block; synchronizes before each pass and at the end.
__device__ __forceinline__ void wht_smem_stages(float* v, uint32_t n)
{
    for (uint32_t S = 16; S < n; S *= 16) {
        const uint32_t R = n / S;
        __syncthreads();
        if (R >= 16) wht_pass<16>(v, n, S);
        else if (R == 8) wht_pass<8>(v, n, S);
        else if (R == 4) wht_pass<4>(v, n, S);
        else wht_pass<2>(v, n, S);
    }
    __syncthreads();
}

// Negate element i of a chunk where bit i of the chunk's 16 sign bits is set.
__device__ __forceinline__ void apply_signs(float2 (&y)[8], uint32_t bits)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        y[i].x = __uint_as_float(__float_as_uint(y[i].x) ^ (((bits >> (2 * i)) & 1u) << 31));
        y[i].y = __uint_as_float(__float_as_uint(y[i].y) ^ (((bits >> (2 * i + 1)) & 1u) << 31));
    }
}

// The 16 sign bits of chunk c (columns 16c .. 16c + 15).
__device__ __forceinline__ uint32_t chunk_sign_bits(const uint32_t* sign_bits, uint32_t c)
{
    return (__ldg(sign_bits + (c >> 1)) >> (16u * (c & 1u))) & 0xFFFFu;
}

__device__ __forceinline__ void store_chunk_f32(float* v, uint32_t c, const float2 (&y)[8])
{
    float4* p = reinterpret_cast<float4*>(v + 16 * c);
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = make_float4(y[2 * i].x, y[2 * i].y, y[2 * i + 1].x, y[2 * i + 1].y);
}

// Chunk c from shared memory, times s.
__device__ __forceinline__ void load_chunk_f32(const float* v, uint32_t c, float s, float2 (&y)[8])
{
    const float4* p = reinterpret_cast<const float4*>(v + 16 * c);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 q = p[i];
        y[2 * i] = make_float2(__fmul_rn(q.x, s), __fmul_rn(q.y, s));
        y[2 * i + 1] = make_float2(__fmul_rn(q.z, s), __fmul_rn(q.w, s));
    }
}

}  // namespace bq
