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
//
// Layout: element o of chunk c (index 16c + o) sits at
//   16c + 16 (c >> 4) + 4 (((o >> 2) + (c >> 1)) & 3) + (o & 3),
// i.e. the chunk's four 16-byte quarters rotated by (c >> 1) & 3, and 16 floats of
// padding after every 16 chunks. Chunk stores and loads by consecutive threads, and
// both kinds of pass below, then touch 32 distinct banks per 32 accesses.
#pragma once

#include "common.cuh"

namespace bq {

// Threads per CTA of the row-transform kernels (a row at a time): 128 keeps every thread
// busy in both passes of a 4096-column row (n / 32 pairs each) and lets 6-8 CTAs, so as
// many rows, share an SM.
constexpr int RT_THREADS = 128;

// Floats of shared memory for a row of n values.
__host__ __device__ constexpr uint32_t rot_row_floats(uint32_t n) { return n + n / 16; }

__device__ __forceinline__ uint32_t rot_chunk_base(uint32_t c) { return 16u * c + 16u * (c >> 4); }

// Quarter j of chunk c (its four floats are contiguous).
__device__ __forceinline__ uint32_t rot_quarter(uint32_t c, uint32_t j)
{
    return rot_chunk_base(c) + 4u * ((j + (c >> 1)) & 3u);
}

// Stage h of R values, two independent groups at once (packed pairs).
template <int R, int H>
__device__ __forceinline__ void wht_stage2(float2 (&t)[R])
{
#pragma unroll
    for (int i = 0; i < R; i += 2 * H) {
#pragma unroll
        for (int j = 0; j < H; ++j) {
            const float2 a = t[i + j], b = t[i + j + H];
            t[i + j] = add2(a, b);
            t[i + j + H] = sub2(a, b);
        }
    }
}

// Stages 1 .. R / 2 of R values (R = 2, 4, 8 or 16), two groups at once.
template <int R>
__device__ __forceinline__ void wht_group2(float2 (&t)[R])
{
    wht_stage2<R, 1>(t);
    if constexpr (R > 2) wht_stage2<R, 2>(t);
    if constexpr (R > 4) wht_stage2<R, 4>(t);
    if constexpr (R > 8) wht_stage2<R, 8>(t);
}

// A thread takes two adjacent groups at a time: groups 2q and 2q + 1 hold elements o
// and o + 1 (o even) of the same chunks, which sit side by side (one 8-byte access).

// Stages S .. S R / 2 for stride S >= 256: the chunks of a group are S / 16 apart, a
// multiple of 16, so each value's quarter rotation is the group's and the k-th value
// sits (S + S / 16) k floats after the first.
template <int R>
__device__ __forceinline__ void wht_pass_wide(float* v, uint32_t n, uint32_t S)
{
    // S is a power of two: the group's position by shifts and masks, not divisions
    const uint32_t lg = (uint32_t)(__ffs((int)S) - 1);
    const uint32_t npairs = n / (2 * R), step = S + S / 16;
    for (uint32_t q = threadIdx.x; q < npairs; q += blockDim.x) {
        const uint32_t g = 2 * q;
        const uint32_t base = (g & (S - 1u)) + ((g >> lg) << lg) * R;
        const uint32_t c = base >> 4, o = base & 15u;
        float2* p0 = reinterpret_cast<float2*>(v + rot_chunk_base(c) + 4u * (((o >> 2) + (c >> 1)) & 3u) + (o & 3u));
        float2 t[R];
#pragma unroll
        for (int k = 0; k < R; ++k) t[k] = p0[(step / 2) * k];
        wht_group2<R>(t);
#pragma unroll
        for (int k = 0; k < R; ++k) p0[(step / 2) * k] = t[k];
    }
}

// Stages 16 .. 128 (S = 16, R = 16, n >= 256): group g holds element o = g % 16 of 16
// consecutive chunks starting at a multiple of 16, so the quarter rotation of the k-th
// value is ((k >> 1) & 3) past the element's own quarter.
__device__ __forceinline__ void wht_pass_16(float* v, uint32_t n)
{
    const uint32_t npairs = n / 32;
    for (uint32_t q = threadIdx.x; q < npairs; q += blockDim.x) {
        const uint32_t o = (2 * q) & 15u, c0 = (q >> 3) * 16u;
        const uint32_t p0 = rot_chunk_base(c0) + (o & 3u), oq = o >> 2;
        float2* pm[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) pm[m] = reinterpret_cast<float2*>(v + p0 + 4u * ((oq + (uint32_t)m) & 3u));
        float2 t[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) t[k] = pm[(k >> 1) & 3][8 * k];
        wht_group2<16>(t);
#pragma unroll
        for (int k = 0; k < 16; ++k) pm[(k >> 1) & 3][8 * k] = t[k];
    }
}

// Stages h = 16 .. n / 2 of the row in v (256 <= n <= 65536, a power of two). Called by
// every thread of the block; synchronizes before each pass and at the end.
__device__ __forceinline__ void wht_smem_stages(float* v, uint32_t n)
{
    __syncthreads();
    wht_pass_16(v, n);
    for (uint32_t S = 256; S < n; S *= 16) {
        const uint32_t R = n / S;
        __syncthreads();
        if (R >= 16) wht_pass_wide<16>(v, n, S);
        else if (R == 8) wht_pass_wide<8>(v, n, S);
        else if (R == 4) wht_pass_wide<4>(v, n, S);
        else wht_pass_wide<2>(v, n, S);
    }
    __syncthreads();
}

// The random signs as XOR masks of bf16 pairs, one 32-bit word per two columns (bit 15:
// column 2j, bit 31: column 2j + 1), built once per CTA in shared memory after the row's
// floats: a chunk's signs are then two 16-byte loads and one XOR per pair of values.
__host__ __device__ constexpr uint32_t rot_smem_bytes(uint32_t n, bool signs)
{
    return rot_row_floats(n) * 4u + (signs ? n / 2 * 4u : 0u);
}

__device__ __forceinline__ void build_sign_masks(uint32_t* m, const uint32_t* sign_bits, uint32_t n)
{
    for (uint32_t j = threadIdx.x; j < n / 2; j += blockDim.x) {
        const uint32_t b = (__ldg(sign_bits + (j >> 4)) >> ((2u * j) & 31u)) & 3u;
        m[j] = ((b & 1u) << 15) | ((b & 2u) << 30);
    }
}

// XOR the 8 bf16-pair words of chunk c with their sign masks.
__device__ __forceinline__ void flip_words(const uint32_t* m, uint32_t c, uint32_t (&w)[8])
{
    const uint4 a = *reinterpret_cast<const uint4*>(m + 8 * c);
    const uint4 b = *reinterpret_cast<const uint4*>(m + 8 * c + 4);
    w[0] ^= a.x; w[1] ^= a.y; w[2] ^= a.z; w[3] ^= a.w;
    w[4] ^= b.x; w[5] ^= b.y; w[6] ^= b.z; w[7] ^= b.w;
}

__device__ __forceinline__ void store_chunk_f32(float* v, uint32_t c, const float2 (&y)[8])
{
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4*>(v + rot_quarter(c, j)) =
            make_float4(y[2 * j].x, y[2 * j].y, y[2 * j + 1].x, y[2 * j + 1].y);
}

// Chunk c from shared memory, times s.
__device__ __forceinline__ void load_chunk_f32(const float* v, uint32_t c, float s, float2 (&y)[8])
{
    const float2 S = splat(s);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 q = *reinterpret_cast<const float4*>(v + rot_quarter(c, j));
        y[2 * j] = mul2(make_float2(q.x, q.y), S);
        y[2 * j + 1] = mul2(make_float2(q.z, q.w), S);
    }
}

}  // namespace bq
