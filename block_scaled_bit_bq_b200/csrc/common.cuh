// common.cuh -- device building blocks of the block-scaled quantization kernels.
//
// Everything here is fp32 IEEE arithmetic without contraction (the library is built
// with -fmad=false; every fused multiply-add is spelled __fmaf_rn on purpose) and
// without flush-to-zero, so the kernels reproduce the CPU oracle bit for bit.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "bq.h"

namespace bq {

// ---------------------------------------------------------------------------
// Programmatic dependent launch. A kernel launched by launch_pdl may be scheduled while
// the kernel before it in the stream is still finishing: its CTAs become resident as the
// earlier kernel's CTAs leave, instead of after the earlier grid has ended and the launch
// has gone through. pdl_wait() returns once every kernel the launch depends on has
// completed and its memory operations are visible; each such kernel calls it before its
// first access to global memory, so no ordering with the earlier work is lost.
// pdl_release() lets the next such launch be scheduled once every CTA has called it (or
// exited). A CTA calls it when its streaming work is done, at the start of its final
// reduction, so that the next grid's CTAs do not share the SMs with the bulk of this
// one (released at kernel start, the dequantize and QSNR passes ran up to 8 % slower);
// kernels without a final reduction release at exit. Without launch_pdl (an ordinary
// launch) both are no-ops.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---------------------------------------------------------------------------
// Element-format traits.
// ---------------------------------------------------------------------------

template <int FMT> struct Fmt;
template <> struct Fmt<BQ_INT8_SYM>   { static constexpr bool is_int = true,  asym = false, four = false; static constexpr int qmin = -127, qmax = 127; static constexpr float qscale = 127.0f; };
template <> struct Fmt<BQ_INT8_ASYM>  { static constexpr bool is_int = true,  asym = true,  four = false; static constexpr int qmin = -128, qmax = 127; static constexpr float qscale = 255.0f; };
template <> struct Fmt<BQ_INT4_SYM>   { static constexpr bool is_int = true,  asym = false, four = true;  static constexpr int qmin = -8,   qmax = 7;   static constexpr float qscale = 7.0f; };
template <> struct Fmt<BQ_UINT4_ASYM> { static constexpr bool is_int = true,  asym = true,  four = true;  static constexpr int qmin = 0,    qmax = 15;  static constexpr float qscale = 15.0f; };
template <> struct Fmt<BQ_FP8_E4M3>   { static constexpr bool is_int = false, asym = false, four = false; static constexpr int qmin = 0,    qmax = 0;   static constexpr float qscale = 448.0f; };
template <> struct Fmt<BQ_FP8_E5M2>   { static constexpr bool is_int = false, asym = false, four = false; static constexpr int qmin = 0,    qmax = 0;   static constexpr float qscale = 57344.0f; };
template <> struct Fmt<BQ_FP4_E2M1>   { static constexpr bool is_int = false, asym = false, four = true;  static constexpr int qmin = 0,    qmax = 0;   static constexpr float qscale = 6.0f; };
// FP6, one code per byte (the low six bits), as the cvt instructions leave them
template <> struct Fmt<BQ_FP6_E2M3>   { static constexpr bool is_int = false, asym = false, four = false; static constexpr int qmin = 0,    qmax = 0;   static constexpr float qscale = 7.5f; };
template <> struct Fmt<BQ_FP6_E3M2>   { static constexpr bool is_int = false, asym = false, four = false; static constexpr int qmin = 0,    qmax = 0;   static constexpr float qscale = 28.0f; };

// Granularity kinds as the kernels see them.
enum { K_TENSOR = 0, K_GROUP = 1, K_MX = 2, K_NV = 3 };

// 1.5 * 2^23: adding it rounds an fp32 value of magnitude < 2^22 to an integer (half
// to even) and leaves that integer, two's complement, in the low bits of the sum.
constexpr float MAGIC = 12582912.0f;
constexpr uint32_t MAGIC_BITS = 0x4B400000u;
// Reciprocal bracket factors 1 -+ 2^-20 (both exact in fp32).
constexpr float BRACKET_LO = 0.99999904632568359375f;
constexpr float BRACKET_HI = 1.00000095367431640625f;
constexpr float FP32_MIN_NORMAL = 1.17549435082228750797e-38f;

// ---------------------------------------------------------------------------
// Memory access: 256-bit loads and stores (sm_100), read-only path for inputs.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&r)[8])
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]),
                   "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}

__device__ __forceinline__ void ld_nc_v4(const void* p, uint32_t (&r)[4])
{
    asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "l"(p));
}

__device__ __forceinline__ void ld_nc_v2(const void* p, uint32_t (&r)[2])
{
    asm volatile("ld.global.nc.L1::no_allocate.v2.b32 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1]) : "l"(p));
}

__device__ __forceinline__ void st_v8(void* p, const uint32_t (&r)[8])
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]),
                    "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]) : "memory");
}

__device__ __forceinline__ void st_v4(void* p, const uint32_t (&r)[4])
{
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]) : "memory");
}

__device__ __forceinline__ void st_v2(void* p, const uint32_t (&r)[2])
{
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" :: "l"(p), "r"(r[0]), "r"(r[1]) : "memory");
}

// 16 bf16 (one 32-byte chunk) -> 16 fp32, exactly. Element 2i sits in the low half
// of word i (little endian).
__device__ __forceinline__ void widen16(const uint32_t (&w)[8], float (&v)[16])
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void load16(const uint32_t* x, uint32_t chunk, float (&v)[16])
{
    uint32_t w[8];
    ld_nc_v8(x + (size_t)chunk * 8, w);
    widen16(w, v);
}

// ---------------------------------------------------------------------------
// 16-point Walsh-Hadamard transform (Sylvester order), scaled by 1/4. H16/4 is
// orthogonal and symmetric, hence its own inverse.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void fwht16(float (&y)[16])
{
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; i += 2 * h) {
#pragma unroll
            for (int j = i; j < i + h; ++j) {
                const float a = y[j], b = y[j + h];
                y[j] = __fadd_rn(a, b);
                y[j + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) y[j] = __fmul_rn(y[j], 0.25f);
}

// ---------------------------------------------------------------------------
// FP element conversions (Blackwell cvt with saturation to the largest finite value).
// The x2 forms put the first operand in the upper half of the result.
// ---------------------------------------------------------------------------

template <int FMT>
__device__ __forceinline__ uint32_t cvt_pair(float hi, float lo)
{
    uint32_t r;
    if constexpr (FMT == BQ_FP8_E4M3) {
        uint16_t h;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
        r = h;
    } else if constexpr (FMT == BQ_FP8_E5M2) {
        uint16_t h;
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
        r = h;
    } else if constexpr (FMT == BQ_FP6_E2M3) {
        uint16_t h;
        asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
        r = h;
    } else if constexpr (FMT == BQ_FP6_E3M2) {
        uint16_t h;
        asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
        r = h;
    } else {
        asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }"
            : "=r"(r) : "f"(hi), "f"(lo));
    }
    return r;
}

// Decode a pair of FP codes (packed as cvt_pair produces them) to two fp32 values,
// exactly (every E4M3 / E5M2 / E2M1 / E2M3 / E3M2 value is an fp16 value).
template <int FMT>
__device__ __forceinline__ float2 dec_pair(uint32_t pair)
{
    uint32_t h;
    if constexpr (FMT == BQ_FP8_E4M3) {
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)pair));
    } else if constexpr (FMT == BQ_FP8_E5M2) {
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"((uint16_t)pair));
    } else if constexpr (FMT == BQ_FP6_E2M3) {
        asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)pair));
    } else if constexpr (FMT == BQ_FP6_E3M2) {
        asm("cvt.rn.f16x2.e3m2x2 %0, %1;" : "=r"(h) : "h"((uint16_t)pair));
    } else {
        asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h) : "r"(pair));
    }
    __half2 hh = *reinterpret_cast<__half2*>(&h);
    return __half22float2(hh);   // .x = low half (first element), .y = high half
}

// E4M3 code of a non-negative fp32 value (round to nearest even, saturating), and back.
__device__ __forceinline__ uint32_t e4m3_code(float v) { return cvt_pair<BQ_FP8_E4M3>(0.0f, v) & 0xFFu; }
__device__ __forceinline__ float e4m3_value(uint32_t code) { return dec_pair<BQ_FP8_E4M3>(code & 0xFFu).x; }

// fp32 -> fp16 storage of a scale (saturating at 65504) and back.
__device__ __forceinline__ float round_scale_f16(float s32)
{
    return __half2float(__float2half_rn(fminf(s32, 65504.0f)));
}

// ---------------------------------------------------------------------------
// UE8M0 exponent: smallest integer e with amax <= qmax * 2^e, clamped to
// [-127, 127]; amax = 0 (or subnormal: far below any qmax * 2^-127) gives -127.
// Decided exactly on the fp32 bit fields: with amax = a * 2^A and qmax = b * 2^B
// (a, b in [1, 2)), e = A - B when a <= b, else A - B + 1.
// ---------------------------------------------------------------------------

template <int FMT>
__device__ __forceinline__ int ue8m0_exponent(float amax)
{
    constexpr float q = Fmt<FMT>::qscale;
    const uint32_t qb = __float_as_uint(q);
    const uint32_t ab = __float_as_uint(amax);
    if (!(amax >= FP32_MIN_NORMAL)) return -127;
    const int A = (int)(ab >> 23) - 127, B = (int)(qb >> 23) - 127;
    int e = A - B + (((ab & 0x7FFFFFu) > (qb & 0x7FFFFFu)) ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^k as fp32 for k in [-149, 127] (exact; subnormal below -126).
__device__ __forceinline__ float exp2i(int k)
{
    return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23)
                     : __uint_as_float(1u << (k + 149));
}

// ---------------------------------------------------------------------------
// Packed fp32 pairs (sm_100 FFMA2 / FMUL2 / FADD2: two IEEE operations per
// instruction, each rounded exactly like its scalar form).
// ---------------------------------------------------------------------------

__device__ __forceinline__ float2 splat(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b, rounded once (fma with -1 is exactly the subtraction)
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, splat(-1.0f), a); }
// -a (exact, sign bits flipped)
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

// max(a, |b|, |c|) in one three-input max
__device__ __forceinline__ float amax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float min3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Packed bf16 pairs. min / max pick one of their inputs, so they are exact; the bit
// patterns of non-negative bf16 values order like unsigned integers, so the largest
// magnitude of a pair is an unsigned 16-bit max of the sign-cleared halves.
__device__ __forceinline__ uint32_t bf2_absmax(uint32_t m, uint32_t w) { return __vmaxu2(m, w & 0x7FFF7FFFu); }

__device__ __forceinline__ uint32_t bf2_min(uint32_t a, uint32_t b)
{
    const __nv_bfloat162 r = __hmin2(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
    return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t bf2_max(uint32_t a, uint32_t b)
{
    const __nv_bfloat162 r = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
    return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16 bf16 -> 8 fp32 pairs (pair i = elements 2i, 2i+1), exactly.
__device__ __forceinline__ void widen16x2(const uint32_t (&w)[8], float2 (&v)[8])
{
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

// 16-point Walsh-Hadamard stages on pairs, unnormalised: the same additions in the same
// order as fwht16 (stage h = 1 inside each pair, stages 2, 4, 8 across pairs).
__device__ __forceinline__ void wht16x2(float2 (&v)[8])
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float a = v[i].x, b = v[i].y;
        v[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; i += 2 * h) {
#pragma unroll
            for (int j = i; j < i + h; ++j) {
                const float2 a = v[j], b = v[j + h];
                v[j] = add2(a, b);
                v[j + h] = sub2(a, b);
            }
        }
    }
}

// The block-16 rotation: those stages, then * 0.25.
__device__ __forceinline__ void fwht16x2(float2 (&v)[8])
{
    wht16x2(v);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = mul2(v[i], splat(0.25f));
}

// Power-of-two p with amax * p in [1, 2) (p = 1 for amax = 0; p kept within
// [2^-127, 2^126]) and 1 / p^2 as a double. Sums of squares are taken on values
// scaled by p, so they neither overflow nor underflow in fp32, and are scaled back
// exactly in double.
struct Pow2 {
    float p;
    double inv_p2;
};

__device__ __forceinline__ Pow2 pow2_for(float amax)
{
    const uint32_t b = __float_as_uint(amax) & 0x7FFFFFFFu;
    int k = (int)(b >> 23) - 127;           // floor(log2) for normal amax
    if ((b >> 23) == 0) k = 0;              // zero: p = 1; subnormal: see below
    if (b != 0 && (b >> 23) == 0) k = -126;
    k = k > 127 ? 127 : (k < -126 ? -126 : k);
    Pow2 r;
    r.p = exp2i(-k);
    r.inv_p2 = __longlong_as_double((long long)(1023 + 2 * k) << 52);
    return r;
}

// ---------------------------------------------------------------------------
// Division x / s decided without a per-element divide.
//
// r ~ 1/s within 2^-23; r_lo = RN(r (1 - 2^-20)) and r_hi = RN(r (1 + 2^-20))
// satisfy x r_lo < RN(x/s) < x r_hi for x > 0 (reversed for x < 0) whenever s and r
// are normal: RN(x/s) is within 2^-24 of x/s, and r_lo, r_hi are at least
// 2^-20 - 2^-23 - 2^-24 away from 1/s. Any monotone rounding rule
// (to the integer grid, or to an FP element grid) therefore returns the same value
// on both bracket ends exactly when it returns that value for RN(x/s). When the two
// ends disagree, the code is recomputed from a correctly rounded division.
// ---------------------------------------------------------------------------

struct Recip {
    float s, rlo, rhi;
    bool fast;
};

__device__ __forceinline__ float rcp_approx(float s)
{
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

// The reciprocal need not be correctly rounded: the hardware approximation is within
// 1 ulp (2^-23 relative), and with the 1 -+ 2^-20 factors r_lo and r_hi still lie
// strictly outside 1/s * (1 -+ 2^-24).
__device__ __forceinline__ Recip make_recip(float s, float amax)
{
    Recip r;
    r.s = s;
    const float inv = rcp_approx(s);
    r.rlo = __fmul_rn(inv, BRACKET_LO);
    r.rhi = __fmul_rn(inv, BRACKET_HI);
    // s well inside the normal range (so 1/s, r_lo, r_hi are normal and the residual
    // x - h s of a tie check is exact when zero); |x/s| < 2^22 keeps the integer magic
    // in range.
    r.fast = (s >= 0x1p-100f) && (s <= 1.0e37f) && (__fmul_rn(amax, r.rhi) < 4194304.0f);
    return r;
}

// ---------------------------------------------------------------------------
// Byte / nibble packing.
// ---------------------------------------------------------------------------

// low bytes of four words -> one word (byte 0 from a)
__device__ __forceinline__ uint32_t pack_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    const uint32_t ab = __byte_perm(a, b, 0x0040);
    const uint32_t cd = __byte_perm(c, d, 0x0040);
    return __byte_perm(ab, cd, 0x5410);
}

// low nibbles of two words -> one byte value (nibble 0 from a)
__device__ __forceinline__ uint32_t pack_nibbles(uint32_t a, uint32_t b)
{
    return (a & 0xFu) | ((b << 4) & 0xF0u);
}

// ---------------------------------------------------------------------------
// Fast unsigned division by a runtime constant (round-down multiply-high method).
// ---------------------------------------------------------------------------

struct FastDiv {
    uint32_t d, m, s;
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d)
{
    FastDiv f;
    f.d = d;
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    f.s = l;
    f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1ull);
    if (d == 1) f.m = 0;
    return f;
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f)
{
    const uint64_t t = (uint64_t)__umulhi(n, f.m) + n;
    return (uint32_t)(t >> f.s);
}

// Block scales in a block-scaled GEMM's layout: the [rows, nb] scale matrix in 128 x 4
// tiles of 512 bytes (row-major tile order), entry (r, c) of a tile at byte
// (r % 32) * 16 + (r / 32) * 4 + c. nb is a multiple of 4 here.
__host__ __device__ inline uint32_t gemm_scale_offset(uint32_t r, uint32_t c, uint32_t nb)
{
    return (((r >> 7) * (nb >> 2) + (c >> 2)) << 9) + ((r & 31u) << 4) + (((r >> 5) & 3u) << 2) + (c & 3u);
}

// The same for the flat unit index u = r * nb + c (nb_div: fast division by nb).
__device__ __forceinline__ uint32_t gemm_unit_offset(uint32_t u, const FastDiv& nb_div)
{
    const uint32_t r = fast_div(u, nb_div);
    return gemm_scale_offset(r, u - r * nb_div.d, nb_div.d);
}

// ---------------------------------------------------------------------------
// Workspace layout and the cross-CTA reduction (last CTA finishes; no waiting).
// ---------------------------------------------------------------------------

constexpr int MAX_GRID = 2048;

struct WsHeader {
    unsigned int counter_range;
    unsigned int counter_stats;
    unsigned int pad0[2];
    float amax, vmin, vmax, pad1;
};

struct RangeSlot { float amax, vmin, vmax, pad; };

struct StatSlot { double err2, x2, ksum, kmax, nunits, ss; };

// stats slots: one per CTA (MAX_GRID), or one per warp for the flat kernel's batches
constexpr int MAX_STAT_SLOTS = 4096;
constexpr size_t WS_HEADER_BYTES = 256;
constexpr size_t WS_RANGE_OFF = WS_HEADER_BYTES;
constexpr size_t WS_STAT_OFF = WS_RANGE_OFF + sizeof(RangeSlot) * MAX_GRID;
constexpr size_t WS_BYTES = WS_STAT_OFF + sizeof(StatSlot) * MAX_STAT_SLOTS;

__device__ __forceinline__ WsHeader* ws_header(uint8_t* ws) { return reinterpret_cast<WsHeader*>(ws); }
__device__ __forceinline__ RangeSlot* ws_range(uint8_t* ws) { return reinterpret_cast<RangeSlot*>(ws + WS_RANGE_OFF); }
__device__ __forceinline__ StatSlot* ws_stats(uint8_t* ws) { return reinterpret_cast<StatSlot*>(ws + WS_STAT_OFF); }

// Per-thread QSNR / crest-factor accumulators (kept small: they live in registers
// through the whole kernel).
struct Acc {
    double err2 = 0.0, x2 = 0.0, ksum = 0.0;
    float kmax = 0.0f;
    uint32_t nunits = 0;
};

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ double warp_max(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

__device__ __forceinline__ float warp_maxf(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

__device__ __forceinline__ float warp_minf(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Block totals in double.
struct AccD {
    double err2 = 0.0, x2 = 0.0, ksum = 0.0, kmax = 0.0, nunits = 0.0;
};

// Sum (max for kmax) over the 32 lanes of a warp: a fixed xor tree, the same in every
// lane, so the result does not depend on timing.
__device__ __forceinline__ AccD warp_reduce_acc(AccD a)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a.err2 += __shfl_xor_sync(0xFFFFFFFFu, a.err2, o);
        a.x2 += __shfl_xor_sync(0xFFFFFFFFu, a.x2, o);
        a.ksum += __shfl_xor_sync(0xFFFFFFFFu, a.ksum, o);
        a.kmax = fmax(a.kmax, __shfl_xor_sync(0xFFFFFFFFu, a.kmax, o));
        a.nunits += __shfl_xor_sync(0xFFFFFFFFu, a.nunits, o);
    }
    return a;
}

// Block-wide reduction (every thread calls it; blockDim.x a multiple of 32, at most
// 1024): warps reduce, then warp 0 reduces the warps' totals. The result is valid in
// warp 0.
__device__ __forceinline__ AccD block_reduce_acc(AccD a)
{
    __shared__ double sh[32][5];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    a = warp_reduce_acc(a);
    __syncthreads();                 // sh may still be read by a previous call
    if (lane == 0) {
        sh[warp][0] = a.err2; sh[warp][1] = a.x2; sh[warp][2] = a.ksum;
        sh[warp][3] = a.kmax; sh[warp][4] = a.nunits;
    }
    __syncthreads();
    AccD t;
    if (warp == 0) {
        if (lane < nw) {
            t.err2 = sh[lane][0]; t.x2 = sh[lane][1]; t.ksum = sh[lane][2];
            t.kmax = sh[lane][3]; t.nunits = sh[lane][4];
        }
        t = warp_reduce_acc(t);
    }
    return t;
}

// Add one to a counter with release (this thread's earlier writes are visible to whoever
// observes the new value) and acquire (later reads see what the earlier adders released).
__device__ __forceinline__ unsigned int atomic_add_acq_rel(unsigned int* p, unsigned int v)
{
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Called by every thread of every CTA at kernel end. Each CTA leaves its partial in
// a workspace slot; the CTA that arrives last sums the slots (in a fixed order: slot by
// slot per thread, then the xor trees) and writes the result. tensor_kappa: the unit is
// the whole tensor; kappa = amax / sqrt(x2 / n_elems) is formed from the totals.
__device__ __forceinline__ void finish_stats(Acc mine, uint8_t* ws, bq_stats* out,
                                             bool tensor_kappa, float tensor_amax,
                                             double n_elems, bool write_kappa)
{
    pdl_release();                   // the CTA's streaming work is done
    __shared__ bool is_last;
    AccD m;
    m.err2 = mine.err2; m.x2 = mine.x2; m.ksum = mine.ksum; m.kmax = (double)mine.kmax; m.nunits = (double)mine.nunits;
    const AccD t = block_reduce_acc(m);
    StatSlot* slots = ws_stats(ws);
    WsHeader* h = ws_header(ws);
    if (threadIdx.x == 0) {
        slots[blockIdx.x] = StatSlot{t.err2, t.x2, t.ksum, t.kmax, t.nunits, 0.0};
        is_last = (atomic_add_acq_rel(&h->counter_stats, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    AccD a;
    for (unsigned i = threadIdx.x; i < gridDim.x; i += blockDim.x) {
        const double* p = reinterpret_cast<const double*>(&slots[i]);
        a.err2 += __ldcg(p + 0); a.x2 += __ldcg(p + 1); a.ksum += __ldcg(p + 2);
        a.kmax = fmax(a.kmax, __ldcg(p + 3)); a.nunits += __ldcg(p + 4);
    }
    const AccD tot = block_reduce_acc(a);
    if (threadIdx.x == 0) {
        bq_stats r;
        r.err2 = tot.err2;
        r.x2 = tot.x2;
        r.kappa_sum = tot.ksum;
        r.kappa_max = tot.kmax;
        r.n_units = tot.nunits;
        if (tensor_kappa) {
            r.kappa_sum = r.kappa_max = r.n_units = 0.0;
            if (tot.x2 > 0.0) {
                const double k = (double)tensor_amax / sqrt(tot.x2 / n_elems);
                r.kappa_sum = k; r.kappa_max = k; r.n_units = 1.0;
            }
        }
        if (!write_kappa) r.kappa_sum = r.kappa_max = r.n_units = 0.0;
        *out = r;
        h->counter_stats = 0u;   // ready for the next call on this workspace
    }
}

// Crest factor of one unit in fp32: amax / sqrt(ss / n).
__device__ __forceinline__ void kappa_add(Acc& a, float amax, float ss, float inv_n)
{
    if (ss > 0.0f) {
        const float k = __fmul_rn(amax, rsqrtf(__fmul_rn(ss, inv_n)));
        a.ksum += (double)k;
        a.kmax = fmaxf(a.kmax, k);
        a.nunits += 1u;
    }
}

}  // namespace bq
