/*
 * Checks the division the quantize kernels' fast paths use instead of a divide:
 * with rn = RN(1/s), q0 = RN(x * rn), rem = fma(-q0, s, x) (exact), the result
 * fma(rem, rn, q0) must equal the IEEE quotient RN(x / s) (Markstein's theorem on
 * division with a correctly rounded reciprocal). The kernels rely on it for scales
 * s in [2^-60, 2^100] and quotients |x / s| in [2^-40, 2^20] (smaller quotients code as
 * zero in every format). Built with hardware FMA and no contraction.
 *
 *   markstein_check A_STEP NRAND Q_STEP
 *     - scales RN(amax / Q) for every A_STEP-th positive normal bf16 amax and each Q
 *       (the formats' Qmax and the NV products), against every bf16 x;
 *     - NRAND random fp32 scales against 256 random fp32 x each;
 *     - division by each Qmax itself (the scale computation): every Q_STEP-th fp32
 *       dividend with quotient in [2^-40, 2^20], with the reciprocal RN(1/Qmax).
 * Prints the counts; exits 1 on any mismatch.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float bf16(uint32_t b) { uint32_t u = b << 16; float f; memcpy(&f, &u, 4); return f; }

static int same(float a, float b) { return memcmp(&a, &b, 4) == 0; }

static float quot(float x, float s, float rn)
{
    const float q0 = x * rn;
    const float rem = fmaf(-q0, s, x);
    return fmaf(rem, rn, q0);
}

static uint64_t st = 88172645463325252ull;
static uint64_t rnd(void) { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; }

int main(int argc, char** argv)
{
    const int astep = argc > 1 ? atoi(argv[1]) : 1;
    const long nrand = argc > 2 ? atol(argv[2]) : 0;
    const float Q[] = {7.f, 15.f, 127.f, 255.f, 448.f, 57344.f, 6.f, 6.f * 448.f, 7.f * 448.f};
    long long n = 0, bad = 0;
    for (int qi = 0; qi < 9; ++qi) {
        for (uint32_t a = 0x0080; a < 0x7F80; a += (uint32_t)astep) {
            const float s = bf16(a) / Q[qi];
            if (!(s >= 0x1p-60f && s <= 0x1p100f)) continue;
            const float rn = 1.0f / s;
            for (uint32_t b = 0x0001; b < 0x7F80; ++b) {
                const float x = bf16(b);
                if (x > s * 0x1p20f) break;
                if (x < s * 0x1p-40f) continue;
                ++n;
                if (!same(quot(x, s, rn), x / s)) ++bad;
            }
        }
    }
    for (long i = 0; i < nrand; ++i) {
        uint32_t us = (uint32_t)(rnd() & 0x007FFFFFu) | ((uint32_t)((int)(rnd() % 160) - 60 + 127) << 23);
        float s;
        memcpy(&s, &us, 4);
        const float rn = 1.0f / s;
        for (int j = 0; j < 256; ++j) {
            const int e = (int)(rnd() % 61) - 40;
            uint32_t um = (uint32_t)(rnd() & 0x007FFFFFu) | (127u << 23);
            float m;
            memcpy(&m, &um, 4);
            const float x = ldexpf(m, e) * s;
            if (!(x > 0.0f) || isinf(x)) continue;
            ++n;
            if (!same(quot(x, s, rn), x / s)) ++bad;
        }
    }
    const long qstep = argc > 3 ? atol(argv[3]) : 0;
    for (int qi = 0; qstep > 0 && qi < 7; ++qi) {
        const float q = Q[qi], rq = 1.0f / q, flo = 0x1p-40f * q, fhi = 0x1p20f * q;
        uint32_t lo, hi;
        memcpy(&lo, &flo, 4);
        memcpy(&hi, &fhi, 4);
        for (uint32_t u = lo; u <= hi; u += (uint32_t)qstep) {
            float a;
            memcpy(&a, &u, 4);
            ++n;
            if (!same(quot(a, q, rq), a / q)) ++bad;
        }
    }
    printf("checked %lld mismatches %lld\n", n, bad);
    return bad != 0;
}
