/*
 * bq_oracle.c -- plain, slow CPU oracle for block-scaled tensor quantization.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the CPU-baseline leg of
 * the benchmark load this file's shared library; the product path never does. It
 * shares no code with the CUDA library: its own format tables, its own
 * rounding, its own loops.
 *
 * What it follows (page = title of the source web page, then section):
 *   - "INT4/INT8/FP8 quantization" (guijiagi) §INT8: q = round(w/scale) + zero_point,
 *     w = scale * (q - zero_point); §INT4: range [-8, 7], group-wise scale
 *     w_max / 7, round then clamp, two codes per byte (0.5 byte per parameter);
 *     §FP8: E4M3 range +-448, E5M2 range +-57344.
 *   - "INT vs FP at fine granularity" (cyqw) §2.1: Xq = clip(round(X/s), Qmin, Qmax)*s
 *     with the AbsMax scale s = max|X| / Qmax, symmetric INT8 [-127, 127], MXINT8
 *     blocks of 32 sharing a UE8M0 scale; §2.2: FP value (-1)^s (1.m) 2^(e-bias),
 *     MXFP8 = E4M3; §3.1: per-tensor / per-channel / block granularity; §4.1: QSNR =
 *     -10 log10(||X - Xq||^2 / ||X||^2) and the crest factor kappa; §4.2 and §7.2:
 *     Hadamard rotation before NVINT4.
 *   - "Quantization survey" (walkerchi) §4.1 FP table: E2M1 +-6, min 0.5; E4M3 +-448,
 *     min ~0.00195; E5M2 +-57344, min ~1.5e-5; bit layouts [s][e..][m..];
 *     §4.3.1: MXFP4 (E2M1, block 32, E8M0 scale) vs NVFP4 (E2M1, block 16, E4M3
 *     block scale, FP32 tensor scale); §4.3.2: x = x_q * s_block * S_tensor;
 *     §5.3: orthogonal Hadamard rotation R^T R = I.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - every division that decides a code is a correctly rounded fp32 division, and
 *     the code is taken from that fp32 quotient (round half to even);
 *   - FP encoders round to nearest, ties to the code with an even mantissa, and
 *     saturate to the largest finite value ("satfinite"); the sign of a value that
 *     rounds to zero is kept;
 *   - asymmetric ranges include zero: min' = min(min, 0), max' = max(max, 0);
 *     zero_point = Qmin + round(-min'/s), clamped; q = clamp(round(x/s) + zp); a range
 *     whose fp32 scale would overflow saturates at the largest finite fp32 value;
 *   - clamping applies to the rounded quotient whatever its magnitude;
 *   - the quantizer divides by the scale as stored (fp16 scales are rounded first,
 *     with saturation to 65504);
 *   - MX exponent: the smallest integer e with amax <= Qmax * 2^e, decided exactly,
 *     clamped to [-127, 127]; amax = 0 gives e = -127;
 *   - NV: S = A / (Qmax * 448); s_b = E4M3((amax_b / Qmax) / S); d = s_b * S;
 *     code = enc(x / d); a block with d = 0 (or S = 0) gets zero codes;
 *     dequant (code * s_b) * S, left to right;
 *   - Hadamard: a 16-point Walsh-Hadamard transform of each run of 16 elements of
 *     a row, stages h = 1, 2, 4, 8 of (a + b, a - b), then * 0.25 (an involution);
 *   - QSNR is measured in the original domain; kappa of a scaling unit is
 *     amax / sqrt(mean of squares) over the values that unit quantizes; units whose
 *     sum of squares is zero are skipped.
 *
 * Every function here has a pin in the not-gpu tests (format tables, exhaustive
 * round trips, hand-worked tensors, closed forms, library cross-checks); none is
 * "parity unpinned".
 */

#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Scheme vocabulary (the oracle's own numbering).                            */
/* ------------------------------------------------------------------------- */

enum { F_INT8_SYM = 0, F_INT8_ASYM = 1, F_INT4_SYM = 2, F_UINT4_ASYM = 3,
       F_E4M3 = 4, F_E5M2 = 5, F_E2M1 = 6, F_E2M3 = 7, F_E3M2 = 8 };
enum { G_TENSOR = 0, G_ROW = 1, G_GROUP = 2, G_MX = 3, G_NV = 4, G_TILE2D = 5 };

/* 2-D tiles: one scale per TILE_ROWS x block (= 128 x 128) tile, the weight scaling of
 * DeepSeek-V3's FP8 training ("Quantization survey" (walkerchi) §4.4: 1x128 activation
 * tiles, 128x128 weight tiles, E4M3 throughout). */
#define TILE_ROWS 128
enum { SD_FP32 = 0, SD_FP16 = 1, SD_UE8M0 = 2, SD_E4M3 = 3 };

/* ------------------------------------------------------------------------- */
/* Small FP formats: decode by the bit-field formula, encode by enumeration.  */
/* ------------------------------------------------------------------------- */

/* E4M3 ("FN" variant: the top exponent holds normals, only S.1111.111 is NaN),
 * E5M2 (IEEE-like: the top exponent is inf/NaN), E2M1, E2M3, E3M2 (no specials).
 * The biases 7, 15, 1 are the ones that give the pages' smallest positive values
 * 2^-9 ~ 0.00195, 2^-16 ~ 1.5e-5 and 0.5 ("Quantization survey" §4.1 table).
 * FP6: that table gives E2M3 range +-7.5 and E3M2 range +-28, which fix the biases at
 * 1 and 3; its smallest positive values (0.0625, ~0.0156) belong to other biases and
 * contradict the ranges. The ranges are kept: the smallest positive values are then
 * 0.125 (E2M3) and 0.0625 (E3M2). */
typedef struct { int ebits, mbits, bias, kind; } fpspec;
enum { KIND_FN = 0, KIND_IEEE = 1, KIND_PLAIN = 2 };

static int spec_of(int fp, fpspec* s)
{
    switch (fp) {
    case F_E4M3: s->ebits = 4; s->mbits = 3; s->bias = 7;  s->kind = KIND_FN;    return 0;
    case F_E5M2: s->ebits = 5; s->mbits = 2; s->bias = 15; s->kind = KIND_IEEE;  return 0;
    case F_E2M1: s->ebits = 2; s->mbits = 1; s->bias = 1;  s->kind = KIND_PLAIN; return 0;
    case F_E2M3: s->ebits = 2; s->mbits = 3; s->bias = 1;  s->kind = KIND_PLAIN; return 0;
    case F_E3M2: s->ebits = 3; s->mbits = 2; s->bias = 3;  s->kind = KIND_PLAIN; return 0;
    default: return -1;
    }
}

/* Decoded value of a code (NaN for NaN codes, +-inf for E5M2 infinities). */
double orc_fp_decode(int fp, unsigned code)
{
    fpspec f;
    if (spec_of(fp, &f)) return NAN;
    unsigned nb = 1 + f.ebits + f.mbits;
    code &= (1u << nb) - 1;
    unsigned sign = code >> (f.ebits + f.mbits);
    unsigned e = (code >> f.mbits) & ((1u << f.ebits) - 1);
    unsigned m = code & ((1u << f.mbits) - 1);
    unsigned etop = (1u << f.ebits) - 1;
    double mag;
    if (f.kind == KIND_FN && e == etop && m == (1u << f.mbits) - 1) return NAN;
    if (f.kind == KIND_IEEE && e == etop) mag = (m == 0) ? INFINITY : NAN;
    else if (e == 0) mag = ldexp((double)m, 1 - f.bias - f.mbits);          /* subnormal */
    else mag = ldexp(1.0 + ldexp((double)m, -f.mbits), (int)e - f.bias);  /* normal */
    if (isnan(mag)) return NAN;
    return sign ? -mag : mag;
}

/* Table of the non-negative finite values, in code order (which is value order). */
typedef struct { int n; double val[128]; unsigned code[128]; unsigned signbit; } fptable;

static void build_table(int fp, fptable* t)
{
    fpspec f;
    spec_of(fp, &f);
    unsigned nb = 1 + f.ebits + f.mbits;
    t->n = 0;
    t->signbit = 1u << (nb - 1);
    for (unsigned c = 0; c < t->signbit; c++) {
        double v = orc_fp_decode(fp, c);
        if (isnan(v) || isinf(v)) continue;
        t->val[t->n] = v;
        t->code[t->n] = c;
        t->n++;
    }
}

static const fptable* table_of(int fp)
{
    static fptable t4, t5, t2, t6a, t6b;
    static int ready = 0;
    if (!ready) {
        build_table(F_E4M3, &t4); build_table(F_E5M2, &t5); build_table(F_E2M1, &t2);
        build_table(F_E2M3, &t6a); build_table(F_E3M2, &t6b);
        ready = 1;
    }
    return fp == F_E4M3 ? &t4 : fp == F_E5M2 ? &t5 : fp == F_E2M1 ? &t2 : fp == F_E2M3 ? &t6a : &t6b;
}

/* Nearest table value to v; ties go to the code whose mantissa LSB is 0 (even);
 * |v| at or beyond the largest finite value saturates to it; the sign is kept,
 * including on zero. */
unsigned orc_fp_encode(int fp, float v)
{
    const fptable* t = table_of(fp);
    unsigned neg = signbit(v) ? t->signbit : 0u;
    double a = fabs((double)v);
    double top = t->val[t->n - 1];
    if (a >= top) return t->code[t->n - 1] | neg;
    int lo = 0, hi = t->n - 1;          /* val[lo] <= a < val[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (t->val[mid] <= a) lo = mid; else hi = mid;
    }
    double dl = a - t->val[lo], dh = t->val[hi] - a;
    unsigned c;
    if (dl < dh) c = t->code[lo];
    else if (dh < dl) c = t->code[hi];
    else c = (t->code[lo] & 1u) == 0 ? t->code[lo] : t->code[hi];
    return c | neg;
}

/* ------------------------------------------------------------------------- */
/* bf16 / fp16 / UE8M0                                                        */
/* ------------------------------------------------------------------------- */

float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest even on the 16 dropped bits. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);  /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* fp32 -> fp16 bits through the compiler's IEEE conversion (round to nearest even). */
uint16_t orc_f32_to_f16(float f)
{
    _Float16 h = (_Float16)f;
    uint16_t b;
    memcpy(&b, &h, 2);
    return b;
}

float orc_f16_to_f32(uint16_t b)
{
    _Float16 h;
    memcpy(&h, &b, 2);
    return (float)h;
}

/* Smallest integer e with amax <= qmax * 2^e (exact comparisons in double), clamped
 * to the UE8M0 range [-127, 127]; amax = 0 (or not positive) gives -127. */
int orc_ue8m0_exponent(float amax, float qmax)
{
    if (!(amax > 0.0f)) return -127;
    double a = (double)amax, q = (double)qmax;
    int e = (int)ceil(log2(a / q));
    while (a > q * ldexp(1.0, e)) e++;
    while (a <= q * ldexp(1.0, e - 1)) e--;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* ------------------------------------------------------------------------- */
/* 16-point Walsh-Hadamard transform, Sylvester order, scaled by 1/4.          */
/* ------------------------------------------------------------------------- */

void orc_fwht16(float* y)
{
    for (int h = 1; h < 16; h *= 2)
        for (int i = 0; i < 16; i += 2 * h)
            for (int j = i; j < i + h; j++) {
                float a = y[j], b = y[j + h];
                y[j] = a + b;
                y[j + h] = a - b;
            }
    for (int j = 0; j < 16; j++) y[j] = y[j] * 0.25f;
}

/* ------------------------------------------------------------------------- */
/* Scheme parameters                                                          */
/* ------------------------------------------------------------------------- */

typedef struct {
    int fmt, gran, block, sdt, had;
    int is_int, is_asym, bits4;  /* format family */
    int qmin, qmax;              /* integer code range */
    float qscale;                /* the Qmax that the scale maps amax (or the range) to */
    int64_t unit;                /* elements sharing one scale along a row (0 = tensor) */
} scheme;

static int make_scheme(int fmt, int gran, int block, int sdt, int had, int64_t cols, scheme* s)
{
    memset(s, 0, sizeof *s);
    s->fmt = fmt; s->gran = gran; s->block = block; s->sdt = sdt; s->had = had ? 1 : 0;
    switch (fmt) {
    case F_INT8_SYM:   s->is_int = 1; s->qmin = -127; s->qmax = 127; s->qscale = 127.0f; break;
    case F_INT8_ASYM:  s->is_int = 1; s->is_asym = 1; s->qmin = -128; s->qmax = 127; s->qscale = 255.0f; break;
    case F_INT4_SYM:   s->is_int = 1; s->bits4 = 1; s->qmin = -8; s->qmax = 7; s->qscale = 7.0f; break;
    case F_UINT4_ASYM: s->is_int = 1; s->is_asym = 1; s->bits4 = 1; s->qmin = 0; s->qmax = 15; s->qscale = 15.0f; break;
    case F_E4M3: s->qscale = 448.0f; break;
    case F_E5M2: s->qscale = 57344.0f; break;
    case F_E2M1: s->bits4 = 1; s->qscale = 6.0f; break;
    case F_E2M3: s->qscale = 7.5f; break;          /* FP6, one code per byte */
    case F_E3M2: s->qscale = 28.0f; break;
    default: return -1;
    }
    if (cols <= 0 || cols % 16) return -2;
    if (s->bits4 && cols % 2) return -2;
    switch (gran) {
    case G_TENSOR:
    case G_ROW:
        if (fmt == F_E2M1 || fmt == F_E2M3 || fmt == F_E3M2) return -1;
        if (sdt != SD_FP32 && sdt != SD_FP16) return -1;
        s->unit = gran == G_ROW ? cols : 0;
        break;
    case G_GROUP:
        if (fmt == F_E2M1 || fmt == F_E2M3 || fmt == F_E3M2) return -1;
        if (sdt != SD_FP32 && sdt != SD_FP16) return -1;
        if (block != 16 && block != 32 && block != 64 && block != 128 && block != 256 && block != 512) return -1;
        if (cols % block) return -2;
        s->unit = block;
        break;
    case G_MX:
        if (!(fmt == F_INT8_SYM || fmt == F_E4M3 || fmt == F_E5M2 || fmt == F_E2M1 ||
              fmt == F_E2M3 || fmt == F_E3M2)) return -1;
        if (block != 32 || sdt != SD_UE8M0) return -1;
        if (cols % 32) return -2;
        s->unit = 32;
        break;
    case G_TILE2D:
        if (fmt == F_E2M1 || fmt == F_E2M3 || fmt == F_E3M2) return -1;
        if (sdt != SD_FP32 && sdt != SD_FP16) return -1;
        if (block != 128) return -1;
        if (cols % 128) return -2;
        s->unit = 128;
        break;
    case G_NV:
        if (!(fmt == F_E2M1 || fmt == F_INT4_SYM)) return -1;
        if (block != 16 || sdt != SD_E4M3) return -1;
        if (fmt == F_INT4_SYM) s->qmin = -7;   /* NVINT4: symmetric [-7, 7] */
        s->unit = 16;
        break;
    default:
        return -1;
    }
    return 0;
}

/* Index of the scale of row r, unit u (u = column / unit). */
static int64_t scale_index(int gran, int64_t r, int64_t u, int64_t upr)
{
    if (gran == G_TENSOR) return 0;
    if (gran == G_TILE2D) return (r / TILE_ROWS) * upr + u;
    return r * upr + u;
}

/* Round a computed fp32 scale to its storage dtype and back (fp16 saturates). */
static float store_scale(float s32, int sdt)
{
    if (sdt == SD_FP16) {
        if (s32 > 65504.0f) s32 = 65504.0f;
        return orc_f16_to_f32(orc_f32_to_f16(s32));
    }
    return s32;
}

static void write_scale(void* arr, int64_t i, float s, int sdt)
{
    if (sdt == SD_FP16) ((uint16_t*)arr)[i] = orc_f32_to_f16(s);
    else ((float*)arr)[i] = s;
}

static float read_scale(const void* arr, int64_t i, int sdt)
{
    if (sdt == SD_FP16) return orc_f16_to_f32(((const uint16_t*)arr)[i]);
    return ((const float*)arr)[i];
}

static int clampi(int v, int lo, int hi) { return v < lo ? lo : v > hi ? hi : v; }

/* clamp(round_half_even(v) + add, lo, hi) for any finite or infinite v: the clamp
 * applies to the rounded value whatever its magnitude (no out-of-range int conversion). */
static int round_clamp(float v, int add, int lo, int hi)
{
    float r = rintf(v);
    if (r < -1.0e9f) return lo;
    if (r > 1.0e9f) return hi;
    return clampi((int)r + add, lo, hi);
}

static void put_code(uint8_t* codes, int64_t row, int64_t cols, int64_t j, unsigned c, int bits4)
{
    if (!bits4) { codes[row * cols + j] = (uint8_t)c; return; }
    uint8_t* b = &codes[row * (cols / 2) + j / 2];
    if (j % 2 == 0) *b = (uint8_t)((*b & 0xF0u) | (c & 0xFu));
    else *b = (uint8_t)((*b & 0x0Fu) | ((c & 0xFu) << 4));
}

static unsigned get_code(const uint8_t* codes, int64_t row, int64_t cols, int64_t j, int bits4)
{
    if (!bits4) return codes[row * cols + j];
    uint8_t b = codes[row * (cols / 2) + j / 2];
    return (j % 2 == 0) ? (b & 0xFu) : (b >> 4);
}

/* two's-complement value of an 8- or 4-bit integer code */
static int int_of_code(unsigned c, int bits4, int is_unsigned)
{
    if (is_unsigned) return (int)c;
    if (bits4) return (c & 0x8u) ? (int)c - 16 : (int)c;
    return (c & 0x80u) ? (int)c - 256 : (int)c;
}

/* The values a row quantizes: x itself, or its 16-blocks rotated. */
static void load_row(const uint16_t* x, int64_t row, int64_t cols, int had, float* y)
{
    for (int64_t j = 0; j < cols; j++) y[j] = orc_bf16_to_f32(x[row * cols + j]);
    if (had)
        for (int64_t j = 0; j < cols; j += 16) orc_fwht16(y + j);
}

/* amax, min and max over the (rotated) tensor: the pre-pass of per-tensor schemes. */
int orc_tensor_range(const uint16_t* x, int64_t rows, int64_t cols, int hadamard, float* out3)
{
    if (cols <= 0 || cols % 16) return -2;
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    if (!y) return -3;
    float amax = 0.0f, mn = 0.0f, mx = 0.0f;
    int first = 1;
    for (int64_t r = 0; r < rows; r++) {
        load_row(x, r, cols, hadamard, y);
        for (int64_t j = 0; j < cols; j++) {
            float a = fabsf(y[j]);
            if (a > amax) amax = a;
            if (first || y[j] < mn) mn = y[j];
            if (first || y[j] > mx) mx = y[j];
            first = 0;
        }
    }
    free(y);
    out3[0] = amax; out3[1] = mn; out3[2] = mx;
    return 0;
}

/* Quantization of one scaling unit: y[0..n) (already rotated if needed), given the
 * unit's range. Writes codes, returns the stored scale / zero point through the
 * pointers and the fp32 dequantized (rotated-domain) values through yhat. */
typedef struct {
    float amax, mn, mx;   /* of y over the unit */
    float S;              /* NV tensor scale */
} unit_range;

static void quant_unit(const scheme* s, const float* y, int64_t n, unit_range ur,
                       unsigned* code, float* scale_out, float* zp_out, uint8_t* scale_code,
                       float* yhat)
{
    if (s->gran == G_MX) {
        int e = orc_ue8m0_exponent(ur.amax, s->qscale);
        *scale_code = (uint8_t)(e + 127);
        float p = (float)ldexp(1.0, -e);         /* exact power of two */
        float back = (float)ldexp(1.0, e);
        for (int64_t i = 0; i < n; i++) {
            float v = y[i] * p;
            float val;
            if (s->is_int) {
                int q = round_clamp(v, 0, s->qmin, s->qmax);
                code[i] = (unsigned)q & 0xFFu;
                val = (float)q;
            } else {
                code[i] = orc_fp_encode(s->fmt, v);
                val = (float)orc_fp_decode(s->fmt, code[i]);
            }
            yhat[i] = val * back;
        }
        return;
    }
    if (s->gran == G_NV) {
        float S = ur.S;
        float sbv = 0.0f;
        unsigned sbc = 0;
        if (S > 0.0f) {
            float sb32 = (ur.amax / s->qscale) / S;
            sbc = orc_fp_encode(F_E4M3, sb32);
            sbv = (float)orc_fp_decode(F_E4M3, sbc);
        }
        *scale_code = (uint8_t)sbc;
        float d = sbv * S;
        for (int64_t i = 0; i < n; i++) {
            if (!(d > 0.0f)) { code[i] = 0; yhat[i] = 0.0f; continue; }
            float v = y[i] / d;
            float val;
            if (s->is_int) {
                int q = round_clamp(v, 0, s->qmin, s->qmax);
                code[i] = (unsigned)q & 0xFu;
                val = (float)q;
            } else {
                code[i] = orc_fp_encode(s->fmt, v);
                val = (float)orc_fp_decode(s->fmt, code[i]);
            }
            float t = val * sbv;                 /* exact */
            yhat[i] = t * S;
        }
        return;
    }
    /* TENSOR / ROW / GROUP with an fp32 or fp16 scale */
    if (s->is_asym) {
        float mn = ur.mn < 0.0f ? ur.mn : 0.0f;
        float mx = ur.mx > 0.0f ? ur.mx : 0.0f;
        float s32 = (mx - mn) / s->qscale;
        if (s32 > FLT_MAX) s32 = FLT_MAX;          /* a range beyond fp32 saturates */
        float sc = store_scale(s32, s->sdt);
        int zp;
        if (sc > 0.0f) zp = round_clamp(-mn / sc, s->qmin, s->qmin, s->qmax);
        else zp = s->qmin;
        *scale_out = sc;
        *zp_out = (float)zp;
        for (int64_t i = 0; i < n; i++) {
            int q = sc > 0.0f ? round_clamp(y[i] / sc, zp, s->qmin, s->qmax) : zp;
            code[i] = (unsigned)q & (s->bits4 ? 0xFu : 0xFFu);
            yhat[i] = sc * (float)(q - zp);
        }
        return;
    }
    float s32 = ur.amax / s->qscale;
    float sc = store_scale(s32, s->sdt);
    *scale_out = sc;
    for (int64_t i = 0; i < n; i++) {
        if (!(sc > 0.0f)) { code[i] = 0; yhat[i] = 0.0f; continue; }
        float v = y[i] / sc;
        if (s->is_int) {
            int q = round_clamp(v, 0, s->qmin, s->qmax);
            code[i] = (unsigned)q & (s->bits4 ? 0xFu : 0xFFu);
            yhat[i] = (float)q * sc;
        } else {
            code[i] = orc_fp_encode(s->fmt, v);
            yhat[i] = (float)orc_fp_decode(s->fmt, code[i]) * sc;
        }
    }
}

static void range_of(const float* y, int64_t n, unit_range* ur)
{
    float amax = 0.0f, mn = y[0], mx = y[0];
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(y[i]);
        if (a > amax) amax = a;
        if (y[i] < mn) mn = y[i];
        if (y[i] > mx) mx = y[i];
    }
    ur->amax = amax; ur->mn = mn; ur->mx = mx;
}

/* stats[0] = sum (x - xhat)^2, stats[1] = sum x^2 (original domain, double),
 * stats[2] = sum of kappa over units, stats[3] = max kappa, stats[4] = units counted. */
static void kappa_add(double* st, float amax, const float* y, int64_t n)
{
    double ss = 0.0;
    for (int64_t i = 0; i < n; i++) ss += (double)y[i] * (double)y[i];
    if (ss > 0.0) {
        double k = (double)amax / sqrt(ss / (double)n);
        st[2] += k;
        if (k > st[3]) st[3] = k;
        st[4] += 1.0;
    }
}

/* 2-D tiles: the range of each TILE_ROWS x 128 tile (rows of the last tile row may be
 * fewer), then every element of the tile quantized with the tile's scale, exactly as a
 * unit of the other granularities; kappa per tile over all its elements. */
static int quantize_tile2d(const scheme* s, const uint16_t* x, int64_t rows, int64_t cols,
                           uint8_t* codes, void* scales, void* zps, double* stats)
{
    const int64_t tpr = cols / 128;
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    float* yh = (float*)malloc(sizeof(float) * (size_t)cols);
    unsigned* cd = (unsigned*)malloc(sizeof(unsigned) * (size_t)cols);
    unit_range* ur = (unit_range*)malloc(sizeof(unit_range) * (size_t)tpr);
    double* ss = (double*)malloc(sizeof(double) * (size_t)tpr);
    if (!y || !yh || !cd || !ur || !ss) { free(y); free(yh); free(cd); free(ur); free(ss); return -3; }
    for (int64_t r0 = 0; r0 < rows; r0 += TILE_ROWS) {
        const int64_t r1 = r0 + TILE_ROWS < rows ? r0 + TILE_ROWS : rows;
        for (int64_t u = 0; u < tpr; u++) { ss[u] = 0.0; ur[u].S = 0.0f; }
        for (int64_t r = r0; r < r1; r++) {
            load_row(x, r, cols, s->had, y);
            for (int64_t u = 0; u < tpr; u++) {
                unit_range t;
                range_of(y + u * 128, 128, &t);
                if (r == r0) ur[u] = t;
                else {
                    if (t.amax > ur[u].amax) ur[u].amax = t.amax;
                    if (t.mn < ur[u].mn) ur[u].mn = t.mn;
                    if (t.mx > ur[u].mx) ur[u].mx = t.mx;
                }
                for (int64_t j = 0; j < 128; j++) ss[u] += (double)y[u * 128 + j] * (double)y[u * 128 + j];
            }
        }
        for (int64_t r = r0; r < r1; r++) {
            load_row(x, r, cols, s->had, y);
            for (int64_t u = 0; u < tpr; u++) {
                float sc = 0.0f, zp = 0.0f;
                uint8_t scode = 0;
                quant_unit(s, y + u * 128, 128, ur[u], cd + u * 128, &sc, &zp, &scode, yh + u * 128);
                const int64_t si = (r0 / TILE_ROWS) * tpr + u;
                write_scale(scales, si, sc, s->sdt);
                if (s->is_asym && zps) write_scale(zps, si, zp, s->sdt);
            }
            for (int64_t j = 0; j < cols; j++) put_code(codes, r, cols, j, cd[j], s->bits4);
            if (s->had)
                for (int64_t j = 0; j < cols; j += 16) orc_fwht16(yh + j);
            if (stats)
                for (int64_t j = 0; j < cols; j++) {
                    double xv = (double)orc_bf16_to_f32(x[r * cols + j]);
                    double e = xv - (double)yh[j];
                    stats[0] += e * e;
                    stats[1] += xv * xv;
                }
        }
        if (stats)
            for (int64_t u = 0; u < tpr; u++)
                if (ss[u] > 0.0) {
                    double k = (double)ur[u].amax / sqrt(ss[u] / (double)((r1 - r0) * 128));
                    stats[2] += k;
                    if (k > stats[3]) stats[3] = k;
                    stats[4] += 1.0;
                }
    }
    free(y); free(yh); free(cd); free(ur); free(ss);
    return 0;
}

/*
 * Quantize x [rows, cols] (bf16 bits, row-major).
 * tensor_range: NULL, or {amax, min, max} of the whole (rotated) tensor when the
 * given rows are only part of it (per-tensor and NV schemes need it).
 * Outputs follow the library's layout: 8-bit codes [rows, cols]; 4-bit codes
 * [rows, cols/2] with element 2j in the low nibble; scales and zero points
 * row-major [rows, cols/unit] (one value for per-tensor; [ceil(rows/128), cols/128] for
 * 2-D tiles); tensor_scale[0] for NV.
 * Returns 0, or a negative value for an invalid scheme or shape.
 */
int orc_quantize(const uint16_t* x, int64_t rows, int64_t cols,
                 int fmt, int gran, int block, int scale_dtype, int hadamard,
                 const float* tensor_range,
                 uint8_t* codes, void* scales, void* zps, float* tensor_scale,
                 double* stats)
{
    scheme s;
    int rc = make_scheme(fmt, gran, block, scale_dtype, hadamard, cols, &s);
    if (rc) return rc;
    if (rows < 0) return -2;
    if (stats) for (int i = 0; i < 5; i++) stats[i] = 0.0;
    if (rows == 0) return 0;
    if (gran == G_TILE2D) return quantize_tile2d(&s, x, rows, cols, codes, scales, zps, stats);

    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    float* yh = (float*)malloc(sizeof(float) * (size_t)cols);
    unsigned* cd = (unsigned*)malloc(sizeof(unsigned) * (size_t)cols);
    if (!y || !yh || !cd) { free(y); free(yh); free(cd); return -3; }

    float tr[3];
    if (gran == G_TENSOR || gran == G_NV) {
        if (tensor_range) { tr[0] = tensor_range[0]; tr[1] = tensor_range[1]; tr[2] = tensor_range[2]; }
        else orc_tensor_range(x, rows, cols, s.had, tr);
    }
    float S = 0.0f;
    if (gran == G_NV) {
        S = tr[0] / (s.qscale * 448.0f);
        if (tensor_scale) tensor_scale[0] = S;
    }

    double ss_tensor = 0.0;
    int64_t unit = gran == G_TENSOR ? cols : s.unit;
    int64_t upr = cols / unit;                 /* units per row */

    for (int64_t r = 0; r < rows; r++) {
        load_row(x, r, cols, s.had, y);
        for (int64_t u = 0; u < upr; u++) {
            const float* yu = y + u * unit;
            unit_range ur;
            if (gran == G_TENSOR) { ur.amax = tr[0]; ur.mn = tr[1]; ur.mx = tr[2]; }
            else range_of(yu, unit, &ur);
            ur.S = S;
            float sc = 0.0f, zp = 0.0f;
            uint8_t scode = 0;
            quant_unit(&s, yu, unit, ur, cd + u * unit, &sc, &zp, &scode, yh + u * unit);
            int64_t si = gran == G_TENSOR ? 0 : r * upr + u;
            if (gran == G_MX || gran == G_NV) ((uint8_t*)scales)[si] = scode;
            else {
                write_scale(scales, si, sc, s.sdt);
                if (s.is_asym && zps) write_scale(zps, si, zp, s.sdt);
            }
            if (stats) {
                if (gran == G_TENSOR) {
                    for (int64_t i = 0; i < unit; i++) ss_tensor += (double)yu[i] * (double)yu[i];
                } else {
                    kappa_add(stats, ur.amax, yu, unit);
                }
            }
        }
        for (int64_t j = 0; j < cols; j++) put_code(codes, r, cols, j, cd[j], s.bits4);
        if (s.had)
            for (int64_t j = 0; j < cols; j += 16) orc_fwht16(yh + j);
        if (stats)
            for (int64_t j = 0; j < cols; j++) {
                double xv = (double)orc_bf16_to_f32(x[r * cols + j]);
                double e = xv - (double)yh[j];
                stats[0] += e * e;
                stats[1] += xv * xv;
            }
    }
    if (stats && gran == G_TENSOR && ss_tensor > 0.0) {
        double n = (double)rows * (double)cols;
        double k = (double)tr[0] / sqrt(ss_tensor / n);
        stats[2] = k; stats[3] = k; stats[4] = 1.0;
    }
    free(y); free(yh); free(cd);
    return 0;
}

/* Dequantize codes [rows, ...] into fp32 out [rows, cols] (inverse rotation applied
 * when the scheme has hadamard set). */
int orc_dequantize(const uint8_t* codes, const void* scales, const void* zps,
                   const float* tensor_scale, int64_t rows, int64_t cols,
                   int fmt, int gran, int block, int scale_dtype, int hadamard,
                   float* out)
{
    scheme s;
    int rc = make_scheme(fmt, gran, block, scale_dtype, hadamard, cols, &s);
    if (rc) return rc;
    if (rows < 0) return -2;
    int64_t unit = gran == G_TENSOR ? cols : s.unit;
    int64_t upr = cols / unit;
    float S = gran == G_NV ? tensor_scale[0] : 0.0f;
    for (int64_t r = 0; r < rows; r++) {
        float* o = out + r * cols;
        for (int64_t j = 0; j < cols; j++) {
            int64_t u = j / unit;
            int64_t si = scale_index(gran, r, u, upr);
            unsigned c = get_code(codes, r, cols, j, s.bits4);
            float v;
            if (gran == G_MX) {
                int e = (int)((const uint8_t*)scales)[si] - 127;
                float val = s.is_int ? (float)int_of_code(c, 0, 0) : (float)orc_fp_decode(s.fmt, c);
                v = val * (float)ldexp(1.0, e);
            } else if (gran == G_NV) {
                float sbv = (float)orc_fp_decode(F_E4M3, ((const uint8_t*)scales)[si]);
                float val = s.is_int ? (float)int_of_code(c, 1, 0) : (float)orc_fp_decode(s.fmt, c);
                float t = val * sbv;
                v = t * S;
            } else {
                float sc = read_scale(scales, si, s.sdt);
                if (s.is_int) {
                    int q = int_of_code(c, s.bits4, s.fmt == F_UINT4_ASYM);
                    if (s.is_asym) {
                        int zp = (int)read_scale(zps, si, s.sdt);
                        v = sc * (float)(q - zp);
                    } else {
                        v = (float)q * sc;
                    }
                } else {
                    v = (float)orc_fp_decode(s.fmt, c) * sc;
                }
            }
            o[j] = v;
        }
        if (s.had)
            for (int64_t j = 0; j < cols; j += 16) orc_fwht16(o + j);
    }
    return 0;
}

/* QSNR sums of x against the dequantized codes: stats[0] = sum (x - xhat)^2,
 * stats[1] = sum x^2; the kappa fields are left at zero. */
int orc_qsnr_sums(const uint16_t* x, const uint8_t* codes, const void* scales, const void* zps,
                  const float* tensor_scale, int64_t rows, int64_t cols,
                  int fmt, int gran, int block, int scale_dtype, int hadamard,
                  double* stats)
{
    scheme s;
    int rc = make_scheme(fmt, gran, block, scale_dtype, hadamard, cols, &s);
    if (rc) return rc;
    for (int i = 0; i < 5; i++) stats[i] = 0.0;
    float* o = (float*)malloc(sizeof(float) * (size_t)cols);
    if (!o) return -3;
    int64_t cb = s.bits4 ? cols / 2 : cols;
    int64_t unit = gran == G_TENSOR ? cols : s.unit;
    int64_t upr = cols / unit;
    size_t sz = (gran == G_MX || gran == G_NV) ? 1 : (scale_dtype == SD_FP16 ? 2 : 4);
    for (int64_t r = 0; r < rows; r++) {
        const uint8_t* cr = codes + r * cb;
        /* the row's scales: dequantize sees a one-row tensor (a 2-D tile row's scales
         * serve every row of that tile row) */
        const int64_t off = gran == G_TENSOR ? 0 : gran == G_TILE2D ? (r / TILE_ROWS) * upr : r * upr;
        const char* sr = (const char*)scales + (size_t)off * sz;
        const char* zr = !zps ? NULL : (const char*)zps + (size_t)off * sz;
        rc = orc_dequantize(cr, sr, zr, tensor_scale, 1, cols, fmt, gran, block, scale_dtype, hadamard, o);
        if (rc) { free(o); return rc; }
        for (int64_t j = 0; j < cols; j++) {
            double xv = (double)orc_bf16_to_f32(x[r * cols + j]);
            double e = xv - (double)o[j];
            stats[0] += e * e;
            stats[1] += xv * xv;
        }
    }
    free(o);
    return 0;
}

/* QSNR in dB from the two sums: -10 log10(err2 / x2). */
double orc_qsnr_db(double err2, double x2)
{
    return -10.0 * log10(err2 / x2);
}

/* Bytes of codes, scales, zero points and tensor scale for a scheme and shape. */
int orc_buffer_sizes(int fmt, int gran, int block, int scale_dtype, int hadamard,
                     int64_t rows, int64_t cols, int64_t* out4)
{
    scheme s;
    int rc = make_scheme(fmt, gran, block, scale_dtype, hadamard, cols, &s);
    if (rc) return rc;
    int64_t n = rows * cols;
    int64_t nscale = gran == G_TENSOR ? 1 : gran == G_TILE2D ? ((rows + TILE_ROWS - 1) / TILE_ROWS) * (cols / s.unit)
                                                               : rows * (cols / s.unit);
    int64_t ssz = (gran == G_MX || gran == G_NV) ? 1 : (scale_dtype == SD_FP16 ? 2 : 4);
    out4[0] = s.bits4 ? n / 2 : n;
    out4[1] = nscale * ssz;
    out4[2] = s.is_asym ? nscale * ssz : 0;
    out4[3] = gran == G_NV ? 4 : 0;
    return 0;
}

/* Elementwise fp32 -> bf16 (round to nearest even) over an array. */
void orc_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_f32_to_bf16(in[i]);
}

/* ------------------------------------------------------------------------- */
/* Row transforms before quantizing: SmoothQuant's per-channel factor          */
/* ("Quantization survey" §3.2 and §5.2: W * s per input channel) and QuaRot's */
/* randomized Hadamard rotation of the whole row (same page §5.3: an           */
/* orthogonal +-1 rotation, R^T R = I, spreads outlier channels over all).     */
/*                                                                            */
/* Readings: x' = RN(x * m_j) with m the caller's per-column factor; the       */
/* rotation is y = (x' * sigma) H_n c with sigma_j = -1 where the caller's     */
/* sign byte is set, H_n the Sylvester-order Walsh-Hadamard matrix (n = cols,  */
/* a power of two), taken as stages h = 1, 2, ..., n/2 of (a + b, a - b), and  */
/* c = the fp32 value nearest 1/sqrt(n); dequantize applies the inverse        */
/* (the same stages, * c, then the signs) and returns x' (the factor stays:    */
/* the operand a GEMM would take); QSNR compares x' with that.                 */
/* ------------------------------------------------------------------------- */

/* Walsh-Hadamard transform (unnormalised) of n = 2^m values in place. */
void orc_fwht(float* v, int64_t n)
{
    for (int64_t h = 1; h < n; h *= 2)
        for (int64_t i = 0; i < n; i += 2 * h)
            for (int64_t k = i; k < i + h; k++) {
                float a = v[k], b = v[k + h];
                v[k] = a + b;
                v[k + h] = a - b;
            }
}

static float rot_norm(int64_t n) { return (float)(1.0 / sqrt((double)n)); }

static int pow2_in(int64_t n, int64_t lo, int64_t hi) { return n >= lo && n <= hi && (n & (n - 1)) == 0; }

/* One row: xs = x' (pre-scaled), y = rotated (or x' when signs is NULL). */
static void rt_forward(const uint16_t* xrow, int64_t n, const float* col_scale, const uint8_t* signs,
                       float* xs, float* y)
{
    for (int64_t j = 0; j < n; j++) {
        float v = orc_bf16_to_f32(xrow[j]);
        if (col_scale) v = v * col_scale[j];
        xs[j] = v;
        y[j] = (signs && signs[j]) ? -v : v;
    }
    if (signs) {
        const float c = rot_norm(n);
        orc_fwht(y, n);
        for (int64_t j = 0; j < n; j++) y[j] = y[j] * c;
    }
}

static void rt_inverse(float* v, int64_t n, const uint8_t* signs)
{
    if (!signs) return;
    const float c = rot_norm(n);
    orc_fwht(v, n);
    for (int64_t j = 0; j < n; j++) {
        v[j] = v[j] * c;
        if (signs[j]) v[j] = -v[j];
    }
}

static int rt_check(const scheme* s, int gran, int64_t cols, const uint8_t* signs)
{
    if (!(gran == G_ROW || gran == G_GROUP || gran == G_MX)) return -1;
    if (s->had) return -1;
    if (signs && !pow2_in(cols, 16, 16384)) return -2;
    return 0;
}

/* The transformed rows' fp32 values (x' rotated), [rows, cols]. */
int orc_rotate_rows(const uint16_t* x, int64_t rows, int64_t cols, const float* col_scale,
                    const uint8_t* signs, float* out)
{
    if (rows < 0 || cols <= 0) return -2;
    if (signs && !pow2_in(cols, 16, 16384)) return -2;
    float* xs = (float*)malloc(sizeof(float) * (size_t)cols);
    if (!xs) return -3;
    for (int64_t r = 0; r < rows; r++) rt_forward(x + r * cols, cols, col_scale, signs, xs, out + r * cols);
    free(xs);
    return 0;
}

/*
 * Quantize x [rows, cols] after the row transforms (col_scale: NULL or [cols];
 * signs: NULL for no rotation, else [cols] bytes, nonzero = -1). Per-row, per-group
 * and MX schemes without the block-16 Hadamard. Outputs as orc_quantize; stats:
 * err2 and x2 against x' in the original (unrotated) domain, kappa over the units'
 * rotated values.
 */
int orc_quantize_rt(const uint16_t* x, int64_t rows, int64_t cols,
                    int fmt, int gran, int block, int scale_dtype,
                    const float* col_scale, const uint8_t* signs,
                    uint8_t* codes, void* scales, void* zps, double* stats)
{
    scheme s;
    int rc = make_scheme(fmt, gran, block, scale_dtype, 0, cols, &s);
    if (rc) return rc;
    rc = rt_check(&s, gran, cols, signs);
    if (rc) return rc;
    if (rows < 0) return -2;
    if (stats) for (int i = 0; i < 5; i++) stats[i] = 0.0;
    const int64_t unit = s.unit, upr = cols / unit;
    float* xs = (float*)malloc(sizeof(float) * (size_t)cols);
    float* y = (float*)malloc(sizeof(float) * (size_t)cols);
    float* yh = (float*)malloc(sizeof(float) * (size_t)cols);
    unsigned* cd = (unsigned*)malloc(sizeof(unsigned) * (size_t)cols);
    if (!xs || !y || !yh || !cd) { free(xs); free(y); free(yh); free(cd); return -3; }
    for (int64_t r = 0; r < rows; r++) {
        rt_forward(x + r * cols, cols, col_scale, signs, xs, y);
        for (int64_t u = 0; u < upr; u++) {
            unit_range ur;
            range_of(y + u * unit, unit, &ur);
            ur.S = 0.0f;
            float sc = 0.0f, zp = 0.0f;
            uint8_t scode = 0;
            quant_unit(&s, y + u * unit, unit, ur, cd + u * unit, &sc, &zp, &scode, yh + u * unit);
            const int64_t si = r * upr + u;
            if (gran == G_MX) ((uint8_t*)scales)[si] = scode;
            else {
                write_scale(scales, si, sc, s.sdt);
                if (s.is_asym && zps) write_scale(zps, si, zp, s.sdt);
            }
            if (stats) kappa_add(stats, ur.amax, y + u * unit, unit);
        }
        for (int64_t j = 0; j < cols; j++) put_code(codes, r, cols, j, cd[j], s.bits4);
        rt_inverse(yh, cols, signs);
        if (stats)
            for (int64_t j = 0; j < cols; j++) {
                double e = (double)xs[j] - (double)yh[j];
                stats[0] += e * e;
                stats[1] += (double)xs[j] * (double)xs[j];
            }
    }
    free(xs); free(y); free(yh); free(cd);
    return 0;
}

/* Dequantize codes written by orc_quantize_rt: x-hat' [rows, cols] (the inverse
 * rotation applied; the per-column factor kept). */
int orc_dequantize_rt(const uint8_t* codes, const void* scales, const void* zps,
                      int64_t rows, int64_t cols, int fmt, int gran, int block, int scale_dtype,
                      const uint8_t* signs, float* out)
{
    scheme s;
    int rc = make_scheme(fmt, gran, block, scale_dtype, 0, cols, &s);
    if (rc) return rc;
    rc = rt_check(&s, gran, cols, signs);
    if (rc) return rc;
    rc = orc_dequantize(codes, scales, zps, NULL, rows, cols, fmt, gran, block, scale_dtype, 0, out);
    if (rc) return rc;
    for (int64_t r = 0; r < rows; r++) rt_inverse(out + r * cols, cols, signs);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Block-scale factors in the layout a block-scaled GEMM reads them in          */
/* ("Quantization survey" §4.3 and the MX/NV recipes: the consumer of the     */
/* codes is a tensor-core GEMM that scales each 1 x 32 (MX) or 1 x 16 (NV)   */
/* block). Reading (the scale-factor layout of NVIDIA's block-scaled MMA and  */
/* its libraries): the scale matrix [rows, nb] (nb blocks per row) is padded   */
/* to [ceil(rows/128) * 128, ceil(nb/4) * 4] and cut into 128 x 4 tiles of    */
/* 512 bytes, tiles in row-major order; inside a tile, entry (r, c) sits at   */
/* byte (r % 32) * 16 + (r / 32) * 4 + c. Padding bytes are not written.      */
/* ------------------------------------------------------------------------- */

int64_t orc_gemm_scale_offset(int64_t r, int64_t c, int64_t nb)
{
    const int64_t tiles_per_row = (nb + 3) / 4;
    const int64_t tile = (r / 128) * tiles_per_row + c / 4;
    const int64_t rr = r % 128;
    return tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (c % 4);
}

int64_t orc_gemm_scale_bytes(int64_t rows, int64_t nb)
{
    return ((rows + 127) / 128) * 128 * ((nb + 3) / 4) * 4;
}

/* Row-major [rows, nb] scale bytes to the GEMM layout (out has
 * orc_gemm_scale_bytes(rows, nb) bytes; padding left as it was). */
void orc_scales_to_gemm(const uint8_t* in, int64_t rows, int64_t nb, uint8_t* out)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < nb; c++) out[orc_gemm_scale_offset(r, c, nb)] = in[r * nb + c];
}

/* And back. */
void orc_scales_from_gemm(const uint8_t* in, int64_t rows, int64_t nb, uint8_t* out)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < nb; c++) out[r * nb + c] = in[orc_gemm_scale_offset(r, c, nb)];
}
