/*
 * bq.h -- C ABI of the block-scaled tensor quantization library (libbq.so).
 *
 * One NVIDIA B200 (sm_100a). Every entry point takes plain pointers and sizes; all
 * tensors are caller-owned device memory unless a parameter says "host". Work is
 * enqueued on the caller's CUDA stream (passed as void*, a cudaStream_t; NULL is the
 * legacy default stream) and results are valid after the caller synchronizes that
 * stream. No entry point allocates device memory, throws, or falls back to the CPU.
 * Argument, shape and alignment checks run on the host before any launch; a failed
 * check launches nothing. A launch failure returns BQ_ERR_CUDA. The quantize, dequantize
 * and QSNR kernels are launched with programmatic stream serialization (programmatic
 * dependent launch): a kernel may become resident while the work ahead of it in the
 * stream is finishing, but it reads and writes no memory before that work has completed,
 * so ordinary stream order holds, in eager use and inside CUDA graphs.
 *
 * Method (source pages cited by title and section):
 *  - AbsMax scale s = max|X| / Qmax and Xq = clip(round(X/s), Qmin, Qmax) * s:
 *    "INT vs FP at fine granularity" §2.1; granularity per tensor / per channel /
 *    per block: same page §3.1.
 *  - Affine INT: q = round(w/scale) + zero_point, w = scale * (q - zero_point):
 *    "INT4/INT8/FP8 quantization" §INT8; INT4 [-8, 7] groups, two codes per byte:
 *    same page §INT4; E4M3 +-448, E5M2 +-57344: same page §FP8.
 *  - FP element formats E2M1 / E4M3 / E5M2 / FP6 E2M3 / FP6 E3M2 and their bit layouts:
 *    "Quantization survey" §4.1 (FP6 biases 1 and 3 follow that table's ranges +-7.5
 *    and +-28; its printed smallest values contradict them); the MX family, MXFP6
 *    included: same page §4.3; MX (block 32, power-of-two E8M0 scale) and NV (block 16, E4M3
 *    block scale plus an FP32 tensor scale, x = x_q * s_block * S_tensor): same page
 *    §4.3.1 and §4.3.2.
 *  - Hadamard rotation before quantizing: "INT vs FP at fine granularity" §4.2 and
 *    §7.2; orthogonal rotation R^T R = I: "Quantization survey" §5.3.
 *  - QSNR = -10 log10(||X - Xq||^2 / ||X||^2) and the crest factor kappa:
 *    "INT vs FP at fine granularity" §4.1.
 *
 * Arithmetic contract (bit-exact with the library's CPU oracle):
 *  - inputs are bf16, widened exactly to fp32; scales and quotients are fp32;
 *  - every code is decided from the correctly rounded fp32 quotient x / s (round half
 *    to even for INT, round-to-nearest-even with saturation to the largest finite
 *    value for FP element formats; the sign of an FP zero is kept);
 *  - the quantizer divides by the scale as stored (an fp16 scale is rounded first,
 *    saturating at 65504);
 *  - asymmetric INT: min' = min(min, 0), max' = max(max, 0), s = (max' - min') / L
 *    (L = 255 or 15), zp = clamp(Qmin + round(-min'/s)), q = clamp(round(x/s) + zp);
 *  - MX: the scale exponent e is the smallest integer with amax <= Qmax * 2^e,
 *    clamped to [-127, 127] (amax = 0 gives -127), stored as e + 127;
 *  - NV: S = A / (Qmax * 448) over the whole tensor; s_b = E4M3((amax_b / Qmax) / S);
 *    d = s_b * S; code = enc(x / d), zero codes where d = 0; dequant (code * s_b) * S;
 *  - Hadamard: each run of 16 elements along a row is replaced by H16 x / 4
 *    (Sylvester order, butterfly stages h = 1, 2, 4, 8 of (a+b, a-b), then * 0.25);
 *    the per-tensor range is taken on rotated values; dequantize applies the same
 *    transform again (it is its own inverse). Rotated schemes take inputs with
 *    |x| <= 2^125 (the rotated values then stay finite); larger inputs, and NaN or
 *    Inf inputs for any scheme, give unspecified codes.
 *
 * Layouts (row-major, rows x cols input):
 *  - codes: 8-bit formats uint8 [rows, cols]; 4-bit formats uint8 [rows, cols/2], element
 *    2j in the low nibble of byte j; FP6 formats one code per byte [rows, cols] (the low
 *    six bits, sign at bit 5); INT codes are two's complement (UINT4 unsigned);
 *  - scales: per tensor 1 value; per row [rows]; per group [rows, cols/block]; 2-D
 *    tiles [ceil(rows/128), cols/128] (tile (i, j) covers rows 128i.., columns 128j..);
 *    MX uint8 [rows, cols/32] (UE8M0 codes); NV uint8 [rows, cols/16] (E4M3 codes);
 *    MX / NV with scale_layout = BQ_LAYOUT_GEMM: the GEMM tile layout below;
 *    fp32 or fp16 as scheme.scale_dtype says for the first four;
 *  - zero points (asymmetric formats only): same shape and dtype as the scales,
 *    holding exact integers;
 *  - tensor_scale: one fp32 (NV only).
 *
 * Shapes: rows >= 0, cols > 0, cols % 16 == 0 (and cols % block == 0); rows * cols <=
 * 2^36 - 2048. rows == 0 is a valid empty call. Alignment: x, codes and out 32-byte aligned;
 * scales, zero points and the tensor scale 4-byte aligned.
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bq_status {
    BQ_OK = 0,
    BQ_ERR_INVALID_ARG = 1,   /* null pointer where one is required, bad enum value */
    BQ_ERR_UNSUPPORTED = 2,   /* format x granularity x scale dtype not offered */
    BQ_ERR_SHAPE = 3,         /* negative rows, cols not a multiple of 16 / block, too large */
    BQ_ERR_ALIGNMENT = 4,     /* x, codes or out not 32-byte aligned, or a scale buffer not 4-byte aligned */
    BQ_ERR_WORKSPACE = 5,     /* workspace missing or smaller than bq_workspace_size() */
    BQ_ERR_CUDA = 6           /* a CUDA call failed (see cudaGetLastError on the caller side) */
} bq_status;

/* data and scale dtypes */
enum { BQ_DT_BF16 = 0, BQ_DT_FP16 = 1, BQ_DT_FP32 = 2, BQ_DT_UE8M0 = 3, BQ_DT_E4M3 = 4 };

/* element formats */
enum {
    BQ_INT8_SYM = 0,     /* [-127, 127], s = amax / 127                        */
    BQ_INT8_ASYM = 1,    /* [-128, 127] with zero point, 255 levels            */
    BQ_INT4_SYM = 2,     /* [-8, 7], s = amax / 7 ([-7, 7] under NV: NVINT4)   */
    BQ_UINT4_ASYM = 3,   /* [0, 15] with zero point, 15 levels                 */
    BQ_FP8_E4M3 = 4,     /* +-448                                              */
    BQ_FP8_E5M2 = 5,     /* +-57344                                            */
    BQ_FP4_E2M1 = 6,     /* +-6 (MX or NV granularity only)                    */
    BQ_FP6_E2M3 = 7,     /* FP6 +-7.5, exponent bias 1 (MX granularity only)   */
    BQ_FP6_E3M2 = 8      /* FP6 +-28, exponent bias 3 (MX granularity only)    */
};

/* scaling granularity */
enum {
    BQ_PER_TENSOR = 0,   /* one scale; per-tensor range pass first (needs a workspace) */
    BQ_PER_ROW = 1,      /* one scale per row (output channel of a weight, or token)   */
    BQ_PER_GROUP = 2,    /* block in {16, 32, 64, 128, 256, 512} contiguous along a row */
    BQ_MX_BLOCK = 3,     /* block 32, UE8M0 scale: INT8_SYM, E4M3, E5M2, E2M1, E2M3, E3M2 */
    BQ_NV_BLOCK = 4,     /* block 16, E4M3 scale + fp32 tensor scale: E2M1, INT4_SYM    */
    BQ_TILE_2D = 5       /* one scale per 128 x 128 tile (block 128; the last tile row  */
                         /* may hold fewer rows), fp32 or fp16: every format but FP4 /  */
                         /* FP6; cols % 128 == 0 ("Quantization survey" §4.4, the       */
                         /* DeepSeek-V3 weight tiles)                                    */
};

typedef struct bq_scheme {
    int32_t format;       /* BQ_INT8_SYM ...                                     */
    int32_t granularity;  /* BQ_PER_TENSOR ...                                   */
    int32_t block;        /* group size for BQ_PER_GROUP; 32 for MX, 16 for NV;  */
                          /* 128 (or 0) for BQ_TILE_2D;                          */
                          /* ignored (0) for per-tensor / per-row                */
    int32_t scale_dtype;  /* BQ_DT_FP32 or BQ_DT_FP16 (tensor/row/group),        */
                          /* BQ_DT_UE8M0 (MX), BQ_DT_E4M3 (NV)                    */
    int32_t hadamard;     /* 0 or 1: rotate each 16-run by H16/4 before scaling  */
    int32_t scale_layout; /* BQ_LAYOUT_ROWS (0) or BQ_LAYOUT_GEMM (1, MX / NV)   */
} bq_scheme;

/* Layout of the MX / NV block scales (scale_layout):
 *  - BQ_LAYOUT_ROWS: row-major [rows, nb] bytes (nb = cols / 32 for MX, cols / 16 for NV);
 *  - BQ_LAYOUT_GEMM: the layout a block-scaled tensor-core GEMM reads its scale factors
 *    in, so the codes and scales go to the GEMM as they are (the scale-factor layout of
 *    NVIDIA's block-scaled MMA and its libraries, e.g. cuBLASLt's and torch's 32x4x4
 *    swizzle): the matrix padded to [ceil(rows / 128) * 128, nb] and cut into 128 x 4
 *    tiles of 512 bytes in row-major tile order; entry (r, c) of a tile sits at byte
 *    (r % 32) * 16 + (r / 32) * 4 + c. Needs cols % 128 == 0 (nb a multiple of 4) and
 *    fewer than 2^32 padded scale bytes (else BQ_ERR_SHAPE);
 *    padding bytes (rows past the last) are not written. Dequantize and QSNR read the
 *    same layout. Other granularities: BQ_ERR_UNSUPPORTED. */
enum { BQ_LAYOUT_ROWS = 0, BQ_LAYOUT_GEMM = 1 };

/* QSNR and crest-factor sums, written by the library into caller device memory.
 * err2 = sum (x - xhat)^2 and x2 = sum x^2 over the whole tensor (original domain);
 * kappa_* over the scaling units (block, group, row, 2-D tile, or the tensor), each unit's
 * kappa = amax / sqrt(mean of squares) of the values it quantizes (rotated values
 * when hadamard = 1); units whose sum of squares is zero are not counted. */
typedef struct bq_stats {
    double err2;
    double x2;
    double kappa_sum;
    double kappa_max;
    double n_units;       /* an exact integer */
} bq_stats;

/* A readable name for a status code (static storage; never NULL). */
const char* bq_status_string(int status);

/* Library version string (static storage). */
const char* bq_version(void);

/* Byte sizes of the four outputs of bq_quantize for this scheme and shape (host
 * pointers; any may be NULL). Zero-point and tensor-scale sizes are 0 when the
 * scheme has none. Validates the scheme and shape like bq_quantize. */
bq_status bq_buffer_sizes(const bq_scheme* scheme, int64_t rows, int64_t cols,
                          size_t* code_bytes, size_t* scale_bytes,
                          size_t* zero_point_bytes, size_t* tensor_scale_bytes);

/* Device workspace needed by bq_quantize / bq_qsnr for this scheme and shape (host
 * pointer out). It is 0 when the call needs none (no stats and not per-tensor or NV).
 * The workspace holds the cross-CTA partial sums and the per-tensor range; it must be
 * zero-filled once after allocation (the library leaves its counters at zero after
 * every call) and must not be used by two calls that can run at the same time. */
bq_status bq_workspace_size(const bq_scheme* scheme, int64_t rows, int64_t cols,
                            int with_stats, size_t* bytes);

/*
 * Quantize x [rows, cols] (device, dtype x_dtype = BQ_DT_BF16) into codes, scales,
 * zero_points (asymmetric formats; else may be NULL) and tensor_scale (NV; else may
 * be NULL), all device buffers of the sizes bq_buffer_sizes gives.
 * stats (device, may be NULL): when given, the QSNR and kappa sums of this call are
 * written there, reduced in a fixed order (bit-reproducible on a given GPU).
 * workspace / workspace_bytes: device scratch of at least bq_workspace_size() bytes
 * (NULL / 0 when that size is 0).
 * Per-tensor and NV schemes take two passes over x (range, then quantize); all other
 * schemes take one.
 */
bq_status bq_quantize(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                      const bq_scheme* scheme,
                      void* codes, void* scales, void* zero_points, float* tensor_scale,
                      bq_stats* stats, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * The two passes of a per-tensor or NV scheme, as separate calls.
 *
 * bq_tensor_range: the range pass alone ("max calibration": the tensor's largest
 * magnitude maps to the format's largest value, "2025 H2 quantization trends" §三;
 * AbsMax, "INT vs FP at fine granularity" §2.1). Writes range[0] = amax = max |y|,
 * range[1] = min(min y, 0) and range[2] = max(max y, 0) of the tensor's values y (each
 * 16-run rotated by H16/4 first when scheme->hadamard is set); the last two only for
 * asymmetric formats under BQ_PER_TENSOR (else 0). range: device fp32 [3], 4-byte
 * aligned. Needs a workspace of bq_workspace_size() bytes (its header holds the
 * cross-CTA hand-off). rows == 0 writes zeros.
 *
 * bq_quantize_with_range: the quantize pass alone, against range = {amax, min, max}
 * (device fp32 [3]; min and max are used as min(min, 0) and max(max, 0)), e.g. from
 * bq_tensor_range on this tensor (bq_tensor_range then bq_quantize_with_range gives
 * exactly bq_quantize's results), from an earlier calibration (static scales), or
 * combined over the row blocks of a tensor split across GPUs (MAX of amax and of max,
 * MIN of min). Outputs, stats and alignment as bq_quantize; the workspace is needed only
 * with stats (NULL / 0 otherwise).
 *
 * Both: per-tensor and NV schemes only (else BQ_ERR_UNSUPPORTED); a NULL range gives
 * BQ_ERR_INVALID_ARG.
 */
bq_status bq_tensor_range(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                          const bq_scheme* scheme, float* range,
                          void* workspace, size_t workspace_bytes, void* stream);

bq_status bq_quantize_with_range(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                 const bq_scheme* scheme, const float* range,
                                 void* codes, void* scales, void* zero_points, float* tensor_scale,
                                 bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream);

/*
 * A batch of same-shape tensors in one call: x is [batch, rows, cols] bf16, contiguous;
 * tensor b is quantized exactly as bq_quantize would quantize it alone (the same codes,
 * scales and zero points), with its QSNR and kappa sums in stats[b] (device, [batch],
 * or NULL). The experiment of "INT vs FP at fine granularity" §4.2 compares formats on
 * thousands of weight tensors of one model; a batch serves such sets (e.g. all FFN
 * weights of a layer type) with one launch instead of one per tensor.
 * Outputs: codes [batch, rows, cols] (4-bit formats [batch, rows, cols / 2]), scales and
 * zero points [batch] x the one-tensor size (bq_buffer_sizes(rows, cols) each), tensor b's
 * at b times that size. Schemes: per-group and MX (either scale layout), and per-row
 * schemes with cols a power-of-two multiple of 64 up to 2048, each with or without the
 * block-16 rotation (else BQ_ERR_UNSUPPORTED: per-tensor and NV schemes need a range
 * per tensor first, use bq_quantize per tensor). batch > 1 needs rows * cols % 64 == 0,
 * and rows % 128 == 0 for scale_layout = BQ_LAYOUT_GEMM (else BQ_ERR_SHAPE). The stats
 * of a tensor are reduced in a fixed order, bit-reproducible for a given batch size on a
 * given GPU (the order differs from a one-tensor call's: the sums agree to rounding).
 * workspace: bq_workspace_size() bytes when stats is given (it does not grow with the
 * batch). batch == 0 does nothing. Alignment as bq_quantize.
 */
bq_status bq_quantize_batch(const void* x, int32_t x_dtype, int64_t batch, int64_t rows, int64_t cols,
                            const bq_scheme* scheme, void* codes, void* scales, void* zero_points,
                            bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dequantize codes (+ scales, zero_points, tensor_scale as written by bq_quantize)
 * into out [rows, cols] (device) of dtype out_dtype = BQ_DT_BF16 (round to nearest
 * even from the fp32 value) or BQ_DT_FP32. Applies the inverse rotation when
 * scheme->hadamard is set. One pass; needs no workspace.
 */
bq_status bq_dequantize(const void* codes, const void* scales, const void* zero_points,
                        const float* tensor_scale, int64_t rows, int64_t cols,
                        const bq_scheme* scheme, void* out, int32_t out_dtype,
                        void* stream);

/*
 * QSNR sums of x against the dequantized codes, computed in one pass without writing
 * the dequantized tensor: stats->err2 and stats->x2 (original domain); the kappa
 * fields are written as zero. Needs a workspace of bq_workspace_size(..., 1, ...).
 */
bq_status bq_qsnr(const void* x, int32_t x_dtype, const void* codes, const void* scales,
                  const void* zero_points, const float* tensor_scale,
                  int64_t rows, int64_t cols, const bq_scheme* scheme,
                  bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Row transforms applied before quantizing ("Quantization survey" §3.2 and §5.2:
 * SmoothQuant's per-channel factor; §5.3: QuaRot's randomized Hadamard rotation, an
 * orthogonal R with R^T R = I that spreads outlier channels over the whole row).
 *  - col_scale (device fp32 [cols], 16-byte aligned, or NULL): x'[i][j] = RN(x[i][j] *
 *    col_scale[j]), e.g. SmoothQuant's 1/s on activations or s on weights;
 *  - sign_bits (device uint32 [cols / 32], 4-byte aligned, or NULL for no rotation):
 *    y = (x' * sigma) H c per row, sigma[j] = -1 where bit j % 32 of word j / 32 is set,
 *    H the cols-point Walsh-Hadamard matrix in Sylvester order (taken as stages
 *    h = 1, 2, ..., cols/2 of (a + b, a - b)), c = the fp32 value nearest 1/sqrt(cols).
 *  - reserved: must be 0.
 * The arrays are read only (caller-owned).
 */
typedef struct bq_row_transform {
    const float* col_scale;
    const uint32_t* sign_bits;
    int64_t reserved;
} bq_row_transform;

/*
 * bq_quantize after the row transforms rt (may be NULL: none). Per-row, per-group and
 * MX schemes with hadamard = 0 (else BQ_ERR_UNSUPPORTED); cols a multiple of 512 up to
 * 16384, a power of two when rotating (else BQ_ERR_SHAPE). The codes, scales and zero
 * points are those of the transformed rows. stats (may be NULL; needs a workspace of
 * bq_workspace_size(..., 1, ...) bytes) holds err2 and x2 summed on the rotated values
 * (equal to the sums against x' up to fp32 rounding: the rotation is orthogonal) and
 * kappa over the units' rotated values. One pass over x; a CTA per row at a time.
 * Pointers and alignment as bq_quantize (tensor_scale is not used), plus the arrays'
 * alignment above (BQ_ERR_ALIGNMENT); rt->reserved != 0 gives BQ_ERR_INVALID_ARG. MX
 * scales may take scale_layout = BQ_LAYOUT_GEMM.
 */
bq_status bq_quantize_rt(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                         const bq_scheme* scheme, const bq_row_transform* rt,
                         void* codes, void* scales, void* zero_points,
                         bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dequantize codes written by bq_quantize_rt into out [rows, cols] (BQ_DT_BF16 or
 * BQ_DT_FP32): the element values, then the inverse rotation (the same stages, times c,
 * then the signs) when rt->sign_bits is given. The per-column factor is not undone:
 * out estimates x' (the operand a GEMM with the inverse factor on the other side
 * takes). Shapes and schemes as bq_quantize_rt.
 */
bq_status bq_dequantize_rt(const void* codes, const void* scales, const void* zero_points,
                           int64_t rows, int64_t cols, const bq_scheme* scheme,
                           const bq_row_transform* rt, void* out, int32_t out_dtype, void* stream);

/*
 * bq_quantize without a caller-provided workspace, for callers that cannot allocate
 * device memory: code running under another component's allocator (a framework or
 * serving runtime that owns all device memory), code that must not call cudaMalloc
 * in the middle of an asynchronous pipeline, or code with a fixed memory budget.
 * The paper has no counterpart of this call (it serves such callers, not the method).
 * Arguments and results are those of bq_quantize. The scratch is a file-scope device
 * array of 229632 bytes (the workspace size of every scheme and shape); every GPU that
 * loads the library holds one copy until the process exits. A call whose scheme would
 * need more returns BQ_ERR_WORKSPACE. Every call looks the array's device address up
 * (cudaGetSymbolAddress), so the address stays right after a device reset; the first
 * call on a device also loads the library's device code there, so make that first
 * call before any stream capture. Every call shares the one array and zeroes its counters on the stream
 * first: calls that may overlap on the GPU (other streams, other threads) race, and
 * must be serialized by the caller. No cudaMalloc or cudaFree is made.
 */
bq_status bq_quantize_noalloc(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                              const bq_scheme* scheme,
                              void* codes, void* scales, void* zero_points, float* tensor_scale,
                              bq_stats* stats, void* stream);

/*
 * Block-scaled GEMM on the tensor cores: D[m, n] = sum_k A[m, k] B[n, k], with A and B
 * quantized by bq_quantize (or bq_quantize_batch) along k under the same scheme, scales
 * in the GEMM layout (scale_layout = BQ_LAYOUT_GEMM), codes and scales passed as
 * bq_quantize wrote them. This is the consumer block scaling serves: "Quantization survey"
 * §4.3 (MX and NV formats feed Blackwell's block-scaled tensor cores) and the FP8
 * training recipe's fp8_matmul of two FP8 operands with fp32 accumulation.
 *  - MXFP8 (scheme: BQ_FP8_E4M3 or BQ_FP8_E5M2, BQ_MX_BLOCK): each product of codes is
 *    scaled by both blocks' 2^e on the tensor cores; k % 128 == 0.
 *  - NVFP4 (BQ_FP4_E2M1, BQ_NV_BLOCK): the E4M3 block scales on the tensor cores, then
 *    D = acc * S_a * S_b with the operands' fp32 tensor scales (a_tensor_scale,
 *    b_tensor_scale: device, one fp32 each); k % 256 == 0.
 *  - scheme->hadamard = 1: both operands carry the block-16 rotation along k; H16/4 is
 *    orthogonal, so the product equals that of the unrotated operands up to rounding.
 * a_codes: [m, k] (FP4: [m, k / 2] bytes), b_codes: [n, k] likewise, row-major (k
 * contiguous: a weight W[out, in] is B with n = out); a_scales / b_scales: the GEMM-layout
 * scale buffers of those tensors (bq_buffer_sizes(scheme, m or n, k)). d: device
 * [m, n] row-major, fp32 (BQ_DT_FP32) or bf16 (BQ_DT_BF16, round to nearest even).
 * Accumulation is fp32 on the tensor cores (not bit-exact with any CPU order).
 * Shapes: m % 128 == 0, n % 128 == 0 (else BQ_ERR_SHAPE); m == 0 or n == 0 does nothing.
 * Alignment: codes, scales and d 16-byte aligned (else BQ_ERR_ALIGNMENT). Other schemes
 * (INT formats, MXFP4 / MXFP6, row-major scales): BQ_ERR_UNSUPPORTED. Every wait in the
 * kernel is bounded as described under bq_wait_timeouts below (which counts the GEMM's
 * too). No workspace; enqueued on stream.
 */
bq_status bq_gemm(const void* a_codes, const void* a_scales, const float* a_tensor_scale,
                  const void* b_codes, const void* b_scales, const float* b_tensor_scale,
                  int64_t m, int64_t n, int64_t k, const bq_scheme* scheme,
                  void* d, int32_t d_dtype, void* stream);

/*
 * Bounded waits. The quantize kernels stage their input tiles in shared memory with
 * tensor-map bulk copies and wait for each on an mbarrier; a wait that has not
 * completed after about one second gives up instead of hanging. The kernel then stops
 * early and the call's outputs are incomplete. This is a failure of the device or
 * driver, not of the arguments.
 *
 * bq_wait_timeouts writes to *count how many such waits gave up on the current device
 * since the library was loaded or last reset (reset != 0 sets the count back to zero).
 * It synchronizes with the device (a blocking copy). count: host pointer.
 * Returns BQ_ERR_INVALID_ARG for a NULL count, BQ_ERR_CUDA if the copy fails.
 * (The source pages have no counterpart: this only reports the library's own waits.)
 */
bq_status bq_wait_timeouts(uint32_t* count, int32_t reset);

/*
 * Fault injection for tests of the bounded waits (no counterpart on the pages). The next
 * call that runs the flat quantize kernel (bq_quantize, bq_quantize_with_range or
 * bq_quantize_batch with a per-tensor, per-group, MX or NV scheme, or a per-row scheme
 * of at most 2048 columns, a power-of-two multiple of 64) issues no copy for the first
 * staged tile of its warp number `warp` (warps are numbered CTA by CTA from 0; warp 0
 * always has work). That warp's wait gives up after the one-second limit, it waits
 * (bounded) for its other copies in flight and stops; the call's outputs are then
 * incomplete and bq_wait_timeouts counts one more. Nothing faults and nothing is left in
 * flight; a following call on the same workspace runs normally. One-shot: the call that
 * consumes it resets it. warp < 0: BQ_ERR_INVALID_ARG.
 */
bq_status bq_debug_skip_tile_copy(int32_t warp);

/* QSNR = -10 log10(err2 / x2) in dB from a host copy of the stats ("INT vs FP at fine
 * granularity" §4.1): +inf when err2 = 0, NaN when x2 = 0 with err2 > 0 or for a NULL
 * pointer. host_stats: host memory, read only. bq_stats_to_db and bq_stats_qsnr_db are
 * the same function under two names. */
double bq_stats_to_db(const bq_stats* host_stats);
double bq_stats_qsnr_db(const bq_stats* host_stats);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
