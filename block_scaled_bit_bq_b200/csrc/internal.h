// internal.h -- launch interface between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "bq.h"
#include "common.cuh"

namespace bq {

// Arguments of the one-pass kernels that see the tensor as a flat run of 16-element
// chunks (per-tensor, per-group, MX and NV granularities). Groups never straddle rows
// because cols is a multiple of the group size.
struct FlatArgs {
    const uint32_t* x;          // bf16 pairs
    uint8_t* codes;
    void* scales;
    void* zps;
    float* tensor_scale;
    bq_stats* stats;
    uint8_t* ws;
    const float* range;         // per-tensor / NV: {amax, min, max} of the (rotated) tensor
    uint32_t n_chunks;          // rows * cols / 16 (of the whole batch)
    uint32_t batch;             // tensors (1: one tensor; > 1: contiguous, same shape, no ragged span)
    uint32_t spans_per_tensor;  // 64-element spans of one tensor (the last one may be partial)
    uint32_t unit_oct;          // octets (8 spans) per partition unit: 1, or lanes_per_group / 8
    int32_t lanes_per_group;    // per-group: 0 (block 16), -1 (block 32), block / 64 (64..512)
    int32_t scale_fp16;         // 1: fp16 scales and zero points
    double n_elems;
    float inv_unit;             // 1 / elements per scaling unit (kappa)
    FastDiv gemm_nb;            // MX / NV scales in the GEMM layout: division by blocks per row
    int32_t gemm_layout;        // 1: scales in the GEMM layout; 0: row-major
    uint32_t skip_tile;         // fault injection for tests: this warp issues no copy for its
                                // first tile (its wait runs out); 0xFFFFFFFF: none
};

// Per-row kernel: one CTA per row at a time.
struct RowArgs {
    const uint32_t* x;
    uint8_t* codes;
    void* scales;
    void* zps;
    bq_stats* stats;
    uint8_t* ws;
    uint32_t rows;
    uint32_t cpr;               // chunks per row = cols / 16
    int32_t scale_fp16;
    float inv_cols;
};

// Per-row quantize of rows of cols % 64 == 0 elements, a warp per row (the row passes
// through the warp's tile ring twice: range, then codes).
struct RowsArgs {
    const uint32_t* x;
    uint8_t* codes;
    void* scales;
    void* zps;
    bq_stats* stats;
    uint8_t* ws;
    uint32_t rows;
    uint32_t cols;
    uint32_t cpr;               // chunks per row = cols / 16
    uint32_t nseg;              // 64-element segments per row = cols / 64
    uint32_t tiles;             // tiles per row = ceil(nseg / 32)
    int32_t scale_fp16;
    float inv_cols;
};

// 2-D tiles: one scale per TILE x TILE tile, a CTA per tile at a time.
constexpr uint32_t TILE = 128;

struct Tile2dArgs {
    const uint32_t* x;
    uint8_t* codes;
    void* scales;
    void* zps;
    bq_stats* stats;
    uint8_t* ws;
    uint32_t rows;
    uint32_t cols;
    uint32_t tpr;               // tiles per tile row = cols / TILE
    uint32_t ntiles;            // ceil(rows / TILE) * tpr
    int32_t scale_fp16;
};

// Row transforms before quantizing (a per-column factor, a randomized full-row
// Hadamard rotation): a CTA per row at a time, the row held in shared memory as fp32.
struct RtArgs {
    const uint32_t* x;
    uint8_t* codes;
    void* scales;
    void* zps;
    bq_stats* stats;            // may be null
    uint8_t* ws;
    const float* col_scale;     // [cols] or null
    const uint32_t* sign_bits;  // [cols / 32] or null (no rotation)
    uint32_t rows;
    uint32_t cols;
    uint32_t cpr;               // chunks per row = cols / 16
    uint32_t lanes;             // chunks per scaling unit (1 .. 32); 0: the whole row
    int32_t scale_fp16;
    float norm;                 // rotation: the fp32 value nearest 1 / sqrt(cols)
    float inv_unit;             // 1 / elements per unit (kappa)
    FastDiv gemm_nb;            // MX scales in the GEMM layout (see FlatArgs)
    int32_t gemm_layout;
};

struct DequantArgs {
    const uint8_t* codes;
    const void* scales;
    const void* zps;
    const float* tensor_scale;
    void* out;
    const uint32_t* x;          // QSNR only
    bq_stats* stats;            // QSNR only
    uint8_t* ws;                // QSNR only
    uint32_t n_chunks;
    uint32_t n_dtiles;
    uint32_t chunks_per_unit;   // chunks sharing one scale (0: one scale for the tensor);
                                // 2-D tiles: chunks per row
    uint32_t fd_m, fd_s;        // fast division by chunks_per_unit
    uint32_t tile_cols;         // 2-D tiles: tiles per tile row (cols / TILE); else 0
    int32_t scale_fp16;
    FastDiv gemm_nb;            // MX / NV scales in the GEMM layout (see FlatArgs)
    int32_t gemm_layout;
};

// Block-scaled GEMM D = A B^T on the tensor cores (codes and GEMM-layout scales as
// bq_quantize writes them).
enum { GEMM_MXF8 = 0, GEMM_NVF4 = 1 };

struct GemmArgs {
    const void* a;              // codes [m, kb] bytes, K-major
    const void* b;              // codes [n, kb] bytes, K-major
    const uint8_t* sfa;         // GEMM-layout scales of A (512-byte tiles)
    const uint8_t* sfb;
    const float* a_tensor_scale;  // NV: fp32 tensor scales (else unused)
    const float* b_tensor_scale;
    void* d;                    // [m, n] row-major, fp32 or bf16
    uint32_t m, n, kb;          // kb: bytes of a row of codes (k, or k / 2 for FP4)
    uint32_t k_stages;          // kb / 128
    uint32_t sf_tiles_per_row;  // scale tiles per 128-row tile (blocks per row / 4)
    uint32_t ldd;               // elements per row of D (n)
    uint32_t elem_fmt;          // MMA element format code (E4M3 0, E5M2 1; E2M1 1 for NV)
    int32_t d_bf16;
};

cudaError_t launch_gemm(int kind, const GemmArgs& g, cudaStream_t st);
// Waits of the GEMM kernel that gave up (each leaves that call's D incomplete). Synchronous.
cudaError_t gemm_wait_timeouts(unsigned int* count, bool reset);

// Scale kinds for dequantize / QSNR.
enum { SK_F32 = 0, SK_F16 = 1, SK_UE8M0 = 2, SK_NV = 3 };

int device_sm_count();
size_t workspace_bytes();

// Range pass into the workspace header (and into out[0..2] when out is not null).
cudaError_t launch_range(const uint32_t* x, uint32_t n_chunks, bool hadamard, bool minmax,
                         uint8_t* ws, float* out, cudaStream_t st);
cudaError_t launch_quant_flat(int fmt, int kind, bool hadamard, bool stats, const FlatArgs& a,
                              cudaStream_t st);
cudaError_t launch_quant_row(int fmt, bool hadamard, bool stats, const RowArgs& a, cudaStream_t st);
cudaError_t launch_quant_rows(int fmt, bool hadamard, bool stats, const RowsArgs& a, cudaStream_t st);
cudaError_t launch_quant_tile2d(int fmt, bool hadamard, bool stats, const Tile2dArgs& a, cudaStream_t st);
cudaError_t launch_quant_rt(int fmt, bool mx, const RtArgs& a, cudaStream_t st);
// rows of 1024, 2048 or 4096 columns with the rotation (rot_quant.cu)
cudaError_t launch_quant_rt64(int fmt, bool mx, const RtArgs& a, cudaStream_t st);
// Dequantize with the inverse full-row rotation (sign_bits [cols / 32], norm as RtArgs).
cudaError_t launch_dequant_rt(int fmt, int sk, int out_dtype, const DequantArgs& a, const uint32_t* sign_bits,
                              uint32_t rows, uint32_t cols, float norm, cudaStream_t st);
cudaError_t launch_dequant(int fmt, int sk, bool hadamard, int out_dtype, const DequantArgs& a,
                           cudaStream_t st);
cudaError_t launch_qsnr(int fmt, int sk, bool hadamard, const DequantArgs& a, cudaStream_t st);

// Tile waits of the quantize kernels that gave up (each leaves that call's results
// incomplete); reset: set the count back to zero. Synchronous.
cudaError_t flat_wait_timeouts(unsigned int* count, bool reset);

}  // namespace bq
