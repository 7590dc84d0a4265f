// api.cu -- the C ABI of libbq.so (declared and documented in include/bq.h):
// argument, shape and alignment checks on the host, buffer sizing, and dispatch to
// the kernels on the caller's stream. Nothing here allocates device memory.
#include "common.cuh"
#include "internal.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstring>

namespace bq {

namespace {

constexpr int MAX_DEVICES = 64;
// elements per call (per launch of a batch): chunk indices stay below 2^32 - 4 with room
// for the flat kernel's "no span" index
constexpr uint64_t MAX_ELEMS = (1ull << 36) - 2048;
// scales of one bq_quantize_batch launch in the GEMM layout (see there)
constexpr uint64_t GEMM_BATCH_SCALE_BYTES = 16ull << 20;
std::atomic<int> g_sm_count[MAX_DEVICES];

struct Plan {
    int fmt, gran, block, sdt, had;
    bool four, asym, is_int;
    uint64_t n;            // elements
    uint32_t n_chunks;     // n / 16
    uint64_t n_scales;
    size_t code_bytes, scale_bytes, zp_bytes, ts_bytes;
    bool needs_range;      // per-tensor and NV schemes take the range pass first
    bool gemm_layout;      // MX / NV block scales in the GEMM layout
    uint32_t nb;           // blocks per row (MX / NV)
};

bool fmt_is_int(int f) { return f == BQ_INT8_SYM || f == BQ_INT8_ASYM || f == BQ_INT4_SYM || f == BQ_UINT4_ASYM; }
bool fmt_four(int f) { return f == BQ_INT4_SYM || f == BQ_UINT4_ASYM || f == BQ_FP4_E2M1; }
bool fmt_asym(int f) { return f == BQ_INT8_ASYM || f == BQ_UINT4_ASYM; }

bq_status make_plan(const bq_scheme* s, int64_t rows, int64_t cols, Plan* p)
{
    if (!s) return BQ_ERR_INVALID_ARG;
    if ((s->scale_layout != BQ_LAYOUT_ROWS && s->scale_layout != BQ_LAYOUT_GEMM) ||
        (s->hadamard != 0 && s->hadamard != 1)) return BQ_ERR_INVALID_ARG;
    if (s->format < BQ_INT8_SYM || s->format > BQ_FP6_E3M2) return BQ_ERR_INVALID_ARG;
    if (s->granularity < BQ_PER_TENSOR || s->granularity > BQ_TILE_2D) return BQ_ERR_INVALID_ARG;
    if (s->scale_dtype < BQ_DT_BF16 || s->scale_dtype > BQ_DT_E4M3) return BQ_ERR_INVALID_ARG;
    std::memset(p, 0, sizeof *p);
    p->fmt = s->format; p->gran = s->granularity; p->sdt = s->scale_dtype; p->had = s->hadamard;
    p->four = fmt_four(p->fmt); p->asym = fmt_asym(p->fmt); p->is_int = fmt_is_int(p->fmt);

    const bool fp6 = p->fmt == BQ_FP6_E2M3 || p->fmt == BQ_FP6_E3M2;
    switch (p->gran) {
    case BQ_PER_TENSOR:
    case BQ_PER_ROW:
        if (p->fmt == BQ_FP4_E2M1 || fp6) return BQ_ERR_UNSUPPORTED;
        if (p->sdt != BQ_DT_FP32 && p->sdt != BQ_DT_FP16) return BQ_ERR_UNSUPPORTED;
        p->block = 0;
        break;
    case BQ_PER_GROUP:
        if (p->fmt == BQ_FP4_E2M1 || fp6) return BQ_ERR_UNSUPPORTED;
        if (p->sdt != BQ_DT_FP32 && p->sdt != BQ_DT_FP16) return BQ_ERR_UNSUPPORTED;
        if (!(s->block == 16 || s->block == 32 || s->block == 64 || s->block == 128 ||
              s->block == 256 || s->block == 512)) return BQ_ERR_UNSUPPORTED;
        p->block = s->block;
        break;
    case BQ_MX_BLOCK:
        if (!(p->fmt == BQ_INT8_SYM || p->fmt == BQ_FP8_E4M3 || p->fmt == BQ_FP8_E5M2 || p->fmt == BQ_FP4_E2M1 || fp6))
            return BQ_ERR_UNSUPPORTED;
        if (!(s->block == 32 || s->block == 0) || p->sdt != BQ_DT_UE8M0) return BQ_ERR_UNSUPPORTED;
        p->block = 32;
        break;
    case BQ_NV_BLOCK:
        if (!(p->fmt == BQ_FP4_E2M1 || p->fmt == BQ_INT4_SYM)) return BQ_ERR_UNSUPPORTED;
        if (!(s->block == 16 || s->block == 0) || p->sdt != BQ_DT_E4M3) return BQ_ERR_UNSUPPORTED;
        p->block = 16;
        break;
    case BQ_TILE_2D:
        if (p->fmt == BQ_FP4_E2M1 || fp6) return BQ_ERR_UNSUPPORTED;
        if (p->sdt != BQ_DT_FP32 && p->sdt != BQ_DT_FP16) return BQ_ERR_UNSUPPORTED;
        if (!(s->block == 128 || s->block == 0)) return BQ_ERR_UNSUPPORTED;
        p->block = TILE;
        break;
    }
    p->gemm_layout = s->scale_layout == BQ_LAYOUT_GEMM;
    if (p->gemm_layout && !(p->gran == BQ_MX_BLOCK || p->gran == BQ_NV_BLOCK)) return BQ_ERR_UNSUPPORTED;
    if (p->gemm_layout && cols % 128 != 0) return BQ_ERR_SHAPE;
    if (rows < 0 || cols <= 0 || cols % 16 != 0) return BQ_ERR_SHAPE;
    if (p->block && cols % p->block != 0) return BQ_ERR_SHAPE;
    if (rows > 0 && (uint64_t)rows > MAX_ELEMS / (uint64_t)cols) return BQ_ERR_SHAPE;
    if (rows >= (1ll << 31) || cols >= (1ll << 31)) return BQ_ERR_SHAPE;

    p->n = (uint64_t)rows * (uint64_t)cols;
    p->n_chunks = (uint32_t)(p->n / 16);
    switch (p->gran) {
    case BQ_PER_TENSOR: p->n_scales = 1; break;
    case BQ_PER_ROW: p->n_scales = (uint64_t)rows; break;
    case BQ_TILE_2D: p->n_scales = (((uint64_t)rows + TILE - 1) / TILE) * ((uint64_t)cols / TILE); break;
    default: p->n_scales = p->n / (uint64_t)p->block; break;
    }
    if (p->gran == BQ_MX_BLOCK || p->gran == BQ_NV_BLOCK) p->nb = (uint32_t)(cols / p->block);
    if (p->gemm_layout) {   // 128 x 4 tiles: rows padded to 128 (nb is a multiple of 4)
        p->n_scales = (((uint64_t)rows + 127) / 128) * 128 * (uint64_t)p->nb;
        if (p->n_scales > 0xFFFFFFFFull) return BQ_ERR_SHAPE;    // byte offsets are 32-bit
    }
    const size_t se = (p->sdt == BQ_DT_FP32) ? 4 : (p->sdt == BQ_DT_FP16) ? 2 : 1;
    p->code_bytes = p->four ? p->n / 2 : p->n;
    p->scale_bytes = p->n_scales * se;
    p->zp_bytes = p->asym ? p->n_scales * se : 0;
    p->ts_bytes = p->gran == BQ_NV_BLOCK ? 4 : 0;
    p->needs_range = (p->gran == BQ_PER_TENSOR || p->gran == BQ_NV_BLOCK);
    return BQ_OK;
}

bool aligned32(const void* ptr) { return ((uintptr_t)ptr & 31u) == 0; }
bool aligned4(const void* ptr) { return ((uintptr_t)ptr & 3u) == 0; }

size_t ws_needed(const Plan& p, bool stats) { return (stats || p.needs_range) ? WS_BYTES : 0; }

int kind_of(int gran)
{
    switch (gran) {
    case BQ_PER_TENSOR: return K_TENSOR;
    case BQ_PER_GROUP: return K_GROUP;
    case BQ_MX_BLOCK: return K_MX;
    default: return K_NV;
    }
}

int scale_kind(const Plan& p)
{
    if (p.gran == BQ_MX_BLOCK) return SK_UE8M0;
    if (p.gran == BQ_NV_BLOCK) return SK_NV;
    return p.sdt == BQ_DT_FP16 ? SK_F16 : SK_F32;
}

DequantArgs dequant_args(const Plan& p, int64_t cols)
{
    DequantArgs a;
    std::memset(&a, 0, sizeof a);
    a.n_chunks = p.n_chunks;
    a.n_dtiles = (uint32_t)((p.n_chunks + 63u) / 64u);
    uint32_t cpu = 0;
    switch (p.gran) {
    case BQ_PER_TENSOR: cpu = 0; break;
    case BQ_PER_ROW: cpu = (uint32_t)(cols / 16); break;
    case BQ_TILE_2D: cpu = (uint32_t)(cols / 16); break;     // divides a chunk index into its row
    default: cpu = (uint32_t)(p.block / 16); break;
    }
    a.chunks_per_unit = cpu;
    if (cpu) {
        const FastDiv f = make_fastdiv(cpu);
        a.fd_m = f.m;
        a.fd_s = f.s;
    }
    a.tile_cols = p.gran == BQ_TILE_2D ? (uint32_t)(cols / TILE) : 0u;
    if (p.gemm_layout) { a.gemm_layout = 1; a.gemm_nb = make_fastdiv(p.nb); }
    a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
    return a;
}

bq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA; }

// The range pass's result in the workspace header: {amax, min, max}.
const float* ws_range_ptr(void* ws)
{
    return reinterpret_cast<const float*>(reinterpret_cast<uint8_t*>(ws) + offsetof(WsHeader, amax));
}

// Test hook (bq_debug_skip_tile_copy): the tile of the next flat quantize launch whose
// copy is not issued; consumed by that launch.
std::atomic<uint32_t> g_skip_tile{0xFFFFFFFFu};

uint32_t take_skip_tile() { return g_skip_tile.exchange(0xFFFFFFFFu, std::memory_order_acq_rel); }

// The quantize pass of bq_quantize / bq_quantize_with_range: every check done; range:
// {amax, min, max} of the (rotated) tensor for per-tensor and NV schemes.
bq_status quantize_pass(const Plan& p, const uint32_t* xw, int64_t rows, int64_t cols, void* codes, void* scales,
                        void* zero_points, float* tensor_scale, bq_stats* stats, uint8_t* ws, const float* range,
                        cudaStream_t s)
{
    const bool want_stats = stats != nullptr;
    if (p.gran == BQ_TILE_2D) {
        Tile2dArgs a;
        std::memset(&a, 0, sizeof a);
        a.x = xw; a.codes = reinterpret_cast<uint8_t*>(codes); a.scales = scales; a.zps = zero_points;
        a.stats = stats; a.ws = ws;
        a.rows = (uint32_t)rows; a.cols = (uint32_t)cols;
        a.tpr = (uint32_t)(cols / TILE);
        a.ntiles = (uint32_t)p.n_scales;
        a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
        return cuda_status(launch_quant_tile2d(p.fmt, p.had != 0, want_stats, a, s));
    }
    const bool pow2_segments = cols % 64 == 0 && ((cols / 64) & (cols / 64 - 1)) == 0;
    if (p.gran == BQ_PER_ROW && pow2_segments && cols <= 2048) {
        // a row is a group of cols elements inside one warp tile (cols / 64 lanes)
        FlatArgs a;
        std::memset(&a, 0, sizeof a);
        a.x = xw; a.codes = reinterpret_cast<uint8_t*>(codes); a.scales = scales; a.zps = zero_points;
        a.stats = stats; a.ws = ws;
        a.n_chunks = p.n_chunks;
        a.lanes_per_group = (int32_t)(cols / 64);
        a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
        a.n_elems = (double)p.n;
        a.inv_unit = 1.0f / (float)cols;
        a.batch = 1;
        a.spans_per_tensor = (p.n_chunks + 3u) / 4u;
        a.unit_oct = a.lanes_per_group > 8 ? (uint32_t)a.lanes_per_group / 8u : 1u;
        a.skip_tile = take_skip_tile();
        return cuda_status(launch_quant_flat(p.fmt, K_GROUP, p.had != 0, want_stats, a, s));
    }
    if (p.gran == BQ_PER_ROW && cols % 64 == 0) {
        RowsArgs a;
        std::memset(&a, 0, sizeof a);
        a.x = xw; a.codes = reinterpret_cast<uint8_t*>(codes); a.scales = scales; a.zps = zero_points;
        a.stats = stats; a.ws = ws;
        a.rows = (uint32_t)rows; a.cols = (uint32_t)cols; a.cpr = (uint32_t)(cols / 16);
        a.nseg = (uint32_t)(cols / 64); a.tiles = (a.nseg + 31u) / 32u;
        a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
        a.inv_cols = 1.0f / (float)cols;
        return cuda_status(launch_quant_rows(p.fmt, p.had != 0, want_stats, a, s));
    }
    if (p.gran == BQ_PER_ROW) {
        RowArgs a;
        std::memset(&a, 0, sizeof a);
        a.x = xw; a.codes = reinterpret_cast<uint8_t*>(codes); a.scales = scales; a.zps = zero_points;
        a.stats = stats; a.ws = ws;
        a.rows = (uint32_t)rows; a.cpr = (uint32_t)(cols / 16);
        a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
        a.inv_cols = 1.0f / (float)cols;
        return cuda_status(launch_quant_row(p.fmt, p.had != 0, want_stats, a, s));
    }
    FlatArgs a;
    std::memset(&a, 0, sizeof a);
    a.x = xw; a.codes = reinterpret_cast<uint8_t*>(codes); a.scales = scales; a.zps = zero_points;
    a.tensor_scale = tensor_scale; a.stats = stats; a.ws = ws;
    a.n_chunks = p.n_chunks;
    // groups: 16 elements -> 0 (four units per lane), 32 -> -1 (two per lane),
    // 64 and up -> lanes per group (one unit over block / 64 lanes)
    a.lanes_per_group = p.gran != BQ_PER_GROUP ? 1 : (p.block == 16 ? 0 : (p.block == 32 ? -1 : p.block / 64));
    a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
    a.n_elems = (double)p.n;
    a.inv_unit = p.block ? 1.0f / (float)p.block : 0.0f;
    if (p.gemm_layout) { a.gemm_layout = 1; a.gemm_nb = make_fastdiv(p.nb); }
    a.range = range;
    a.batch = 1;
    a.spans_per_tensor = (p.n_chunks + 3u) / 4u;
    a.unit_oct = a.lanes_per_group > 8 ? (uint32_t)a.lanes_per_group / 8u : 1u;
    a.skip_tile = take_skip_tile();
    return cuda_status(launch_quant_flat(p.fmt, kind_of(p.gran), p.had != 0, want_stats, a, s));
}

// Flat-kernel arguments of a batch of `batch` tensors of one plan (p describes one tensor).
FlatArgs batch_args(const Plan& p, int64_t cols, uint32_t batch)
{
    FlatArgs a;
    std::memset(&a, 0, sizeof a);
    a.n_chunks = p.n_chunks * batch;
    a.lanes_per_group = p.gran == BQ_PER_ROW ? (int32_t)(cols / 64)
                      : p.gran != BQ_PER_GROUP ? 1 : (p.block == 16 ? 0 : (p.block == 32 ? -1 : p.block / 64));
    a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
    a.n_elems = (double)p.n;
    a.inv_unit = p.gran == BQ_PER_ROW ? 1.0f / (float)cols : 1.0f / (float)p.block;
    if (p.gemm_layout) { a.gemm_layout = 1; a.gemm_nb = make_fastdiv(p.nb); }
    a.batch = batch;
    a.spans_per_tensor = p.n_chunks / 4u;
    a.unit_oct = a.lanes_per_group > 8 ? (uint32_t)a.lanes_per_group / 8u : 1u;
    a.skip_tile = take_skip_tile();
    return a;
}

}  // namespace

int device_sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) dev = 0;
    int v = g_sm_count[dev].load(std::memory_order_relaxed);
    if (v <= 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        g_sm_count[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

size_t workspace_bytes() { return WS_BYTES; }

}  // namespace bq

using namespace bq;

extern "C" {

const char* bq_status_string(int status)
{
    switch (status) {
    case BQ_OK: return "BQ_OK";
    case BQ_ERR_INVALID_ARG: return "BQ_ERR_INVALID_ARG: null pointer or bad enum value";
    case BQ_ERR_UNSUPPORTED: return "BQ_ERR_UNSUPPORTED: format / granularity / scale dtype combination not offered";
    case BQ_ERR_SHAPE: return "BQ_ERR_SHAPE: rows < 0, cols not a positive multiple of 16 (and of the block), or too large";
    case BQ_ERR_ALIGNMENT: return "BQ_ERR_ALIGNMENT: x, codes and out must be 32-byte aligned, scales, zero points and tensor scale 4-byte aligned";
    case BQ_ERR_WORKSPACE: return "BQ_ERR_WORKSPACE: workspace missing or too small";
    case BQ_ERR_CUDA: return "BQ_ERR_CUDA: a CUDA launch or call failed";
    default: return "unknown bq_status";
    }
}

const char* bq_version(void) { return "bq 0.1 (sm_100a)"; }

bq_status bq_buffer_sizes(const bq_scheme* scheme, int64_t rows, int64_t cols,
                          size_t* code_bytes, size_t* scale_bytes,
                          size_t* zero_point_bytes, size_t* tensor_scale_bytes)
{
    Plan p;
    const bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (code_bytes) *code_bytes = p.code_bytes;
    if (scale_bytes) *scale_bytes = p.scale_bytes;
    if (zero_point_bytes) *zero_point_bytes = p.zp_bytes;
    if (tensor_scale_bytes) *tensor_scale_bytes = p.ts_bytes;
    return BQ_OK;
}

bq_status bq_workspace_size(const bq_scheme* scheme, int64_t rows, int64_t cols, int with_stats, size_t* bytes)
{
    Plan p;
    const bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (!bytes) return BQ_ERR_INVALID_ARG;
    *bytes = ws_needed(p, with_stats != 0);
    return BQ_OK;
}

bq_status bq_quantize(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                      const bq_scheme* scheme,
                      void* codes, void* scales, void* zero_points, float* tensor_scale,
                      bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (x_dtype != BQ_DT_BF16) return BQ_ERR_UNSUPPORTED;
    const bool want_stats = stats != nullptr;
    const size_t need_ws = ws_needed(p, want_stats);
    if (need_ws && (!workspace || workspace_bytes < need_ws)) return BQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (p.n == 0) {
        if (want_stats) return cuda_status(cudaMemsetAsync(stats, 0, sizeof(bq_stats), s));
        return BQ_OK;
    }
    if (!x || !codes || !scales) return BQ_ERR_INVALID_ARG;
    if (p.asym && !zero_points) return BQ_ERR_INVALID_ARG;
    if (p.gran == BQ_NV_BLOCK && !tensor_scale) return BQ_ERR_INVALID_ARG;
    if (!aligned32(x) || !aligned32(codes)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(scales) || !aligned4(zero_points) || !aligned4(tensor_scale)) return BQ_ERR_ALIGNMENT;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    const uint32_t* xw = reinterpret_cast<const uint32_t*>(x);

    if (p.needs_range) {
        const cudaError_t e = launch_range(xw, p.n_chunks, p.had != 0, p.gran == BQ_PER_TENSOR && p.asym, ws,
                                           nullptr, s);
        if (e != cudaSuccess) return BQ_ERR_CUDA;
    }
    return quantize_pass(p, xw, rows, cols, codes, scales, zero_points, tensor_scale, stats, ws,
                         p.needs_range ? ws_range_ptr(ws) : nullptr, s);
}

bq_status bq_tensor_range(const void* x, int32_t x_dtype, int64_t rows, int64_t cols, const bq_scheme* scheme,
                          float* range, void* workspace, size_t workspace_bytes, void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (x_dtype != BQ_DT_BF16) return BQ_ERR_UNSUPPORTED;
    if (!p.needs_range) return BQ_ERR_UNSUPPORTED;
    if (!range) return BQ_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < WS_BYTES) return BQ_ERR_WORKSPACE;
    if (!aligned4(range)) return BQ_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (p.n == 0) return cuda_status(cudaMemsetAsync(range, 0, 3 * sizeof(float), s));
    if (!x) return BQ_ERR_INVALID_ARG;
    if (!aligned32(x)) return BQ_ERR_ALIGNMENT;
    return cuda_status(launch_range(reinterpret_cast<const uint32_t*>(x), p.n_chunks, p.had != 0,
                                    p.gran == BQ_PER_TENSOR && p.asym, reinterpret_cast<uint8_t*>(workspace), range,
                                    s));
}

bq_status bq_quantize_with_range(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                 const bq_scheme* scheme, const float* range,
                                 void* codes, void* scales, void* zero_points, float* tensor_scale,
                                 bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (x_dtype != BQ_DT_BF16) return BQ_ERR_UNSUPPORTED;
    if (!p.needs_range) return BQ_ERR_UNSUPPORTED;
    const bool want_stats = stats != nullptr;
    if (want_stats && (!workspace || workspace_bytes < WS_BYTES)) return BQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (p.n == 0) {
        if (want_stats) return cuda_status(cudaMemsetAsync(stats, 0, sizeof(bq_stats), s));
        return BQ_OK;
    }
    if (!x || !codes || !scales || !range) return BQ_ERR_INVALID_ARG;
    if (p.asym && !zero_points) return BQ_ERR_INVALID_ARG;
    if (p.gran == BQ_NV_BLOCK && !tensor_scale) return BQ_ERR_INVALID_ARG;
    if (!aligned32(x) || !aligned32(codes)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(scales) || !aligned4(zero_points) || !aligned4(tensor_scale) || !aligned4(range))
        return BQ_ERR_ALIGNMENT;
    return quantize_pass(p, reinterpret_cast<const uint32_t*>(x), rows, cols, codes, scales, zero_points,
                         tensor_scale, stats, reinterpret_cast<uint8_t*>(workspace), range, s);
}

bq_status bq_debug_skip_tile_copy(int32_t warp)
{
    if (warp < 0) return BQ_ERR_INVALID_ARG;
    g_skip_tile.store((uint32_t)warp, std::memory_order_release);
    return BQ_OK;
}

bq_status bq_quantize_batch(const void* x, int32_t x_dtype, int64_t batch, int64_t rows, int64_t cols,
                            const bq_scheme* scheme, void* codes, void* scales, void* zero_points,
                            bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (x_dtype != BQ_DT_BF16) return BQ_ERR_UNSUPPORTED;
    // row-local schemes that run on the flat kernel
    const bool pow2_segments = cols % 64 == 0 && ((cols / 64) & (cols / 64 - 1)) == 0;
    if (!(p.gran == BQ_PER_GROUP || p.gran == BQ_MX_BLOCK || (p.gran == BQ_PER_ROW && pow2_segments && cols <= 2048)))
        return BQ_ERR_UNSUPPORTED;
    if (batch < 0) return BQ_ERR_SHAPE;
    if (batch > 1 && p.n % 64 != 0) return BQ_ERR_SHAPE;           // tensors of whole 64-element spans
    if (batch > 1 && p.gemm_layout && rows % 128 != 0) return BQ_ERR_SHAPE;
    const bool want_stats = stats != nullptr;
    if (want_stats && (!workspace || workspace_bytes < WS_BYTES)) return BQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (batch == 0) return BQ_OK;
    if (p.n == 0) {
        if (want_stats) return cuda_status(cudaMemsetAsync(stats, 0, sizeof(bq_stats) * (size_t)batch, s));
        return BQ_OK;
    }
    if (!x || !codes || !scales) return BQ_ERR_INVALID_ARG;
    if (p.asym && !zero_points) return BQ_ERR_INVALID_ARG;
    if (!aligned32(x) || !aligned32(codes)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(scales) || !aligned4(zero_points)) return BQ_ERR_ALIGNMENT;
    // launches of at most one tensor per stats slot and MAX_ELEMS elements
    uint64_t per = std::min<uint64_t>((uint64_t)MAX_STAT_SLOTS, MAX_ELEMS / p.n);
    // GEMM-layout scales: a 512-byte scale tile gathers the scales of 128 rows, and each
    // warp fills 2-4 bytes of it at a time as it goes down its own rows, so a tile is
    // complete only when the launch is. Launches of at most GEMM_BATCH_SCALE_BYTES of
    // scales keep the partly written tiles in L2 meanwhile (64 MXFP8 tensors of
    // 4096 x 11008 in one launch, 90 MB of scales, ran 1.45 times as long as with
    // row-major scales).
    if (p.gemm_layout)
        per = std::max<uint64_t>(1, std::min<uint64_t>(per, GEMM_BATCH_SCALE_BYTES / std::max<size_t>(p.scale_bytes, 1)));
    const size_t scale_b = p.scale_bytes, zp_b = p.zp_bytes, code_b = p.code_bytes, x_b = p.n * 2;
    for (uint64_t b0 = 0; b0 < (uint64_t)batch; b0 += per) {
        const uint32_t nb = (uint32_t)std::min<uint64_t>(per, (uint64_t)batch - b0);
        FlatArgs a = batch_args(p, cols, nb);
        a.x = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(x) + b0 * x_b);
        a.codes = reinterpret_cast<uint8_t*>(codes) + b0 * code_b;
        a.scales = reinterpret_cast<uint8_t*>(scales) + b0 * scale_b;
        a.zps = zero_points ? reinterpret_cast<uint8_t*>(zero_points) + b0 * zp_b : nullptr;
        a.stats = want_stats ? stats + b0 : nullptr;
        a.ws = reinterpret_cast<uint8_t*>(workspace);
        const int kind = p.gran == BQ_MX_BLOCK ? K_MX : K_GROUP;
        const cudaError_t e = launch_quant_flat(p.fmt, kind, p.had != 0, want_stats, a, s);
        if (e != cudaSuccess) return BQ_ERR_CUDA;
    }
    return BQ_OK;
}

bq_status bq_dequantize(const void* codes, const void* scales, const void* zero_points,
                        const float* tensor_scale, int64_t rows, int64_t cols,
                        const bq_scheme* scheme, void* out, int32_t out_dtype, void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (out_dtype != BQ_DT_BF16 && out_dtype != BQ_DT_FP32) return BQ_ERR_UNSUPPORTED;
    if (p.n == 0) return BQ_OK;
    if (!codes || !scales || !out) return BQ_ERR_INVALID_ARG;
    if (p.asym && !zero_points) return BQ_ERR_INVALID_ARG;
    if (p.gran == BQ_NV_BLOCK && !tensor_scale) return BQ_ERR_INVALID_ARG;
    if (!aligned32(codes) || !aligned32(out)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(scales) || !aligned4(zero_points) || !aligned4(tensor_scale)) return BQ_ERR_ALIGNMENT;
    DequantArgs a = dequant_args(p, cols);
    a.codes = reinterpret_cast<const uint8_t*>(codes);
    a.scales = scales; a.zps = zero_points; a.tensor_scale = tensor_scale; a.out = out;
    return cuda_status(launch_dequant(p.fmt, scale_kind(p), p.had != 0, out_dtype, a,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

bq_status bq_qsnr(const void* x, int32_t x_dtype, const void* codes, const void* scales,
                  const void* zero_points, const float* tensor_scale,
                  int64_t rows, int64_t cols, const bq_scheme* scheme,
                  bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (x_dtype != BQ_DT_BF16) return BQ_ERR_UNSUPPORTED;
    if (!stats) return BQ_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < WS_BYTES) return BQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (p.n == 0) return cuda_status(cudaMemsetAsync(stats, 0, sizeof(bq_stats), s));
    if (!x || !codes || !scales) return BQ_ERR_INVALID_ARG;
    if (p.asym && !zero_points) return BQ_ERR_INVALID_ARG;
    if (p.gran == BQ_NV_BLOCK && !tensor_scale) return BQ_ERR_INVALID_ARG;
    if (!aligned32(x) || !aligned32(codes)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(scales) || !aligned4(zero_points) || !aligned4(tensor_scale)) return BQ_ERR_ALIGNMENT;
    DequantArgs a = dequant_args(p, cols);
    a.codes = reinterpret_cast<const uint8_t*>(codes);
    a.scales = scales; a.zps = zero_points; a.tensor_scale = tensor_scale;
    a.x = reinterpret_cast<const uint32_t*>(x);
    a.stats = stats;
    a.ws = reinterpret_cast<uint8_t*>(workspace);
    return cuda_status(launch_qsnr(p.fmt, scale_kind(p), p.had != 0, a, s));
}

namespace {

// Checks shared by the row-transform entry points: per-row, per-group and MX schemes
// without the block-16 rotation; cols a multiple of 512 up to 16384 (a power of two
// when rotating); the factor array 16-byte aligned.
bq_status rt_check(const Plan& p, int64_t cols, const bq_row_transform* rt)
{
    if (!(p.gran == BQ_PER_ROW || p.gran == BQ_PER_GROUP || p.gran == BQ_MX_BLOCK) || p.had) return BQ_ERR_UNSUPPORTED;
    if (cols % 512 != 0 || cols > 16384) return BQ_ERR_SHAPE;
    if (rt && rt->sign_bits && (cols & (cols - 1)) != 0) return BQ_ERR_SHAPE;
    if (rt && rt->reserved != 0) return BQ_ERR_INVALID_ARG;
    if (rt && rt->col_scale && ((uintptr_t)rt->col_scale & 15u) != 0) return BQ_ERR_ALIGNMENT;
    if (rt && rt->sign_bits && !aligned4(rt->sign_bits)) return BQ_ERR_ALIGNMENT;
    return BQ_OK;
}

float rt_norm(int64_t cols) { return (float)(1.0 / std::sqrt((double)cols)); }

}  // namespace

bq_status bq_quantize_rt(const void* x, int32_t x_dtype, int64_t rows, int64_t cols, const bq_scheme* scheme,
                         const bq_row_transform* rt, void* codes, void* scales, void* zero_points,
                         bq_stats* stats, void* workspace, size_t workspace_bytes, void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    if (x_dtype != BQ_DT_BF16) return BQ_ERR_UNSUPPORTED;
    st = rt_check(p, cols, rt);
    if (st != BQ_OK) return st;
    const bool want_stats = stats != nullptr;
    if (want_stats && (!workspace || workspace_bytes < WS_BYTES)) return BQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (p.n == 0) {
        if (want_stats) return cuda_status(cudaMemsetAsync(stats, 0, sizeof(bq_stats), s));
        return BQ_OK;
    }
    if (!x || !codes || !scales) return BQ_ERR_INVALID_ARG;
    if (p.asym && !zero_points) return BQ_ERR_INVALID_ARG;
    if (!aligned32(x) || !aligned32(codes)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(scales) || !aligned4(zero_points)) return BQ_ERR_ALIGNMENT;
    RtArgs a;
    std::memset(&a, 0, sizeof a);
    a.x = reinterpret_cast<const uint32_t*>(x); a.codes = reinterpret_cast<uint8_t*>(codes);
    a.scales = scales; a.zps = zero_points; a.stats = stats; a.ws = reinterpret_cast<uint8_t*>(workspace);
    a.col_scale = rt ? rt->col_scale : nullptr;
    a.sign_bits = rt ? rt->sign_bits : nullptr;
    a.rows = (uint32_t)rows; a.cols = (uint32_t)cols; a.cpr = (uint32_t)(cols / 16);
    a.lanes = p.gran == BQ_PER_ROW ? 0u : (uint32_t)(p.block / 16);
    a.scale_fp16 = p.sdt == BQ_DT_FP16 ? 1 : 0;
    a.norm = rt_norm(cols);
    a.inv_unit = 1.0f / (float)(p.gran == BQ_PER_ROW ? cols : p.block);
    if (p.gemm_layout) { a.gemm_layout = 1; a.gemm_nb = make_fastdiv(p.nb); }
    return cuda_status(launch_quant_rt(p.fmt, p.gran == BQ_MX_BLOCK, a, s));
}

bq_status bq_dequantize_rt(const void* codes, const void* scales, const void* zero_points, int64_t rows, int64_t cols,
                           const bq_scheme* scheme, const bq_row_transform* rt, void* out, int32_t out_dtype,
                           void* stream)
{
    Plan p;
    bq_status st = make_plan(scheme, rows, cols, &p);
    if (st != BQ_OK) return st;
    st = rt_check(p, cols, rt);
    if (st != BQ_OK) return st;
    if (!rt || !rt->sign_bits)          // no rotation to invert: the plain dequantize
        return bq_dequantize(codes, scales, zero_points, nullptr, rows, cols, scheme, out, out_dtype, stream);
    if (out_dtype != BQ_DT_BF16 && out_dtype != BQ_DT_FP32) return BQ_ERR_UNSUPPORTED;
    if (p.n == 0) return BQ_OK;
    if (!codes || !scales || !out) return BQ_ERR_INVALID_ARG;
    if (p.asym && !zero_points) return BQ_ERR_INVALID_ARG;
    if (!aligned32(codes) || !aligned32(out)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(scales) || !aligned4(zero_points)) return BQ_ERR_ALIGNMENT;
    DequantArgs a = dequant_args(p, cols);
    a.codes = reinterpret_cast<const uint8_t*>(codes);
    a.scales = scales; a.zps = zero_points; a.out = out;
    return cuda_status(launch_dequant_rt(p.fmt, scale_kind(p), out_dtype, a, rt->sign_bits, (uint32_t)rows,
                                         (uint32_t)cols, rt_norm(cols), reinterpret_cast<cudaStream_t>(stream)));
}

bq_status bq_wait_timeouts(uint32_t* count, int32_t reset)
{
    if (!count) return BQ_ERR_INVALID_ARG;
    unsigned int c = 0, g = 0;
    if (bq::flat_wait_timeouts(&c, reset != 0) != cudaSuccess) return BQ_ERR_CUDA;
    if (bq::gemm_wait_timeouts(&g, reset != 0) != cudaSuccess) return BQ_ERR_CUDA;
    *count = c + g;
    return BQ_OK;
}

bq_status bq_gemm(const void* a_codes, const void* a_scales, const float* a_tensor_scale,
                  const void* b_codes, const void* b_scales, const float* b_tensor_scale,
                  int64_t m, int64_t n, int64_t k, const bq_scheme* scheme,
                  void* d, int32_t d_dtype, void* stream)
{
    if (!scheme) return BQ_ERR_INVALID_ARG;
    Plan p;
    bq_status st = make_plan(scheme, 1, k, &p);
    if (st != BQ_OK) return st;
    int kind;
    uint32_t fmt_code;
    if (p.gran == BQ_MX_BLOCK && (p.fmt == BQ_FP8_E4M3 || p.fmt == BQ_FP8_E5M2)) {
        kind = GEMM_MXF8;
        fmt_code = p.fmt == BQ_FP8_E4M3 ? 0u : 1u;
    } else if (p.gran == BQ_NV_BLOCK && p.fmt == BQ_FP4_E2M1) {
        kind = GEMM_NVF4;
        fmt_code = 1u;
    } else {
        return BQ_ERR_UNSUPPORTED;
    }
    if (!p.gemm_layout) return BQ_ERR_UNSUPPORTED;
    if (d_dtype != BQ_DT_FP32 && d_dtype != BQ_DT_BF16) return BQ_ERR_UNSUPPORTED;
    const int64_t kstep = kind == GEMM_MXF8 ? 128 : 256;
    if (m < 0 || n < 0 || k <= 0 || m % 128 != 0 || n % 128 != 0 || k % kstep != 0) return BQ_ERR_SHAPE;
    if (m >= (1ll << 31) || n >= (1ll << 31) || k >= (1ll << 31) || (uint64_t)m * (uint64_t)n >= (1ull << 40))
        return BQ_ERR_SHAPE;
    if (m == 0 || n == 0) return BQ_OK;
    if (!a_codes || !a_scales || !b_codes || !b_scales || !d) return BQ_ERR_INVALID_ARG;
    if (kind == GEMM_NVF4 && (!a_tensor_scale || !b_tensor_scale)) return BQ_ERR_INVALID_ARG;
    auto al16 = [](const void* q) { return ((uintptr_t)q & 15u) == 0; };
    if (!al16(a_codes) || !al16(b_codes) || !al16(a_scales) || !al16(b_scales) || !al16(d)) return BQ_ERR_ALIGNMENT;
    if (!aligned4(a_tensor_scale) || !aligned4(b_tensor_scale)) return BQ_ERR_ALIGNMENT;
    GemmArgs g;
    std::memset(&g, 0, sizeof g);
    g.a = a_codes; g.b = b_codes;
    g.sfa = reinterpret_cast<const uint8_t*>(a_scales);
    g.sfb = reinterpret_cast<const uint8_t*>(b_scales);
    g.a_tensor_scale = a_tensor_scale; g.b_tensor_scale = b_tensor_scale;
    g.d = d;
    g.m = (uint32_t)m; g.n = (uint32_t)n;
    g.kb = (uint32_t)(kind == GEMM_MXF8 ? k : k / 2);
    g.k_stages = g.kb / 128u;
    g.sf_tiles_per_row = p.nb / 4u;
    g.ldd = (uint32_t)n;
    g.elem_fmt = fmt_code;
    g.d_bf16 = d_dtype == BQ_DT_BF16 ? 1 : 0;
    return cuda_status(launch_gemm(kind, g, reinterpret_cast<cudaStream_t>(stream)));
}

double bq_stats_qsnr_db(const bq_stats* host_stats)
{
    if (!host_stats) return NAN;
    if (host_stats->err2 == 0.0) return INFINITY;
    return -10.0 * std::log10(host_stats->err2 / host_stats->x2);
}

double bq_stats_to_db(const bq_stats* host_stats) { return bq_stats_qsnr_db(host_stats); }

}  // extern "C"
