// noalloc.cu -- bq_quantize for callers that cannot allocate device memory.
//
// bq_quantize needs a caller-provided workspace for per-tensor and NV schemes and
// whenever QSNR sums are requested. Some callers cannot make that allocation: code
// that runs under another component's allocator (a framework or serving runtime that
// owns all device memory and hands out fixed arenas), code that must not call
// cudaMalloc because it can synchronize the device in the middle of an asynchronous
// pipeline, and code with a fixed memory budget decided at start-up. This file gives
// them bq_quantize_noalloc, which runs the same kernels with the workspace placed in a
// file-scope device array instead.
#include "common.cuh"
#include "internal.h"

namespace bq {

namespace {

// The scratch every bq_quantize_noalloc call uses: WS_BYTES (224 KiB + 256 B), enough
// for the largest grid the kernels launch. Every GPU that loads the library holds one
// copy until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[WS_BYTES];

// Device address of the scratch on the current device. In host code the array's name is
// only a stand-in, not a device address. The address is looked up on every call rather
// than cached: after cudaDeviceReset (or any teardown of the primary context) the module
// is loaded again and the array may sit elsewhere. The first lookup on a device loads the
// library's device code there (lazy loading), which is why the first call should come
// before any stream capture; later lookups are a host-side table read.
cudaError_t scratch_address(void** out)
{
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

}  // namespace bq

extern "C" bq_status bq_quantize_noalloc(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                         const bq_scheme* scheme,
                                         void* codes, void* scales, void* zero_points, float* tensor_scale,
                                         bq_stats* stats, void* stream)
{
    size_t need = 0;
    bq_status st = bq_workspace_size(scheme, rows, cols, stats != nullptr, &need);
    if (st != BQ_OK) return st;
    if (need > sizeof(bq::g_noalloc_scratch)) return BQ_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0) {
        if (bq::scratch_address(&ws) != cudaSuccess) return BQ_ERR_CUDA;
        // The array keeps whatever the previous call left; the kernels need their
        // last-CTA counters (the header) at zero.
        if (cudaMemsetAsync(ws, 0, bq::WS_HEADER_BYTES, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
            return BQ_ERR_CUDA;
    }
    return bq_quantize(x, x_dtype, rows, cols, scheme, codes, scales, zero_points, tensor_scale, stats,
                       ws, need > 0 ? sizeof(bq::g_noalloc_scratch) : 0, stream);
}
