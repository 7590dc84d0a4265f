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

#include <atomic>
#include <mutex>

namespace bq {

namespace {

// The scratch every bq_quantize_noalloc call uses: WS_BYTES (128 KiB + 256 B), enough
// for the largest grid the kernels launch. Every GPU that loads the library holds one
// copy until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[WS_BYTES];

constexpr int MAX_DEV = 64;
std::atomic<void*> g_scratch_ptr[MAX_DEV];
std::mutex g_scratch_mu;

// Device address of the scratch on the current device (looked up once per device; in
// host code the array's name is only a stand-in, not a device address).
cudaError_t scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= MAX_DEV) return cudaErrorInvalidDevice;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        p = g_scratch_ptr[dev].load(std::memory_order_acquire);
        if (!p) {
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess) return e;
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
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
