// llmint8_quantize_rowwise_noalloc: the row-wise quantizer for callers that
// cannot hand the library a workspace.
//
// Some host programs cannot call cudaMalloc when they need this quantizer:
// an inference server that reserved all device memory for its own pool at
// start-up (a later cudaMalloc fails or would break its accounting), a plugin
// running inside a host process that forbids device allocations after
// initialisation, or a latency-critical loop where an allocation's implicit
// device synchronisation is not acceptable. They still own the inputs and
// outputs; only the quantizer's small scratch (the compacted outlier list,
// its count and the kernel's barrier words) moves into the fixed array below.
//
// The array lives in this library's module, so every GPU that uses this entry
// point holds it (about 256 KB) from its first call until the process exits.
// All calls on a device share it and it keeps the last call's contents, so
// two calls whose work overlaps on the GPU (different streams, no ordering
// between them) race on it; calls ordered on one stream are safe.
//
// Its status word keeps the bits of every call since it was last cleared
// (a kernel that gave up on a bounded wait sets one and leaves its outputs
// incomplete); llmint8_noalloc_read_status reads and clears it.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "llmint8.h"

namespace llmint8 {
namespace {

constexpr int64_t kMaxRows = LLMINT8_NOALLOC_MAX_ROWS;
constexpr int64_t kMaxCols = LLMINT8_NOALLOC_MAX_COLS;
// The array's header uses the first words of a workspace header (carve() in
// internal.h): uint32 status at 0, int32 |O| at 4, the grid barrier's 64-bit
// word at 8, the late-outlier flag at 16. Change the two together.
constexpr size_t kNoallocHeaderBytes = 256;
constexpr size_t kNoallocStatusOff = 0;
constexpr size_t kNoallocCountOff = 4;
constexpr size_t kNoallocSyncOff = 8;
constexpr size_t kNoallocColIdxOff = kNoallocHeaderBytes;
constexpr size_t kScratchBytes = kNoallocColIdxOff + (size_t)kMaxCols * 4;

// The scratch. In host code this name is only a stand-in: the device address
// comes from cudaGetSymbolAddress below, once per device.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[64] = {};

// Device address of g_scratch on the current device `dev`, looked up on the
// first call for that device and cached for the life of the process (a
// cudaDeviceReset on that device invalidates it; this entry point must not be
// used after one).
cudaError_t scratch_address(int dev, void **out)
{
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

} // namespace
} // namespace llmint8

using namespace llmint8;

extern "C" llmint8_status llmint8_quantize_rowwise_noalloc(const void *X_f16, int64_t rows, int64_t cols,
                                                           float threshold, int8_t *codes, float *row_absmax,
                                                           uint32_t *outlier_bitmap, llmint8_stream_t stream)
{
    if (rows < 0)
        return LLMINT8_ERR_INVALID_ARG;
    if (cols <= 0 || cols % 16 != 0 || cols > LLMINT8_MAX_K)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (rows > kMaxRows || cols > kMaxCols)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    const float t = (threshold > 0.f && !std::isinf(threshold)) ? threshold : 0.f;
    if (!X_f16 || !codes || !row_absmax || (t > 0.f && !outlier_bitmap))
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X_f16) || !aligned16(codes) || !aligned16(row_absmax) ||
        (outlier_bitmap && !aligned16(outlier_bitmap)))
        return LLMINT8_ERR_ALIGNMENT;
    if (rows == 0) // no rows, no outlier columns: the bitmap is still written
        return (!outlier_bitmap ||
                cudaMemsetAsync(outlier_bitmap, 0, (size_t)((cols + 31) / 32) * 4, stream) == cudaSuccess)
                   ? LLMINT8_OK
                   : LLMINT8_ERR_CUDA;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    void *base = nullptr;
    if (scratch_address(dev.device, &base) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    char *s = static_cast<char *>(base);
    uint32_t *status = reinterpret_cast<uint32_t *>(s + kNoallocStatusOff);
    int32_t *count = reinterpret_cast<int32_t *>(s + kNoallocCountOff);
    uint32_t *sync = reinterpret_cast<uint32_t *>(s + kNoallocSyncOff);
    int32_t *col_idx = reinterpret_cast<int32_t *>(s + kNoallocColIdxOff);
    // The array keeps the previous call's contents: clear the count, the
    // grid-barrier word and the late-outlier flag (bytes 4..19, not the status
    // word, which accumulates until read), and the caller's bitmap, which the
    // kernels OR into.
    if (cudaMemsetAsync(count, 0, 16, stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (outlier_bitmap &&
        cudaMemsetAsync(outlier_bitmap, 0, (size_t)((cols + 31) / 32) * 4, stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    cudaError_t e = launch_quantize(X_f16, rows, cols, t, codes, row_absmax, outlier_bitmap, col_idx, count, sync,
                                    status, dev, stream);
    return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

extern "C" llmint8_status llmint8_noalloc_read_status(int clear, uint32_t *out)
{
    if (!out)
        return LLMINT8_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    void *base = nullptr;
    if (scratch_address(dev.device, &base) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    uint32_t *status = reinterpret_cast<uint32_t *>(static_cast<char *>(base) + kNoallocStatusOff);
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(out, status, sizeof(uint32_t), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear)
        e = cudaMemset(status, 0, sizeof(uint32_t));
    if (e != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    return *out ? LLMINT8_ERR_DEVICE : LLMINT8_OK;
}
