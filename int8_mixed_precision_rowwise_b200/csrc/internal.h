// Host-side interfaces between the C-ABI front end and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace llmint8 {

// Workspace layout (byte offsets; every region 256-byte aligned):
//   [0]      uint32 status word (bits LLMINT8_DEV_*)
//   [4]      int32  |O| (outlier column count)
//   [8]      uint32 grid-barrier counter and generation, late-outlier flag
//   [256]    uint32 outlier bitmap [ceil(K/32)]
//   ...      int32  ascending outlier columns [K]
//   ...      fp32   SX [M]
//   ...      int8   CX [M x K]
struct Workspace {
    uint32_t *status;
    int32_t *count;
    uint32_t *sync;
    uint32_t *bitmap;
    int32_t *col_idx;
    float *sx;
    int8_t *cx;
    size_t bytes;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t carve(char *base, int64_t M, int64_t K, bool with_codes, Workspace *ws)
{
    size_t off = 0;
    auto take = [&](size_t n) {
        size_t o = off;
        off = align256(off + n);
        return base ? base + o : nullptr;
    };
    char *hdr = take(256);
    size_t nwords = (size_t)((K + 31) / 32);
    char *bm = take(nwords * 4);
    char *ci = take((size_t)K * 4);
    char *sx = with_codes ? take((size_t)M * 4) : nullptr;
    char *cx = with_codes ? take((size_t)M * (size_t)K) : nullptr;
    if (ws) {
        ws->status = reinterpret_cast<uint32_t *>(hdr);
        ws->count = hdr ? reinterpret_cast<int32_t *>(hdr + 4) : nullptr;
        ws->sync = hdr ? reinterpret_cast<uint32_t *>(hdr + 8) : nullptr;
        ws->bitmap = reinterpret_cast<uint32_t *>(bm);
        ws->col_idx = reinterpret_cast<int32_t *>(ci);
        ws->sx = reinterpret_cast<float *>(sx);
        ws->cx = reinterpret_cast<int8_t *>(cx);
        ws->bytes = off;
    }
    return off;
}

struct DeviceInfo {
    int device;
    int num_sms;
    int max_smem_optin;
};

// Cached per-device properties (first call per device queries them).
cudaError_t device_info(DeviceInfo *out);

// Quantize rows of X (fp16) with outlier detection at threshold t: codes,
// absmax over the non-outlier columns, the outlier bitmap and (t > 0) its
// compaction into col_idx/count. `bitmap` must be zeroed before the call.
// `sync` is two zeroed uint32 words (grid barrier); `status` receives
// LLMINT8_DEV_* bits.
cudaError_t launch_quantize(const void *X, int64_t rows, int64_t cols, float t, int8_t *codes,
                            float *absmax, uint32_t *bitmap, int32_t *col_idx, int32_t *count, uint32_t *sync,
                            uint32_t *status, const DeviceInfo &dev, cudaStream_t stream);

// Bitmap -> ascending column list and count (one CTA).
cudaError_t launch_compact(const uint32_t *bitmap, int64_t cols, int32_t *col_idx, int32_t *count,
                           cudaStream_t stream);

enum class Epilogue { MixedFp16, RawInt32 };

struct GemmArgs {
    const int8_t *A;     // [M x K] codes of X
    const int8_t *B;     // [N x K] codes of W
    int64_t M, N, K;
    Epilogue epi;
    // MixedFp16 epilogue inputs
    const float *sx;     // [M]
    const float *sb;     // [N]
    const void *X16;     // [M x K] fp16 (outlier values)
    const void *W16;     // [N x K] fp16 or null (then CB * SB / 127)
    const int32_t *col_idx;
    const int32_t *count;
    void *Y;             // fp16 [M x N]  (MixedFp16) or int32 [M x N] (RawInt32)
    uint32_t *status;
};

cudaError_t launch_gemm(const GemmArgs &args, const DeviceInfo &dev, cudaStream_t stream);

} // namespace llmint8
