// Host-side interfaces between the C-ABI front end and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "llmint8.h"

namespace llmint8 {

// Decode (M <= kDecodeMaxM tokens) runs as one fused kernel with at most
// kDecodeMaxCtas CTAs.
constexpr int kDecodeMaxM = 32;
constexpr int kDecodeMaxCtas = 160;
constexpr int kHeaderBytes = 256;
constexpr size_t kSetWords = (LLMINT8_MAX_K + 31) / 32; // bitmap words of the widest X
// Outlier columns whose operands the prefill GEMM's epilogue reads from
// per-call gathered copies (more columns: it gathers them in place).
constexpr int kGatherCols = 32;
// Stream-K slots of the CTA-pair GEMM: one per pair (two CTAs x 128 rows x
// up to 256 int32 columns) and a ready flag per CTA.
constexpr int kSkMaxPairs = 80;
constexpr size_t kSkSlotBytes = 2 * 128 * 256 * 4;
// Row strides (in floats) of the gathered copies: the W side leaves room for
// a whole last tile (up to 256 columns past N), both are 16-byte multiples.
inline int64_t gather_stride_n(int64_t N) { return (N + 256 + 3) / 4 * 4; }
inline int64_t gather_stride_m(int64_t M) { return (M + 3) / 4 * 4; }

// Workspace layout (byte offsets; every region 256-byte aligned):
//   [0]      uint32 status word (bits LLMINT8_DEV_*)
//   [4]      int32  |O| (outlier column count)
//   [8]      uint64 grid barrier: arrival count (low half), generation (high
//            half); never cleared by the library after workspace_init
//   [16]     uint32 late-outlier flag, [20] decode outlier-list flag
//   [24]     uint32 calls of the shared-memory quantizer so far
//   [32]     uint64 arrivals at the shared-memory quantizer's grid barrier so
//            far (one per CTA per call: a multiple of the grid between calls)
//   [256]    uint32 two outlier bitmaps [2][kSetWords] of the shared-memory
//            quantizer: call n ORs into set[n & 1] and clears set[(n+1) & 1]
//            for the next call. Their place and size depend on no shape, so
//            that whatever shapes share the workspace nothing else is
//            written there.
//   ...      uint32 outlier bitmap [ceil(K/32)]
//   ...      int32  ascending outlier columns [K]
//   ...      fp32   SX [M]
//   ...      int8   CX [M x K]
//   decode only (1 <= M <= kDecodeMaxM), every entry rewritten by each call:
//   ...      uint8  outlier mask per 8 columns [K/8]
//   ...      fp32   partial row maxima [kDecodeMaxM x kDecodeMaxCtas]
//   ...      int32  partial accumulators per CTA [kDecodeMaxCtas x kDecodeMaxM x 128]
//   ...      uint32 partial-ready flags per CTA [kDecodeMaxCtas] (tagged with the
//            call's grid-barrier generation, so never cleared)
//   prefill GEMM (gather_n > 0), rewritten by each call before it is read:
//   ...      fp32   W's outlier columns, column-major [kGatherCols x np] (np = gather_stride_n(N))
//   ...      fp32   SB, zero-padded [np]
//   ...      fp32   X's outlier columns, column-major [kGatherCols x mp] (mp = gather_stride_m(M))
//   CTA-pair GEMM (gather_n > 0 and M >= 256):
//   ...      int32  stream-K partial accumulators [kSkMaxPairs] x kSkSlotBytes, rewritten
//            by each call before they are read
//   ...      uint32 stream-K ready flags [kSkMaxPairs x 2]: raised (1) by the parking CTA,
//            cleared by the CTA that reads the partial, so 0 between calls
struct Workspace {
    uint32_t *status;
    int32_t *count;
    uint32_t *sync;
    uint32_t *bitmap;
    uint32_t *sets;   // [2][kSetWords]
    uint32_t *calls;
    unsigned long long *arrivals;
    int32_t *col_idx;
    float *sx;
    int8_t *cx;
    uint8_t *hitmask;
    float *prow;
    int32_t *slots;
    uint32_t *pflags;
    float *wt_t;      // null without the gather regions
    float *sb_p;
    float *xo_t;
    int64_t np, mp;
    int32_t *sk_part; // null without the stream-K regions
    uint32_t *sk_flag;
    size_t bytes;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Shapes that llmint8_matmul_mixed runs with the fused decode kernel.
inline bool decode_shape(int64_t M, int64_t N) { return M >= 1 && M <= kDecodeMaxM && N >= 1; }

// Lay out (base != null) or size a workspace; `decode` adds the regions of
// the fused decode kernel, gather_n > 0 those of the prefill GEMM's gathered
// outlier operands for an N-row weight.
inline size_t carve(char *base, int64_t M, int64_t K, bool with_codes, bool decode, Workspace *ws,
                    int64_t gather_n = 0)
{
    size_t off = 0;
    auto take = [&](size_t n) {
        size_t o = off;
        off = align256(off + n);
        return base ? base + o : nullptr;
    };
    char *hdr = take(kHeaderBytes);
    char *tg = take(kSetWords * 8);
    size_t nwords = (size_t)((K + 31) / 32);
    char *bm = take(nwords * 4);
    char *ci = take((size_t)K * 4);
    char *sx = with_codes ? take((size_t)M * 4) : nullptr;
    char *cx = with_codes ? take((size_t)M * (size_t)K) : nullptr;
    char *hm = decode ? take((size_t)(K / 8)) : nullptr;
    char *pr = decode ? take((size_t)kDecodeMaxCtas * kDecodeMaxM * 4) : nullptr;
    char *sl = decode ? take((size_t)kDecodeMaxCtas * kDecodeMaxM * 128 * 4) : nullptr;
    char *pf = decode ? take((size_t)kDecodeMaxCtas * 4) : nullptr;
    const int64_t np = gather_n > 0 ? gather_stride_n(gather_n) : 0;
    const int64_t mp = gather_n > 0 ? gather_stride_m(M) : 0;
    char *wt = gather_n > 0 ? take((size_t)kGatherCols * np * 4) : nullptr;
    char *sp = gather_n > 0 ? take((size_t)np * 4) : nullptr;
    char *xo = gather_n > 0 ? take((size_t)kGatherCols * mp * 4) : nullptr;
    const bool sk = gather_n > 0 && M >= 256;
    char *skp = sk ? take((size_t)kSkMaxPairs * kSkSlotBytes) : nullptr;
    char *skf = sk ? take((size_t)kSkMaxPairs * 2 * 4) : nullptr;
    if (ws) {
        ws->status = reinterpret_cast<uint32_t *>(hdr);
        ws->count = hdr ? reinterpret_cast<int32_t *>(hdr + 4) : nullptr;
        ws->sync = hdr ? reinterpret_cast<uint32_t *>(hdr + 8) : nullptr;
        ws->bitmap = reinterpret_cast<uint32_t *>(bm);
        ws->sets = reinterpret_cast<uint32_t *>(tg);
        ws->calls = hdr ? reinterpret_cast<uint32_t *>(hdr + 24) : nullptr;
        ws->arrivals = hdr ? reinterpret_cast<unsigned long long *>(hdr + 32) : nullptr;
        ws->col_idx = reinterpret_cast<int32_t *>(ci);
        ws->sx = reinterpret_cast<float *>(sx);
        ws->cx = reinterpret_cast<int8_t *>(cx);
        ws->hitmask = reinterpret_cast<uint8_t *>(hm);
        ws->prow = reinterpret_cast<float *>(pr);
        ws->slots = reinterpret_cast<int32_t *>(sl);
        ws->pflags = reinterpret_cast<uint32_t *>(pf);
        ws->wt_t = reinterpret_cast<float *>(wt);
        ws->sb_p = reinterpret_cast<float *>(sp);
        ws->xo_t = reinterpret_cast<float *>(xo);
        ws->np = np;
        ws->mp = mp;
        ws->sk_part = reinterpret_cast<int32_t *>(skp);
        ws->sk_flag = reinterpret_cast<uint32_t *>(skf);
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

// The smallest fp16 value >= t, so that for fp16 x, |x| >= t exactly when
// |x| >= threshold_fp16(t) (+inf when no finite value qualifies, 0 for t <= 0).
__half threshold_fp16(float t);

// The quantizer for an X whose rows fit in the shared memory of one CTA per
// SM (one read of X, one grid barrier, nothing to clear before the call):
// `sets`/`calls`/`arrivals` are the workspace's two bitmaps, call counter and
// barrier arrival counter,
// bitmap_out (may be null) receives the outlier bitmap, col_idx/count the
// ascending outlier columns. With `zero` the codes are the zero-point ones
// (as launch_quantize_asym writes them against the complete set): absmax
// then receives the scale s and zero the zero point of each row.
bool quantize_smem_fits(int64_t rows, int64_t cols, const DeviceInfo &dev);
cudaError_t launch_quantize_smem(const void *X, int64_t rows, int64_t cols, float t, int8_t *codes, float *absmax,
                                 uint32_t *bitmap_out, uint32_t *sets, uint32_t *calls,
                                 unsigned long long *arrivals, int32_t *col_idx, int32_t *count,
                                 uint32_t *status, const DeviceInfo &dev, cudaStream_t stream,
                                 int32_t *zero = nullptr);

// Zero-point codes of X's rows against a complete outlier bitmap (null: no
// outliers): codes int8 (q - 128), scale s and zero point z per row.
cudaError_t launch_quantize_asym(const void *X, int64_t rows, int64_t cols, const uint32_t *bitmap, int8_t *codes,
                                 float *scale, int32_t *zero, const DeviceInfo &dev, cudaStream_t stream);
// R[j] = sum of the int8 codes of row j of CB [N x K] (K a multiple of 16).
cudaError_t launch_code_row_sums(const int8_t *CB, int64_t N, int64_t K, int32_t *R, const DeviceInfo &dev,
                                 cudaStream_t stream);

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
    const void *bias;    // fp16 [N] or null, added after dequantization
    int act;             // LLMINT8_ACT_* applied after the bias
    void *Y;             // fp16 [M x N]  (MixedFp16) or int32 [M x N] (RawInt32)
    uint32_t *status;
    // Zero-point codes of X (null: absmax codes): sx then holds the scale s
    // per row, zx the zero point per row, rsum the code row sums of B.
    const int32_t *zx;
    const int32_t *rsum;
    // MixedFp16 epilogue only: 1 stores Y as fp32 [M x N] (a partial sum of a
    // tensor-parallel row split), 0 as fp16.
    int out_f32;
    // Gathered outlier operands (launch_gather_outliers; null: the epilogue
    // gathers W's and X's outlier values in place).
    const float *wt_t, *sb_p, *xo_t;
    int64_t np, mp;
    // Stream-K slots and flags of the CTA-pair GEMM (null: whole tiles only).
    int32_t *sk_part;
    uint32_t *sk_flag;
};

cudaError_t launch_gemm(const GemmArgs &args, const DeviceInfo &dev, cudaStream_t stream);

// Before the prefill GEMM, once per call: W's outlier columns (the fp16 W, or
// CB * SB / 127 per row) and X's, column-major into the workspace's gather
// regions, and SB zero-padded, when |O| <= kGatherCols. Launched as a
// programmatic dependent of the quantizer (it waits for its outlier list).
cudaError_t launch_gather_outliers(const GemmArgs &args, float *wt_t, float *sb_p, float *xo_t, int64_t np,
                                   int64_t mp, const DeviceInfo &dev, cudaStream_t stream);

// The whole LLM.int8() linear for at most kDecodeMaxM tokens in one kernel:
// outlier detection, quantization of X, the int8 product streamed over all
// SMs, dequantization and the outlier product.
struct DecodeArgs {
    const void *X;       // [M x K] fp16
    int64_t M, N, K;
    float t;             // threshold (0: no decomposition)
    const int8_t *CB;    // [N x K]
    const float *sb;     // [N]
    const void *W16;     // [N x K] fp16 or null
    const void *bias;    // fp16 [N] or null
    int act;             // LLMINT8_ACT_*
    void *Y;             // [M x N] fp16
    int32_t *acc_out;    // [M x N] int32 products (before dequantization), or null
    Workspace ws;
};

bool decode_fused_fits(int64_t M, int64_t N, int64_t K, const DeviceInfo &dev);
cudaError_t launch_decode(const DecodeArgs &args, const DeviceInfo &dev, cudaStream_t stream);

// Row-major int8 [rows x K] as a 2-D TMA tensor map (128-byte x box_rows box,
// 128-byte swizzle, zero fill out of bounds); cached per device and buffer.
bool make_map_i8(CUtensorMap *map, int device, const void *base, int64_t rows, int64_t K, int box_rows);

} // namespace llmint8
