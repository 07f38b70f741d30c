// C-ABI front end: argument checks, workspace layout and launch order for the
// LLM.int8() linear. Argument errors return before anything is queued.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "llmint8.h"
#include "internal.h"

namespace llmint8 {

cudaError_t device_info(DeviceInfo *out)
{
    static std::mutex mu;
    static DeviceInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && have[dev]) {
        *out = cache[dev];
        return cudaSuccess;
    }
    DeviceInfo d{};
    d.device = dev;
    if ((e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
        cudaSuccess)
        return e;
    if (dev >= 0 && dev < 64) {
        cache[dev] = d;
        have[dev] = true;
    }
    *out = d;
    return cudaSuccess;
}

} // namespace llmint8

using namespace llmint8;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Thresholds that switch the decomposition off: t <= 0, +inf, NaN.
float effective_threshold(float t)
{
    if (!(t > 0.f) || std::isinf(t))
        return 0.f;
    return t;
}

llmint8_status check_k(int64_t K)
{
    if (K <= 0 || K % 16 != 0 || K > LLMINT8_MAX_K)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    return LLMINT8_OK;
}

llmint8_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA; }

// The intermediate results a caller asked for in `dbg`: the raw int32
// accumulators (with `run_acc`, one more int8 GEMM of the same codes; the
// decode kernel writes them itself) and copies of the codes, row absmax and
// outlier columns from the workspace.
llmint8_status copy_debug(const llmint8_debug *dbg, const Workspace &ws, int64_t M, int64_t N, int64_t K,
                          const int8_t *CB, const float *SCB, const void *X_f16, const void *W_f16, bool run_acc,
                          const DeviceInfo &dev, cudaStream_t stream)
{
    if (!dbg)
        return LLMINT8_OK;
    if (dbg->acc && run_acc) {
        GemmArgs r{};
        r.A = ws.cx;
        r.B = CB;
        r.M = M;
        r.N = N;
        r.K = K;
        r.sx = ws.sx;
        r.sb = SCB;
        r.X16 = X_f16;
        r.W16 = W_f16;
        r.col_idx = ws.col_idx;
        r.count = ws.count;
        r.status = ws.status;
        r.epi = Epilogue::RawInt32;
        r.Y = dbg->acc;
        if (launch_gemm(r, dev, stream) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
    }
    if (dbg->codes &&
        cudaMemcpyAsync(dbg->codes, ws.cx, (size_t)M * K, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (dbg->row_absmax &&
        cudaMemcpyAsync(dbg->row_absmax, ws.sx, (size_t)M * 4, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (dbg->col_idx &&
        cudaMemcpyAsync(dbg->col_idx, ws.col_idx, (size_t)K * 4, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (dbg->count && cudaMemcpyAsync(dbg->count, ws.count, 4, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    return LLMINT8_OK;
}

// The fused-epilogue GEMM of a linear. Prefill shapes (more than
// kDecodeMaxM rows) with the workspace's gather regions first copy the outlier
// operands into them, so that the epilogue stages each tile by bulk copies.
cudaError_t gather_then_gemm(GemmArgs g, const Workspace &ws, const DeviceInfo &dev, cudaStream_t stream)
{
    if (ws.wt_t && g.M > kDecodeMaxM) {
        cudaError_t e = launch_gather_outliers(g, ws.wt_t, ws.sb_p, ws.xo_t, ws.np, ws.mp, dev, stream);
        if (e != cudaSuccess)
            return e;
        g.wt_t = ws.wt_t;
        g.sb_p = ws.sb_p;
        g.xo_t = ws.xo_t;
        g.np = ws.np;
        g.mp = ws.mp;
    }
    g.sk_part = ws.sk_part;
    g.sk_flag = ws.sk_flag;
    return launch_gemm(g, dev, stream);
}

} // namespace

extern "C" {

const char *llmint8_status_string(int status)
{
    switch (status) {
    case LLMINT8_OK: return "LLMINT8_OK";
    case LLMINT8_ERR_INVALID_ARG: return "LLMINT8_ERR_INVALID_ARG: null pointer, negative size or bad flag";
    case LLMINT8_ERR_ALIGNMENT: return "LLMINT8_ERR_ALIGNMENT: device pointers must be 16-byte aligned";
    case LLMINT8_ERR_UNSUPPORTED_SHAPE:
        return "LLMINT8_ERR_UNSUPPORTED_SHAPE: K must be a positive multiple of 16 and at most 133143, sizes "
               "below 2^31";
    case LLMINT8_ERR_WORKSPACE: return "LLMINT8_ERR_WORKSPACE: workspace too small";
    case LLMINT8_ERR_CUDA: return "LLMINT8_ERR_CUDA: a CUDA call or kernel launch failed";
    case LLMINT8_ERR_DEVICE: return "LLMINT8_ERR_DEVICE: a kernel reported a failure in the status word";
    default: return "LLMINT8_ERR_UNKNOWN";
    }
}

size_t llmint8_quantize_workspace_size(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0)
        return 0;
    return carve(nullptr, rows, cols, false, false, nullptr);
}

size_t llmint8_workspace_size(int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K < 0)
        return 0;
    const bool dec = decode_shape(M, N);
    return carve(nullptr, M, K, true, dec, nullptr, dec ? 0 : N);
}

size_t llmint8_workspace_size_fp16w(int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K < 0)
        return 0;
    return align256(llmint8_workspace_size(M, N, K)) + align256((size_t)N * (size_t)K) + align256((size_t)N * 4);
}

llmint8_status llmint8_workspace_init(void *workspace, size_t ws_bytes, llmint8_stream_t stream)
{
    if (!workspace || ws_bytes < 256)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(workspace))
        return LLMINT8_ERR_ALIGNMENT;
    return cuda_status(cudaMemsetAsync(workspace, 0, ws_bytes, stream));
}

llmint8_status llmint8_read_status(void *workspace, size_t ws_bytes, int clear, uint32_t *out)
{
    if (!workspace || !out || ws_bytes < 256)
        return LLMINT8_ERR_INVALID_ARG;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(out, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear)
        e = cudaMemset(workspace, 0, sizeof(uint32_t));
    if (e != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    return *out ? LLMINT8_ERR_DEVICE : LLMINT8_OK;
}

llmint8_status llmint8_quantize_rowwise(const void *X_f16, int64_t rows, int64_t cols, float threshold,
                                        int8_t *codes, float *row_absmax, uint32_t *outlier_bitmap,
                                        void *workspace, size_t ws_bytes, llmint8_stream_t stream)
{
    if (rows < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_k(cols);
    if (st != LLMINT8_OK)
        return st;
    if (rows > INT32_MAX || rows * cols > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    const float t = effective_threshold(threshold);
    if (!X_f16 || !codes || !row_absmax || !workspace || (t > 0.f && !outlier_bitmap))
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X_f16) || !aligned16(codes) || !aligned16(row_absmax) || !aligned16(workspace) ||
        (outlier_bitmap && !aligned16(outlier_bitmap)))
        return LLMINT8_ERR_ALIGNMENT;
    Workspace ws;
    const size_t need = carve(static_cast<char *>(workspace), rows, cols, false, false, &ws);
    if (ws_bytes < need)
        return LLMINT8_ERR_WORKSPACE;
    if (rows == 0) // no rows, no outlier columns: the bitmap is still written
        return outlier_bitmap ? cuda_status(cudaMemsetAsync(outlier_bitmap, 0, (size_t)((cols + 31) / 32) * 4, stream))
                              : LLMINT8_OK;
    DeviceInfo dev;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (quantize_smem_fits(rows, cols, dev)) {
        // X fits in shared memory: one kernel, nothing to clear first.
        e = launch_quantize_smem(X_f16, rows, cols, t, codes, row_absmax, outlier_bitmap, ws.sets, ws.calls,
                                 ws.arrivals, ws.col_idx, ws.count, ws.status, dev, stream);
        return cuda_status(e);
    }
    // The streaming quantizer ORs into the caller's bitmap: clear it. (Its
    // other state clears itself; the barrier word keeps its generation.)
    const size_t nwords = (size_t)((cols + 31) / 32);
    if (outlier_bitmap) {
        if ((e = cudaMemsetAsync(outlier_bitmap, 0, nwords * 4, stream)) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
    }
    e = launch_quantize(X_f16, rows, cols, t, codes, row_absmax, outlier_bitmap, ws.col_idx, ws.count, ws.sync,
                        ws.status, dev, stream);
    return cuda_status(e);
}

llmint8_status llmint8_find_outlier_cols(const uint32_t *outlier_bitmap, int64_t cols, int32_t *col_idx,
                                         int32_t *d_count, int32_t *h_count, llmint8_stream_t stream)
{
    if (cols <= 0 || cols > INT32_MAX - 32)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!outlier_bitmap || !col_idx || !d_count)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(outlier_bitmap) || !aligned16(col_idx) || (reinterpret_cast<uintptr_t>(d_count) & 3u))
        return LLMINT8_ERR_ALIGNMENT;
    if ((cols + 31) / 32 * 4 > 200 * 1024)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    cudaError_t e = launch_compact(outlier_bitmap, cols, col_idx, d_count, stream);
    if (e != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (h_count) {
        if ((e = cudaMemcpyAsync(h_count, d_count, sizeof(int32_t), cudaMemcpyDeviceToHost, stream)) !=
            cudaSuccess)
            return LLMINT8_ERR_CUDA;
        if ((e = cudaStreamSynchronize(stream)) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
    }
    return LLMINT8_OK;
}

llmint8_status llmint8_matmul_mixed(const void *X_f16, int64_t M, int64_t K, const int8_t *CB,
                                    const float *SCB, const void *W_f16, int64_t N, float threshold,
                                    void *Y_f16, void *workspace, size_t ws_bytes, const llmint8_debug *dbg,
                                    llmint8_stream_t stream)
{
    return llmint8_matmul_mixed_ex(X_f16, M, K, CB, SCB, W_f16, N, threshold, nullptr, LLMINT8_ACT_NONE, Y_f16,
                                   workspace, ws_bytes, dbg, stream);
}

llmint8_status llmint8_matmul_mixed_ex(const void *X_f16, int64_t M, int64_t K, const int8_t *CB,
                                       const float *SCB, const void *W_f16, int64_t N, float threshold,
                                       const void *bias_f16, int activation, void *Y_f16, void *workspace,
                                       size_t ws_bytes, const llmint8_debug *dbg, llmint8_stream_t stream)
{
    if (M < 0 || N < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_k(K);
    if (st != LLMINT8_OK)
        return st;
    if (M > INT32_MAX || N > INT32_MAX || M * K > (int64_t)1 << 40 || N * K > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!X_f16 || !CB || !SCB || !Y_f16 || !workspace)
        return LLMINT8_ERR_INVALID_ARG;
    if (activation != LLMINT8_ACT_NONE && activation != LLMINT8_ACT_GELU_TANH)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X_f16) || !aligned16(CB) || !aligned16(SCB) || !aligned16(Y_f16) || !aligned16(workspace) ||
        (W_f16 && !aligned16(W_f16)) || (bias_f16 && !aligned16(bias_f16)))
        return LLMINT8_ERR_ALIGNMENT;
    if (dbg) {
        if ((dbg->codes && !aligned16(dbg->codes)) || (dbg->row_absmax && !aligned16(dbg->row_absmax)) ||
            (dbg->col_idx && !aligned16(dbg->col_idx)) || (dbg->acc && !aligned16(dbg->acc)) ||
            (dbg->count && (reinterpret_cast<uintptr_t>(dbg->count) & 3u)))
            return LLMINT8_ERR_ALIGNMENT;
    }
    Workspace ws;
    const bool dec = decode_shape(M, N);
    const size_t need = carve(static_cast<char *>(workspace), M, K, true, dec, &ws, dec ? 0 : N);
    if (ws_bytes < need)
        return LLMINT8_ERR_WORKSPACE;
    if (M == 0 || N == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    const float t = effective_threshold(threshold);

    if (decode_fused_fits(M, N, K, dev)) {
        // A few tokens: the whole layer in one kernel.
        DecodeArgs d{X_f16, M, N, K, t, CB, SCB, W_f16, bias_f16, activation, Y_f16, dbg ? dbg->acc : nullptr, ws};
        if (dbg && dbg->gemm_begin &&
            cudaEventRecord(static_cast<cudaEvent_t>(dbg->gemm_begin), stream) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
        if ((e = launch_decode(d, dev, stream)) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
        if (dbg && dbg->gemm_end &&
            cudaEventRecord(static_cast<cudaEvent_t>(dbg->gemm_end), stream) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
        return copy_debug(dbg, ws, M, N, K, CB, SCB, X_f16, W_f16, false, dev, stream);
    }

    if (quantize_smem_fits(M, K, dev)) {
        // X fits in shared memory: one kernel, nothing to clear first.
        if ((e = launch_quantize_smem(X_f16, M, K, t, ws.cx, ws.sx, nullptr, ws.sets, ws.calls, ws.arrivals,
                                      ws.col_idx, ws.count, ws.status, dev, stream)) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
    } else {
        // The streaming quantizer ORs into the bitmap: clear it. (Its other
        // state clears itself; the barrier word keeps its generation.)
        if ((e = cudaMemsetAsync(ws.bitmap, 0, (size_t)((K + 31) / 32) * 4, stream)) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
        if ((e = launch_quantize(X_f16, M, K, t, ws.cx, ws.sx, ws.bitmap, ws.col_idx, ws.count, ws.sync,
                                 ws.status, dev, stream)) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
    }

    GemmArgs g{};
    g.A = ws.cx;
    g.B = CB;
    g.M = M;
    g.N = N;
    g.K = K;
    g.sx = ws.sx;
    g.sb = SCB;
    g.X16 = X_f16;
    g.W16 = W_f16;
    g.col_idx = ws.col_idx;
    g.count = ws.count;
    g.bias = bias_f16;
    g.act = activation;
    g.status = ws.status;
    g.epi = Epilogue::MixedFp16;
    g.Y = Y_f16;
    if (dbg && dbg->gemm_begin &&
        cudaEventRecord(static_cast<cudaEvent_t>(dbg->gemm_begin), stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if ((e = gather_then_gemm(g, ws, dev, stream)) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (dbg && dbg->gemm_end && cudaEventRecord(static_cast<cudaEvent_t>(dbg->gemm_end), stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;

    return copy_debug(dbg, ws, M, N, K, CB, SCB, X_f16, W_f16, true, dev, stream);
}

llmint8_status llmint8_matmul_mixed_fp16w(const void *X_f16, int64_t M, int64_t K, const void *W_f16, int64_t N,
                                          float threshold, const void *bias_f16, int activation, void *Y_f16,
                                          void *workspace, size_t ws_bytes, const llmint8_debug *dbg,
                                          llmint8_stream_t stream)
{
    // The checks of llmint8_matmul_mixed_ex that matter before W is quantized.
    if (M < 0 || N < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_k(K);
    if (st != LLMINT8_OK)
        return st;
    if (M > INT32_MAX || N > INT32_MAX || M * K > (int64_t)1 << 40 || N * K > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!X_f16 || !W_f16 || !Y_f16 || !workspace)
        return LLMINT8_ERR_INVALID_ARG;
    if (activation != LLMINT8_ACT_NONE && activation != LLMINT8_ACT_GELU_TANH)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X_f16) || !aligned16(W_f16) || !aligned16(Y_f16) || !aligned16(workspace) ||
        (bias_f16 && !aligned16(bias_f16)))
        return LLMINT8_ERR_ALIGNMENT;
    if (ws_bytes < llmint8_workspace_size_fp16w(M, N, K))
        return LLMINT8_ERR_WORKSPACE;
    if (M == 0 || N == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    // W's codes and row absmax live after the linear's own workspace.
    const size_t base = align256(llmint8_workspace_size(M, N, K));
    char *w = static_cast<char *>(workspace);
    int8_t *cb = reinterpret_cast<int8_t *>(w + base);
    float *sb = reinterpret_cast<float *>(w + base + align256((size_t)N * (size_t)K));
    Workspace ws;
    const bool dec = decode_shape(M, N);
    carve(w, M, K, true, dec, &ws, dec ? 0 : N);
    if (launch_quantize(W_f16, N, K, 0.f, cb, sb, nullptr, ws.col_idx, ws.count, ws.sync, ws.status, dev,
                        stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    return llmint8_matmul_mixed_ex(X_f16, M, K, cb, sb, W_f16, N, threshold, bias_f16, activation, Y_f16, workspace,
                                   base, dbg, stream);
}

llmint8_status llmint8_gemm_s8s8s32(const int8_t *A, int64_t M, const int8_t *B, int64_t N, int64_t K,
                                    int32_t *acc, void *workspace, size_t ws_bytes, llmint8_stream_t stream)
{
    if (M < 0 || N < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_k(K);
    if (st != LLMINT8_OK)
        return st;
    if (M > INT32_MAX || N > INT32_MAX)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!A || !B || !acc || !workspace)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(acc) || !aligned16(workspace))
        return LLMINT8_ERR_ALIGNMENT;
    Workspace ws;
    const bool dec = decode_shape(M, N);
    const size_t need = carve(static_cast<char *>(workspace), M, K, true, dec, &ws, dec ? 0 : N);
    if (ws_bytes < need)
        return LLMINT8_ERR_WORKSPACE;
    if (M == 0 || N == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    GemmArgs g{};
    g.sk_part = ws.sk_part;
    g.sk_flag = ws.sk_flag;
    g.A = A;
    g.B = B;
    g.M = M;
    g.N = N;
    g.K = K;
    g.epi = Epilogue::RawInt32;
    g.Y = acc;
    g.status = ws.status;
    return cuda_status(launch_gemm(g, dev, stream));
}

} // extern "C"

// ---------------------------------------------------------------- zero-point variant

namespace {

llmint8_status check_k_asym(int64_t K)
{
    if (K <= 0 || K % 16 != 0 || K > LLMINT8_MAX_K_ASYM)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    return LLMINT8_OK;
}

// Outlier detection for the zero-point path: the absmax quantizer's bitmap
// and column list (its codes and row maxima go to the given scratch and are
// overwritten by the zero-point codes right after).
cudaError_t detect_outliers(const void *X_f16, int64_t rows, int64_t cols, float t, int8_t *codes_scratch,
                            float *rowmax_scratch, uint32_t *bitmap, const Workspace &ws, const DeviceInfo &dev,
                            cudaStream_t stream)
{
    if (quantize_smem_fits(rows, cols, dev))
        return launch_quantize_smem(X_f16, rows, cols, t, codes_scratch, rowmax_scratch, bitmap, ws.sets, ws.calls,
                                    ws.arrivals, ws.col_idx, ws.count, ws.status, dev, stream);
    cudaError_t e = cudaMemsetAsync(bitmap, 0, (size_t)((cols + 31) / 32) * 4, stream);
    if (e != cudaSuccess)
        return e;
    return launch_quantize(X_f16, rows, cols, t, codes_scratch, rowmax_scratch, bitmap, ws.col_idx, ws.count,
                           ws.sync, ws.status, dev, stream);
}

} // namespace

size_t llmint8_workspace_size_asym(int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K < 0)
        return 0;
    return align256(carve(nullptr, M, K, true, false, nullptr, N)) + align256((size_t)M * 4);
}

llmint8_status llmint8_quantize_rowwise_asym(const void *X_f16, int64_t rows, int64_t cols, float threshold,
                                             int8_t *codes, float *scale, int32_t *zero, uint32_t *outlier_bitmap,
                                             void *workspace, size_t ws_bytes, llmint8_stream_t stream)
{
    if (rows < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_k_asym(cols);
    if (st != LLMINT8_OK)
        return st;
    if (rows > INT32_MAX || rows * cols > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    const float t = effective_threshold(threshold);
    if (!X_f16 || !codes || !scale || !zero || !workspace || (t > 0.f && !outlier_bitmap))
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X_f16) || !aligned16(codes) || !aligned16(scale) || !aligned16(zero) || !aligned16(workspace) ||
        (outlier_bitmap && !aligned16(outlier_bitmap)))
        return LLMINT8_ERR_ALIGNMENT;
    Workspace ws;
    const size_t need = carve(static_cast<char *>(workspace), rows, cols, false, false, &ws);
    if (ws_bytes < need)
        return LLMINT8_ERR_WORKSPACE;
    if (rows == 0) // no rows, no outlier columns: the bitmap is still written
        return outlier_bitmap ? cuda_status(cudaMemsetAsync(outlier_bitmap, 0, (size_t)((cols + 31) / 32) * 4, stream))
                              : LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (quantize_smem_fits(rows, cols, dev)) // X fits in shared memory: one kernel, one read of X
        return cuda_status(launch_quantize_smem(X_f16, rows, cols, t, codes, scale, outlier_bitmap, ws.sets, ws.calls,
                                                ws.arrivals, ws.col_idx, ws.count, ws.status, dev, stream, zero));
    cudaError_t e = cudaSuccess;
    if (t > 0.f) {
        if ((e = detect_outliers(X_f16, rows, cols, t, codes, scale, outlier_bitmap, ws, dev, stream)) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
    } else if (outlier_bitmap &&
               (e = cudaMemsetAsync(outlier_bitmap, 0, (size_t)((cols + 31) / 32) * 4, stream)) != cudaSuccess) {
        return LLMINT8_ERR_CUDA;
    }
    e = launch_quantize_asym(X_f16, rows, cols, t > 0.f ? outlier_bitmap : nullptr, codes, scale, zero, dev, stream);
    return cuda_status(e);
}

llmint8_status llmint8_code_row_sums(const int8_t *CB, int64_t N, int64_t K, int32_t *row_sums,
                                     llmint8_stream_t stream)
{
    if (N < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_k_asym(K);
    if (st != LLMINT8_OK)
        return st;
    if (N > INT32_MAX || N * K > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!CB || !row_sums)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(CB) || (reinterpret_cast<uintptr_t>(row_sums) & 3u))
        return LLMINT8_ERR_ALIGNMENT;
    if (N == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    return cuda_status(launch_code_row_sums(CB, N, K, row_sums, dev, stream));
}

llmint8_status llmint8_matmul_mixed_asym(const void *X_f16, int64_t M, int64_t K, const int8_t *CB,
                                         const float *SCB, const int32_t *CB_row_sums, const void *W_f16,
                                         int64_t N, float threshold, void *Y_f16, void *workspace, size_t ws_bytes,
                                         const llmint8_debug *dbg, llmint8_stream_t stream)
{
    if (M < 0 || N < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_k_asym(K);
    if (st != LLMINT8_OK)
        return st;
    if (M > INT32_MAX || N > INT32_MAX || M * K > (int64_t)1 << 40 || N * K > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!X_f16 || !CB || !SCB || !CB_row_sums || !Y_f16 || !workspace)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X_f16) || !aligned16(CB) || !aligned16(SCB) || !aligned16(Y_f16) || !aligned16(workspace) ||
        (W_f16 && !aligned16(W_f16)) || (reinterpret_cast<uintptr_t>(CB_row_sums) & 3u))
        return LLMINT8_ERR_ALIGNMENT;
    if (dbg) {
        if ((dbg->codes && !aligned16(dbg->codes)) || (dbg->row_absmax && !aligned16(dbg->row_absmax)) ||
            (dbg->col_idx && !aligned16(dbg->col_idx)) || (dbg->acc && !aligned16(dbg->acc)) ||
            (dbg->count && (reinterpret_cast<uintptr_t>(dbg->count) & 3u)))
            return LLMINT8_ERR_ALIGNMENT;
    }
    Workspace ws;
    const size_t base = align256(carve(static_cast<char *>(workspace), M, K, true, false, &ws, N));
    if (ws_bytes < base + align256((size_t)M * 4))
        return LLMINT8_ERR_WORKSPACE;
    int32_t *zx = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + base);
    if (M == 0 || N == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    const float t = effective_threshold(threshold);
    if (quantize_smem_fits(M, K, dev)) {
        // X fits in shared memory: detection and the zero-point codes in one kernel, one read of X
        if (launch_quantize_smem(X_f16, M, K, t, ws.cx, ws.sx, nullptr, ws.sets, ws.calls, ws.arrivals, ws.col_idx,
                                 ws.count, ws.status, dev, stream, zx) != cudaSuccess)
            return LLMINT8_ERR_CUDA;
    } else {
        if (t > 0.f) {
            if (detect_outliers(X_f16, M, K, t, ws.cx, ws.sx, ws.bitmap, ws, dev, stream) != cudaSuccess)
                return LLMINT8_ERR_CUDA;
        } else if (cudaMemsetAsync(ws.count, 0, sizeof(int32_t), stream) != cudaSuccess) {
            return LLMINT8_ERR_CUDA;
        }
        if (launch_quantize_asym(X_f16, M, K, t > 0.f ? ws.bitmap : nullptr, ws.cx, ws.sx, zx, dev, stream) !=
            cudaSuccess)
            return LLMINT8_ERR_CUDA;
    }
    GemmArgs g{};
    g.A = ws.cx;
    g.B = CB;
    g.M = M;
    g.N = N;
    g.K = K;
    g.sx = ws.sx;
    g.sb = SCB;
    g.X16 = X_f16;
    g.W16 = W_f16;
    g.col_idx = ws.col_idx;
    g.count = ws.count;
    g.status = ws.status;
    g.epi = Epilogue::MixedFp16;
    g.Y = Y_f16;
    g.zx = zx;
    g.rsum = CB_row_sums;
    if (dbg && dbg->gemm_begin &&
        cudaEventRecord(static_cast<cudaEvent_t>(dbg->gemm_begin), stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (gather_then_gemm(g, ws, dev, stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    if (dbg && dbg->gemm_end && cudaEventRecord(static_cast<cudaEvent_t>(dbg->gemm_end), stream) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    return copy_debug(dbg, ws, M, N, K, CB, SCB, X_f16, W_f16, true, dev, stream);
}
