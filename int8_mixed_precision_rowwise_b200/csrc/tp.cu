// The pieces a tensor-parallel LLM.int8() linear needs beyond the one-GPU
// layer: row quantization against an outlier set and (optionally) row absmax
// that came from other ranks, the int8 GEMM with its LLM.int8() epilogue on
// codes quantized elsewhere (fp16 or fp32 output), the last step after a sum
// across ranks (bias, activation, fp16), and the reassembly of column blocks
// after an all-gather.
//
// Method: page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
// accelerate" for the arithmetic (sections "模型量化简介", "LLM.int8() 的简要
// 总结", "MatMul 内部"); page "优化故事：Bloom 推理", section "支持 TP", for the
// deployment: every GPU owns a part of the weights, and the partial results
// are combined with NCCL all-reduces (section "唾手可得的优化").
//
// How the splits use these (each keeps the one-GPU result: same outlier set,
// same row absmax, same codes, the int32 products summed exactly per rank):
//   column split (W's output rows across ranks): every rank runs the whole
//     layer on the full X against its rows of W; outputs are column blocks,
//     reassembled by llmint8_gather_column_blocks after an all-gather.
//   row split (K across ranks): a column's outlier status depends only on that
//     column, so each rank finds its own outlier columns and the row absmax
//     over its own other columns; a max all-reduce gives the full row absmax,
//     llmint8_quantize_rowwise_given codes the rank's columns with it,
//     llmint8_matmul_codes writes an fp32 partial product, a sum all-reduce
//     adds them and llmint8_bias_act_to_f16 finishes.
//   token split (rows of X across ranks, W replicated): the outlier set is the
//     union of the ranks' sets (their bitmaps all-gathered), and each rank
//     quantizes its rows against it with llmint8_quantize_rowwise_given.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "internal.h"
#include "llmint8.h"

namespace llmint8 {
namespace {

// One warp per row. The outlier set is the OR of `nbm` bitmaps of `nwords`
// words each, kept in shared memory (CTA 0 also writes it to bitmap_out).
// Row absmax: taken from absmax_in if given, else the maximum |x| over the
// columns outside the set (written to absmax_out). Codes: rint(x * s) with
// s = 127 / absmax in fp32 (two separate roundings), 0 for set columns and
// for an all-zero row.
__global__ void __launch_bounds__(256)
    k_quant_given(const uint4 *__restrict__ X, int64_t rows, int cols, const uint32_t *__restrict__ bitmaps, int nbm,
                  const float *__restrict__ absmax_in, int8_t *__restrict__ codes, float *__restrict__ absmax_out,
                  uint32_t *__restrict__ bitmap_out)
{
    extern __shared__ uint32_t s_set[];
    const int nvec = cols >> 3, nwords = (cols + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += blockDim.x) {
        uint32_t v = 0u;
        for (int b = 0; b < nbm; ++b)
            v |= bitmaps[(int64_t)b * nwords + w];
        s_set[w] = v;
        if (blockIdx.x == 0 && bitmap_out)
            bitmap_out[w] = v;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nwarps) {
        const uint4 *xr = X + r * nvec;
        float amax;
        if (absmax_in) {
            amax = __ldg(absmax_in + r);
        } else {
            __half2 m2 = __float2half2_rn(0.f);
            for (int vi = lane; vi < nvec; vi += 32) {
                uint4 v = __ldg(xr + vi);
                const uint32_t kb = (s_set[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
                if (kb)
                    mask_known(v, kb);
                __half2 a[4];
                m2 = __hmax2(m2, vec_abs_max(v, a));
            }
            amax = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        }
        const float s = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        int8_t *cr = codes + r * (int64_t)cols;
        for (int vi = lane; vi < nvec; vi += 32) {
            uint4 v = __ldg(xr + vi);
            const uint32_t kb = (s_set[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
            if (kb)
                mask_known(v, kb);
            *reinterpret_cast<uint2 *>(cr + (int64_t)vi * 8) = codes8(v, s);
        }
        if (lane == 0 && absmax_out && !absmax_in)
            absmax_out[r] = amax;
    }
}

// Y16[i, j] = fp16(act(Y32[i, j] + bias[j])), four values a thread.
__global__ void __launch_bounds__(256) k_bias_act_to_f16(const float4 *__restrict__ Y32, int64_t n4, int N,
                                                         const __half *__restrict__ bias, int act,
                                                         uint2 *__restrict__ Y16)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 y = Y32[i];
        const int j = (int)((i * 4) % N);
        float b[4] = {0.f, 0.f, 0.f, 0.f};
        if (bias) { // N is a multiple of 4, so j .. j + 3 lie in one row
#pragma unroll
            for (int e = 0; e < 4; ++e)
                b[e] = __half2float(bias[j + e]);
        }
        __half2 lo = __floats2half2_rn(bias_act(y.x, b[0], act), bias_act(y.y, b[1], act));
        __half2 hi = __floats2half2_rn(bias_act(y.z, b[2], act), bias_act(y.w, b[3], act));
        uint2 o;
        o.x = *reinterpret_cast<uint32_t *>(&lo);
        o.y = *reinterpret_cast<uint32_t *>(&hi);
        Y16[i] = o;
    }
}

// dst[i, p * Nr + j] = src[p][i][j] for fp16 blocks [P][M][Nr], 16 bytes
// (8 values) a thread.
__global__ void __launch_bounds__(256) k_gather_column_blocks(const uint4 *__restrict__ src, int64_t P, int64_t M,
                                                              int64_t nr8, uint4 *__restrict__ dst)
{
    const int64_t total = P * M * nr8;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = e % nr8, i = (e / nr8) % M, p = e / (nr8 * M);
        dst[(i * P + p) * nr8 + j] = src[e];
    }
}

unsigned grid_for(int64_t work, int per_block, const DeviceInfo &dev)
{
    const int64_t want = (work + per_block - 1) / per_block;
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)dev.num_sms * 8));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

llmint8_status check_cols(int64_t cols)
{
    if (cols <= 0 || cols % 16 != 0 || cols > LLMINT8_MAX_K)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    return LLMINT8_OK;
}

} // namespace
} // namespace llmint8

using namespace llmint8;

extern "C" {

llmint8_status llmint8_quantize_rowwise_given(const void *X_f16, int64_t rows, int64_t cols,
                                              const uint32_t *outlier_bitmaps, int n_bitmaps,
                                              const float *row_absmax_in, int8_t *codes, float *row_absmax_out,
                                              uint32_t *bitmap_out, llmint8_stream_t stream)
{
    if (rows < 0 || n_bitmaps < 0 || n_bitmaps > 4096)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_cols(cols);
    if (st != LLMINT8_OK)
        return st;
    if (rows > INT32_MAX || rows * cols > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    // (with no rows, X, codes and the absmax pointers may be NULL: empty tensors)
    if ((rows > 0 && (!X_f16 || !codes || (!row_absmax_in && !row_absmax_out))) ||
        (n_bitmaps > 0 && !outlier_bitmaps))
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X_f16) || !aligned16(codes) || (outlier_bitmaps && !aligned16(outlier_bitmaps)) ||
        (row_absmax_in && !aligned16(row_absmax_in)) || (row_absmax_out && !aligned16(row_absmax_out)) ||
        (bitmap_out && !aligned16(bitmap_out)))
        return LLMINT8_ERR_ALIGNMENT;
    if (rows == 0 && !bitmap_out) // (with bitmap_out the kernel still writes the union)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    const int nwords = (int)((cols + 31) / 32);
    const size_t smem = (size_t)nwords * 4;
    k_quant_given<<<grid_for(rows, 8, dev), 256, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(X_f16), rows, (int)cols, outlier_bitmaps, n_bitmaps, row_absmax_in, codes,
        row_absmax_out, bitmap_out);
    return cudaGetLastError() == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

llmint8_status llmint8_matmul_codes(const int8_t *CX, const float *SX, const void *X_f16, int64_t M, int64_t K,
                                    const int8_t *CB, const float *SCB, const void *W_f16, int64_t N,
                                    const int32_t *col_idx, const int32_t *d_count, const void *bias_f16,
                                    int activation, int out_dtype, void *Y, void *workspace, size_t ws_bytes,
                                    llmint8_stream_t stream)
{
    if (M < 0 || N < 0)
        return LLMINT8_ERR_INVALID_ARG;
    llmint8_status st = check_cols(K);
    if (st != LLMINT8_OK)
        return st;
    if (M > INT32_MAX || N > INT32_MAX || M * K > (int64_t)1 << 40 || N * K > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!CX || !SX || !X_f16 || !CB || !SCB || !col_idx || !d_count || !Y || !workspace)
        return LLMINT8_ERR_INVALID_ARG;
    if (activation != LLMINT8_ACT_NONE && activation != LLMINT8_ACT_GELU_TANH)
        return LLMINT8_ERR_INVALID_ARG;
    if (out_dtype != LLMINT8_OUT_F16 && out_dtype != LLMINT8_OUT_F32)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(CX) || !aligned16(SX) || !aligned16(X_f16) || !aligned16(CB) || !aligned16(SCB) ||
        !aligned16(col_idx) || (reinterpret_cast<uintptr_t>(d_count) & 3u) || !aligned16(Y) || !aligned16(workspace) ||
        (W_f16 && !aligned16(W_f16)) || (bias_f16 && !aligned16(bias_f16)))
        return LLMINT8_ERR_ALIGNMENT;
    if (ws_bytes < kHeaderBytes)
        return LLMINT8_ERR_WORKSPACE;
    if (M == 0 || N == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    GemmArgs g{};
    g.A = CX;
    g.B = CB;
    g.M = M;
    g.N = N;
    g.K = K;
    g.sx = SX;
    g.sb = SCB;
    g.X16 = X_f16;
    g.W16 = W_f16;
    g.col_idx = col_idx;
    g.count = d_count;
    g.bias = bias_f16;
    g.act = activation;
    g.status = static_cast<uint32_t *>(workspace);
    g.epi = Epilogue::MixedFp16;
    g.Y = Y;
    g.out_f32 = out_dtype == LLMINT8_OUT_F32 ? 1 : 0;
    return launch_gemm(g, dev, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? LLMINT8_OK
                                                                                       : LLMINT8_ERR_CUDA;
}

llmint8_status llmint8_bias_act_to_f16(const float *Y32, int64_t M, int64_t N, const void *bias_f16, int activation,
                                       void *Y_f16, llmint8_stream_t stream)
{
    if (M < 0 || N < 0)
        return LLMINT8_ERR_INVALID_ARG;
    if (M > INT32_MAX || N > INT32_MAX)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (N % 4 != 0)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!Y32 || !Y_f16)
        return LLMINT8_ERR_INVALID_ARG;
    if (activation != LLMINT8_ACT_NONE && activation != LLMINT8_ACT_GELU_TANH)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(Y32) || !aligned16(Y_f16) || (bias_f16 && !aligned16(bias_f16)))
        return LLMINT8_ERR_ALIGNMENT;
    if (M == 0 || N == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    const int64_t n4 = M * N / 4;
    k_bias_act_to_f16<<<grid_for(n4, 256, dev), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float4 *>(Y32), n4, (int)N, reinterpret_cast<const __half *>(bias_f16), activation,
        reinterpret_cast<uint2 *>(Y_f16));
    return cudaGetLastError() == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

llmint8_status llmint8_gather_column_blocks(const void *src_f16, int64_t P, int64_t M, int64_t Nr, void *dst_f16,
                                            llmint8_stream_t stream)
{
    if (P < 0 || M < 0 || Nr < 0)
        return LLMINT8_ERR_INVALID_ARG;
    if (Nr % 8 != 0 || P * M * Nr > (int64_t)1 << 40)
        return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (!src_f16 || !dst_f16)
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(src_f16) || !aligned16(dst_f16))
        return LLMINT8_ERR_ALIGNMENT;
    if (P == 0 || M == 0 || Nr == 0)
        return LLMINT8_OK;
    DeviceInfo dev;
    if (device_info(&dev) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    const int64_t nr8 = Nr / 8;
    k_gather_column_blocks<<<grid_for(P * M * nr8, 256, dev), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(src_f16), P, M, nr8, reinterpret_cast<uint4 *>(dst_f16));
    return cudaGetLastError() == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

} // extern "C"
