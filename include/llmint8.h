/*
 * llmint8 — the LLM.int8() mixed-precision linear layer Y = X . W^T on B200
 * (sm_100a), as a plain C ABI.
 *
 * Source of the method: the page "Hugging Face 将 LLM.int8() 8-bit 量化集成进
 * transformers 与 accelerate" (a translation of the Hugging Face blog post "A
 * Gentle Introduction to 8-bit Matrix Multiplication for transformers at
 * scale"). Sections cited below:
 *   [Q]  "模型量化简介" (Introduction to model quantization): absmax
 *        quantization (scale 127 / absmax, round, int8 range [-127, 127]) and
 *        vector-wise quantization dequantized by the outer product of the row
 *        and column absmax vectors.
 *   [S]  "LLM.int8() 的简要总结" (A gentle summary of LLM.int8()): the three
 *        steps - outlier columns of the hidden states to fp16, the rest to an
 *        int8 matmul, dequantize and add.
 *   [M]  "MatMul 内部" (Inside the MatMul): threshold "magnitude 6 or greater",
 *        hidden states quantized per row, weights per output row.
 *   [U]  "用法" (Usage): the int8 weight CB and its row statistics SCB, and the
 *        recovery CB * SCB / 127 of fp16 weights for the outlier matmul.
 *
 * Conventions for every entry point:
 *   - Pointers marked (device) are CUDA device pointers the CALLER allocated
 *     and owns. The library never allocates or frees memory, and keeps no
 *     state besides cached device properties and function pointers.
 *   - All device pointers must be 16-byte aligned; matrices are dense and
 *     row-major with the last dimension contiguous. K (cols) must be a
 *     multiple of 16 and at most LLMINT8_MAX_K (so int32 sums of int8
 *     products cannot overflow: 133143 * 127^2 < 2^31).
 *   - Work is queued on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and returns without waiting, except where stated.
 *   - Argument errors are returned before anything is queued. A failed launch
 *     returns LLMINT8_ERR_CUDA. Kernels never trap: a bounded wait that runs
 *     out sets a bit in the workspace status word. Compute calls only queue
 *     work, so they return LLMINT8_OK before any kernel has run and never
 *     report such a failure themselves; llmint8_read_status (after the
 *     stream has finished) is the one place it shows, as LLMINT8_ERR_DEVICE.
 *   - fp16 inputs must be finite; NaN or Inf inputs are outside the contract.
 *   - M (rows) == 0 or N == 0 is a no-op that returns LLMINT8_OK.
 */
#ifndef LLMINT8_H
#define LLMINT8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LLMINT8_API __attribute__((visibility("default")))
#else
#define LLMINT8_API
#endif

typedef struct CUstream_st *llmint8_stream_t; /* same type as cudaStream_t */

typedef enum llmint8_status {
    LLMINT8_OK = 0,
    LLMINT8_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad flag */
    LLMINT8_ERR_ALIGNMENT = 2,         /* a pointer is not 16-byte aligned */
    LLMINT8_ERR_UNSUPPORTED_SHAPE = 3, /* K % 16 != 0, K > LLMINT8_MAX_K, sizes past 2^31 */
    LLMINT8_ERR_WORKSPACE = 4,         /* workspace smaller than the *_workspace_size() answer */
    LLMINT8_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    LLMINT8_ERR_DEVICE = 6             /* a kernel reported a failure in the status word */
} llmint8_status;

#define LLMINT8_MAX_K 133143
/* Device status word bits (llmint8_read_status). */
#define LLMINT8_DEV_TIMEOUT_PRODUCER 0x1u
#define LLMINT8_DEV_TIMEOUT_MMA 0x2u
#define LLMINT8_DEV_TIMEOUT_EPILOGUE 0x4u
#define LLMINT8_DEV_TIMEOUT_QUANT 0x8u
#define LLMINT8_DEV_BAD_STORE 0x10u /* an epilogue store failed its self-check and was skipped */

/* Human-readable name of a status code. Never NULL. */
LLMINT8_API const char *llmint8_status_string(int status);

/* Bytes of workspace needed by llmint8_quantize_rowwise for `rows` x `cols`. */
LLMINT8_API size_t llmint8_quantize_workspace_size(int64_t rows, int64_t cols);

/* Bytes of workspace needed by llmint8_matmul_mixed for X [M x K], W [N x K].
 * For M >= 256 it includes about 21 MB of stream-K slots: the CTA-pair GEMM
 * may split its last tiles over the SMs by K and sum the int32 parts there. */
LLMINT8_API size_t llmint8_workspace_size(int64_t M, int64_t N, int64_t K);

/* Zero a workspace (a cudaMemsetAsync). A workspace must be zeroed once before
 * its first use; every call leaves it ready for the next one. Calls of any
 * entry point and any shape may share one workspace; between calls it holds
 * the library's state (a grid-barrier generation, epoch-tagged words), so the
 * caller must not write into it. */
LLMINT8_API llmint8_status llmint8_workspace_init(void *workspace, size_t ws_bytes, llmint8_stream_t stream);

/* Synchronously read (and, if clear != 0, reset) the device status word of a
 * workspace after the stream has finished. Waits for the whole device
 * (cudaDeviceSynchronize). *out receives the word (LLMINT8_DEV_* bits). Returns
 * LLMINT8_OK when it is 0, LLMINT8_ERR_DEVICE when a kernel reported a
 * failure (its outputs are then incomplete; re-zero the workspace with
 * llmint8_workspace_init before its next use), LLMINT8_ERR_CUDA if the
 * synchronisation or the copy failed. */
LLMINT8_API llmint8_status llmint8_read_status(void *workspace, size_t ws_bytes, int clear, uint32_t *out);

/*
 * Row-wise absmax quantization with outlier-column decomposition ([Q], [M]).
 *
 *   X_f16        (device) fp16 [rows x cols], read only.
 *   threshold    t. If t > 0, column c is an outlier when some row holds
 *                |x| >= t; the outlier columns are OR-ed into outlier_bitmap,
 *                row_absmax[i] = max |x[i,c]| over the NON-outlier columns c,
 *                and codes of outlier columns are 0. If t <= 0 (or +inf) there
 *                is no decomposition: row_absmax is over the whole row.
 *   codes        (device) int8 [rows x cols] out: round-half-even(x * s) with
 *                s = 127 / row_absmax[i] computed in fp32 (0 for a zero row).
 *   row_absmax   (device) fp32 [rows] out (the "SCB" statistics of [U]).
 *   outlier_bitmap (device) uint32 [ceil(cols/32)] out, bit (c & 31) of word
 *                c >> 5 set for outlier column c. Required when t > 0; may be
 *                NULL when t <= 0 (if given, it is cleared). It is written, not
 *                accumulated: the call clears it first.
 *   workspace    (device) at least llmint8_quantize_workspace_size(rows, cols)
 *                bytes, zeroed once before first use.
 * Weight preparation (offline, [U]) is this call with t <= 0 on W [N x K]:
 * it yields CB = codes and SCB = row_absmax.
 */
LLMINT8_API llmint8_status llmint8_quantize_rowwise(const void *X_f16, int64_t rows, int64_t cols,
                                        float threshold, int8_t *codes, float *row_absmax,
                                        uint32_t *outlier_bitmap, void *workspace,
                                        size_t ws_bytes, llmint8_stream_t stream);

/*
 * The outlier column set as ascending column indices ([S] step 1).
 *   outlier_bitmap (device) uint32 [ceil(cols/32)] in (as written above).
 *   col_idx      (device) int32 [cols] out: the first *count entries are the
 *                set columns in ascending order; the rest is left untouched.
 *   d_count      (device) int32 [1] out: |O|, written on the device (no sync).
 *   h_count      (host, may be NULL) if given, the call waits for the stream
 *                and copies |O| here.
 */
LLMINT8_API llmint8_status llmint8_find_outlier_cols(const uint32_t *outlier_bitmap, int64_t cols,
                                         int32_t *col_idx, int32_t *d_count, int32_t *h_count,
                                         llmint8_stream_t stream);

/* Optional outputs of llmint8_matmul_mixed for parity checks. Every pointer is
 * a device pointer or NULL (not written). */
typedef struct llmint8_debug {
    int8_t *codes;      /* [M x K] CX: X's int8 codes after decomposition */
    float *row_absmax;  /* [M]     SX: X's row absmax over non-outlier columns */
    int32_t *col_idx;   /* [K]     ascending outlier columns (first |O| valid) */
    int32_t *count;     /* [1]     |O| */
    int32_t *acc;       /* [M x N] int32 accumulators of the int8 part (M <= 32:
                           written by the fused decode kernel itself; larger M:
                           the int8 GEMM runs a second time with a raw int32
                           epilogue) */
    void *gemm_begin;   /* cudaEvent_t or NULL: recorded on `stream` right before */
    void *gemm_end;     /* and right after the fused GEMM launch (kernel timing)  */
} llmint8_debug;

/*
 * The LLM.int8() linear: Y = X . W^T with mixed-precision decomposition
 * ([S], [M], [U]):
 *   O      = outlier columns of X at threshold t (none if t <= 0),
 *   CX, SX = row-wise int8 codes / absmax of X over the columns not in O,
 *   acc    = CX . CB^T exactly in int32 (columns in O contribute 0),
 *   Y[i,j] = fp16( acc[i,j] * SX[i] * SCB[j] / 127^2
 *                  + sum_{c in O} X[i,c] * Wt[j,c] ),   evaluated in fp32,
 * where Wt[j,c] = W_f16[j,c] if W_f16 is given ("has fp16 weights"), else
 * CB[j,c] * SCB[j] / 127 in fp32 (the recovery of [U], per output row).
 *
 *   X_f16      (device) fp16 [M x K]
 *   CB         (device) int8 [N x K], SCB (device) fp32 [N]: W's codes and row
 *              absmax, from llmint8_quantize_rowwise(W, t <= 0).
 *   W_f16      (device, may be NULL) fp16 [N x K]
 *   Y_f16      (device) fp16 [M x N] out
 *   workspace  (device) >= llmint8_workspace_size(M, N, K) bytes, zeroed once
 *              (llmint8_workspace_init). After a call that left an error bit in
 *              the status word, zero it again before the next call.
 *   dbg        (host struct of device pointers, may be NULL)
 * M <= 32 runs one fused, cooperatively launched decode
 * kernel: the outlier columns and codes of X are computed across all SMs
 * while the weight codes already stream in, W is split evenly over the SMs
 * and split tiles are summed exactly in int32. Larger M runs the quantizer
 * and then the persistent prefill GEMM (CTA pairs from M = 256; when the
 * tiles do not fill the last round, the last ones are split over the pairs
 * by K and their int32 parts summed exactly through the workspace).
 * Calls that share a workspace must be ordered (one stream, or events).
 */
LLMINT8_API llmint8_status llmint8_matmul_mixed(const void *X_f16, int64_t M, int64_t K, const int8_t *CB,
                                    const float *SCB, const void *W_f16, int64_t N,
                                    float threshold, void *Y_f16, void *workspace,
                                    size_t ws_bytes, const llmint8_debug *dbg,
                                    llmint8_stream_t stream);

/* Activations the epilogue can apply after the bias. */
typedef enum {
    LLMINT8_ACT_NONE = 0,
    /* BLOOM's GELU, tanh form (page "优化故事：Bloom 推理", section
     * "唾手可得的优化"): g(y) = 0.5 y (1 + tanh(0.79788456 y (1 + 0.044715 y^2))). */
    LLMINT8_ACT_GELU_TANH = 1
} llmint8_activation;

/*
 * llmint8_matmul_mixed with the two steps that follow the linear in a
 * transformer block fused into its epilogue. The output is
 *   Y[i,j] = fp16( act( y[i,j] + bias[j] ) )
 * where y[i,j] is the fp32 value llmint8_matmul_mixed rounds, bias is added
 * in fp32 (nn.Linear's bias, which the Linear8bitLt replacing each nn.Linear
 * keeps: page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
 * accelerate", section "accelerate 就是你需要的一切"), and
 * act is evaluated in fp32 (tanhf). Rounding to fp16 happens once, at the end.
 *   bias_f16   (device, may be NULL) fp16 [N]
 *   activation LLMINT8_ACT_NONE or LLMINT8_ACT_GELU_TANH; anything else
 *              returns LLMINT8_ERR_INVALID_ARG.
 * Every other argument, and the behaviour on errors, as for
 * llmint8_matmul_mixed (which is this call with bias NULL and no activation).
 */
LLMINT8_API llmint8_status llmint8_matmul_mixed_ex(const void *X_f16, int64_t M, int64_t K, const int8_t *CB,
                                       const float *SCB, const void *W_f16, int64_t N,
                                       float threshold, const void *bias_f16, int activation,
                                       void *Y_f16, void *workspace, size_t ws_bytes,
                                       const llmint8_debug *dbg, llmint8_stream_t stream);

/* Bytes of workspace needed by llmint8_matmul_mixed_fp16w: that of
 * llmint8_matmul_mixed plus room for W's codes [N x K] and row absmax [N]. */
LLMINT8_API size_t llmint8_workspace_size_fp16w(int64_t M, int64_t N, int64_t K);

/*
 * The linear in the "has fp16 weights" mode of Linear8bitLt (page "Hugging
 * Face 将 LLM.int8() 8-bit 量化集成进 transformers 与 accelerate", section
 * "用法": the default, meant for mixed int8/fp16 training): W stays in fp16
 * and is quantized per output row on every call (llmint8_quantize_rowwise
 * with t <= 0, into the workspace), then the call proceeds as
 * llmint8_matmul_mixed_ex with W_f16 supplying the outlier columns. The
 * result is identical to quantizing W once and calling llmint8_matmul_mixed_ex.
 *   W_f16      (device) fp16 [N x K], required
 *   workspace  >= llmint8_workspace_size_fp16w(M, N, K) bytes, zeroed once
 *   dbg        as for llmint8_matmul_mixed
 * Other arguments and errors as for llmint8_matmul_mixed_ex.
 */
LLMINT8_API llmint8_status llmint8_matmul_mixed_fp16w(const void *X_f16, int64_t M, int64_t K, const void *W_f16,
                                          int64_t N, float threshold, const void *bias_f16, int activation,
                                          void *Y_f16, void *workspace, size_t ws_bytes,
                                          const llmint8_debug *dbg, llmint8_stream_t stream);

/*
 * Zero-point (unsigned int8) variant of the activation quantization: the
 * alternative to absmax in section "模型量化简介" of the page "Hugging Face 将
 * LLM.int8() 8-bit 量化集成进 transformers 与 accelerate" (subtract the minimum,
 * scale by the range, 0 exactly representable). Per row of X, over the
 * non-outlier columns: range [lo, hi] = [min(0, min x), max(0, max x)],
 * s = 255 / (hi - lo) in fp32 (0 for an all-zero row), zero point
 * z = rint(-lo * s), code q = clamp(rint(x * s) + z, 0, 255) stored as the
 * int8 value q - 128 (rint: round half to even); outlier columns get q = z.
 * The weight keeps its absmax codes (CB, SCB). With c = q - 128,
 *   sum_k (q - z_i) CB[j,k] = acc[i,j] + (128 - z_i) * R[j],  R[j] = sum_k CB[j,k],
 * so the int8 product is the same tensor-core GEMM and the epilogue adds
 * (128 - z_i) R[j] before dequantizing by SB[j] / (127 s_i). K is limited to
 * LLMINT8_MAX_K_ASYM so that these int8 sums fit in int32 (|c| <= 128).
 */
#define LLMINT8_MAX_K_ASYM 132104

/* Zero-point codes of X [rows x cols] (fp16, device): codes int8 [rows x cols]
 * out, scale fp32 [rows] out (s), zero int32 [rows] out (z). threshold and
 * outlier_bitmap as in llmint8_quantize_rowwise (the bitmap is written; the
 * outlier columns are found first, then the rows are coded against them).
 * workspace: at least llmint8_quantize_workspace_size(rows, cols) bytes,
 * zeroed once. Device pointers 16-byte aligned. Errors as
 * llmint8_quantize_rowwise, with cols > LLMINT8_MAX_K_ASYM unsupported. */
LLMINT8_API llmint8_status llmint8_quantize_rowwise_asym(const void *X_f16, int64_t rows, int64_t cols,
                                             float threshold, int8_t *codes, float *scale, int32_t *zero,
                                             uint32_t *outlier_bitmap, void *workspace, size_t ws_bytes,
                                             llmint8_stream_t stream);

/* R[j] = sum over K of CB[j, :] (int8 [N x K], device, 16-byte aligned) into
 * row_sums int32 [N] (device, 4-byte aligned): the weight-side term of the
 * zero-point product, computed once per weight like SCB. */
LLMINT8_API llmint8_status llmint8_code_row_sums(const int8_t *CB, int64_t N, int64_t K, int32_t *row_sums,
                                     llmint8_stream_t stream);

/* Bytes of workspace needed by llmint8_matmul_mixed_asym. */
LLMINT8_API size_t llmint8_workspace_size_asym(int64_t M, int64_t N, int64_t K);

/* The LLM.int8() linear with zero-point codes for X: as llmint8_matmul_mixed,
 * plus CB_row_sums (int32 [N], from llmint8_code_row_sums). Always runs the
 * GEMM path (no fused decode kernel). dbg->row_absmax receives the scales s,
 * dbg->codes the int8 codes q - 128, dbg->acc the int32 product of the stored
 * codes. workspace >= llmint8_workspace_size_asym(M, N, K) bytes, zeroed once. */
LLMINT8_API llmint8_status llmint8_matmul_mixed_asym(const void *X_f16, int64_t M, int64_t K, const int8_t *CB,
                                         const float *SCB, const int32_t *CB_row_sums, const void *W_f16,
                                         int64_t N, float threshold, void *Y_f16, void *workspace,
                                         size_t ws_bytes, const llmint8_debug *dbg, llmint8_stream_t stream);

/*
 * Plain int8 GEMM with int32 output: acc[i,j] = sum_k A[i,k] * B[j,k]
 * (the int8 product of vector-wise quantization, [Q]).
 *   A (device) int8 [M x K], B (device) int8 [N x K], acc (device) int32 [M x N].
 *   workspace: >= llmint8_workspace_size(M, N, K) bytes, zeroed once (its
 *   status word, and for M >= 256 its stream-K slots and flags).
 */
LLMINT8_API llmint8_status llmint8_gemm_s8s8s32(const int8_t *A, int64_t M, const int8_t *B, int64_t N,
                                    int64_t K, int32_t *acc, void *workspace, size_t ws_bytes,
                                    llmint8_stream_t stream);

/*
 * Tensor parallelism: the pieces a linear split over several GPUs needs (page
 * "优化故事：Bloom 推理", section "支持 TP": every GPU owns a part of the
 * weights; the parts are combined with NCCL all-reduces, section "唾手可得的
 * 优化"). The collectives themselves are the caller's (NCCL); these calls
 * are the per-GPU steps around them. Each split reproduces the one-GPU
 * result of [S]/[M]: the same outlier set, row absmax and codes.
 *   - Column split (rows of W across GPUs): llmint8_matmul_mixed on the full X
 *     and this GPU's rows of CB/SCB/W; outputs are column blocks, put back in
 *     place by llmint8_gather_column_blocks after an all-gather.
 *   - Row split (K across GPUs; CB/SCB quantized over the FULL rows of W):
 *     llmint8_quantize_rowwise on this GPU's columns of X gives its outlier
 *     bitmap and the row absmax over its other columns; a max all-reduce of
 *     that absmax gives the full one; llmint8_quantize_rowwise_given codes the
 *     columns with it; llmint8_find_outlier_cols lists the outlier columns;
 *     llmint8_matmul_codes writes an fp32 partial product; a sum all-reduce
 *     adds the partials and llmint8_bias_act_to_f16 applies bias, activation
 *     and the single fp16 rounding.
 *   - Token split (rows of X across GPUs, W replicated): every GPU's outlier
 *     bitmap is all-gathered; llmint8_quantize_rowwise_given codes this GPU's
 *     rows against their union; llmint8_matmul_codes gives its rows of Y.
 */

/* Output types of llmint8_matmul_codes. */
#define LLMINT8_OUT_F16 0
#define LLMINT8_OUT_F32 1

/*
 * Row-wise absmax quantization against a GIVEN outlier set ([Q], [M]).
 *   X_f16          (device) fp16 [rows x cols], cols a multiple of 16.
 *   outlier_bitmaps (device) uint32 [n_bitmaps x ceil(cols/32)]: the outlier
 *                  set is the OR of the n_bitmaps bitmaps (n_bitmaps = 0: no
 *                  outlier columns; the pointer may then be NULL).
 *   row_absmax_in  (device, may be NULL) fp32 [rows]: if given, row i is
 *                  coded with this absmax (e.g. the max all-reduced over the
 *                  GPUs of a row split) and row_absmax_out is not written;
 *                  if NULL, the absmax over the columns outside the set is
 *                  computed and written to row_absmax_out (then required).
 *   codes          (device) int8 [rows x cols] out: round-half-even(x * s),
 *                  s = 127 / absmax in fp32 (0 for absmax 0); 0 in set columns.
 *   bitmap_out     (device, may be NULL) uint32 [ceil(cols/32)] out: the union.
 * No workspace. Errors: as llmint8_quantize_rowwise; n_bitmaps > 4096 or
 * neither row_absmax pointer given (rows > 0) is LLMINT8_ERR_INVALID_ARG.
 * With rows == 0 only bitmap_out is written (X, codes and the absmax pointers
 * may be NULL).
 */
LLMINT8_API llmint8_status llmint8_quantize_rowwise_given(const void *X_f16, int64_t rows, int64_t cols,
                                              const uint32_t *outlier_bitmaps, int n_bitmaps,
                                              const float *row_absmax_in, int8_t *codes, float *row_absmax_out,
                                              uint32_t *bitmap_out, llmint8_stream_t stream);

/*
 * The int8 GEMM with the LLM.int8() epilogue ([Q], [S], [M], [U]) on codes
 * quantized beforehand:
 *   Y[i,j] = act( acc[i,j] * SX[i] * SCB[j] / 127^2
 *                 + sum_{c in O} X[i,c] * Wt[j,c] + bias[j] ),  acc = CX . CB^T (int32),
 * with O the first *d_count entries of col_idx and Wt as in
 * llmint8_matmul_mixed.
 *   CX (device) int8 [M x K], SX (device) fp32 [M]: X's codes and row absmax
 *   X_f16 (device) fp16 [M x K]: read only at the outlier columns
 *   CB, SCB, W_f16 (may be NULL): as llmint8_matmul_mixed
 *   col_idx (device) int32 [>= *d_count], d_count (device) int32 [1]: the
 *       outlier columns (llmint8_find_outlier_cols), read on the device
 *   bias_f16 (device, may be NULL), activation: as llmint8_matmul_mixed_ex
 *   out_dtype LLMINT8_OUT_F16: Y fp16 [M x N]; LLMINT8_OUT_F32: Y fp32 [M x N]
 *       (an unrounded partial sum, e.g. of a row split)
 *   workspace (device) >= 256 bytes, zeroed once (only its status word is used)
 * Errors as llmint8_matmul_mixed_ex; a bad out_dtype is LLMINT8_ERR_INVALID_ARG.
 */
LLMINT8_API llmint8_status llmint8_matmul_codes(const int8_t *CX, const float *SX, const void *X_f16, int64_t M,
                                    int64_t K, const int8_t *CB, const float *SCB, const void *W_f16, int64_t N,
                                    const int32_t *col_idx, const int32_t *d_count, const void *bias_f16,
                                    int activation, int out_dtype, void *Y, void *workspace, size_t ws_bytes,
                                    llmint8_stream_t stream);

/* Y_f16[i,j] = fp16( act( Y32[i,j] + bias[j] ) ) in fp32 (the last step of a
 * row split, after the partial outputs are summed). Y32 (device) fp32
 * [M x N], N a multiple of 4; bias_f16 (device, may be NULL) fp16 [N];
 * activation as llmint8_matmul_mixed_ex; Y_f16 (device) fp16 [M x N]. */
LLMINT8_API llmint8_status llmint8_bias_act_to_f16(const float *Y32, int64_t M, int64_t N, const void *bias_f16,
                                       int activation, void *Y_f16, llmint8_stream_t stream);

/* dst[i, p*Nr + j] = src[p][i][j]: the column blocks [P][M x Nr] of a column
 * split (as an all-gather leaves them) into one fp16 [M x P*Nr] matrix.
 * src, dst (device) fp16, 16-byte aligned, Nr a multiple of 8. */
LLMINT8_API llmint8_status llmint8_gather_column_blocks(const void *src_f16, int64_t P, int64_t M, int64_t Nr,
                                            void *dst_f16, llmint8_stream_t stream);

/*
 * Allocation-free row-wise quantizer. The source page has no counterpart: it
 * exists for callers that cannot allocate device memory, such as a server
 * that reserved all device memory for its own pool at start-up, a plugin in a
 * host process that forbids device allocations after initialisation, or a
 * latency-critical loop that cannot afford an allocation's implicit
 * synchronisation.
 *
 * Same arguments and results as llmint8_quantize_rowwise, without the
 * workspace: the scratch sits in a fixed array inside the library (about
 * 256 KB, held by every GPU that uses this call until the process exits).
 *   - rows <= LLMINT8_NOALLOC_MAX_ROWS and cols <= LLMINT8_NOALLOC_MAX_COLS;
 *     larger sizes return LLMINT8_ERR_UNSUPPORTED_SHAPE before any work.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress); make that first call before any stream
 *     capture on the device.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents. Calls ordered on one stream are safe; calls whose work
 *     overlaps on the GPU (unordered streams) race and give wrong results.
 *   - The address lookup is cached for the life of the process: after a
 *     cudaDeviceReset of that device this entry point must not be called.
 *   - A kernel that gives up on a bounded wait sets a bit in the array's own
 *     status word (the outputs are then incomplete). The word keeps its bits
 *     across calls until llmint8_noalloc_read_status reads and clears it.
 */
#define LLMINT8_NOALLOC_MAX_ROWS 65536
#define LLMINT8_NOALLOC_MAX_COLS 65536
LLMINT8_API llmint8_status llmint8_quantize_rowwise_noalloc(const void *X_f16, int64_t rows, int64_t cols,
                                                float threshold, int8_t *codes, float *row_absmax,
                                                uint32_t *outlier_bitmap, llmint8_stream_t stream);

/* Status word of llmint8_quantize_rowwise_noalloc's fixed array on the current
 * device: waits for the device (cudaDeviceSynchronize), copies the word to
 * *out (LLMINT8_DEV_* bits, 0 if no call since the last clear gave up on a
 * wait) and, if clear != 0, resets it. Returns LLMINT8_OK when the word is 0,
 * LLMINT8_ERR_DEVICE when it is not, LLMINT8_ERR_CUDA if a CUDA call failed,
 * LLMINT8_ERR_INVALID_ARG for a NULL out. Allocates nothing. */
LLMINT8_API llmint8_status llmint8_noalloc_read_status(int clear, uint32_t *out);

#ifdef __cplusplus
}
#endif

#endif /* LLMINT8_H */
