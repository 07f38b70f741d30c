/*
 * CPU oracle for the LLM.int8() mixed-precision linear Y = X . W^T.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it. It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Plain, slow, single-threaded C. Every function follows one passage of the
 * source page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
 * accelerate" (a translation of the Hugging Face blog post "A Gentle
 * Introduction to 8-bit Matrix Multiplication for transformers at scale"):
 *
 *   - absmax quantization: section "模型量化简介" (Introduction to model
 *     quantization), the absmax worked example: scale = 127 / absmax, multiply,
 *     round; int8 range [-127, 127].
 *   - vector-wise quantization and outer-product dequantization: same
 *     section, the paragraph on row-/vector-wise quantization of A*B=C.
 *   - the three-step decomposition (outlier columns in fp16, the rest in
 *     int8, dequantize and add): section "LLM.int8() 的简要总结" (A gentle
 *     summary of LLM.int8()).
 *   - threshold "magnitude 6 or greater", hidden states row-wise, weights per
 *     output row: section "MatMul 内部" (Inside the MatMul).
 *   - weight dequantization CB * SCB / 127 (with the scale taken per output
 *     row, SCB[:, None]): section "用法" (Usage).
 *
 * Inputs arrive as fp32 arrays; fp16 data is widened exactly by the caller.
 * All float arithmetic here is IEEE fp32 with round-to-nearest-even (x86-64
 * SSE, compiled with -ffp-contract=off -fno-fast-math), and the final output
 * is accumulated in fp64.
 *
 * Parity status: every function is pinned by the CPU tests (worked examples,
 * printed weights, library matmuls, closed forms, error bound); the fp16
 * output beyond its stated tolerance has no printed value to pin against.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

/* Step 1 of the decomposition: the outlier columns. Column c is an outlier
 * when any row holds |x| >= t (the page keeps "all outliers of magnitude 6
 * or greater"). t <= 0 switches the decomposition off (no outliers).
 * Writes is_outlier[c] in {0,1} and returns the number of outlier columns. */
int64_t oracle_outlier_cols(const float *X, int64_t rows, int64_t cols, float t,
                            uint8_t *is_outlier)
{
    for (int64_t c = 0; c < cols; ++c)
        is_outlier[c] = 0;
    if (t > 0.0f) {
        for (int64_t i = 0; i < rows; ++i)
            for (int64_t c = 0; c < cols; ++c)
                if (fabsf(X[i * cols + c]) >= t)
                    is_outlier[c] = 1;
    }
    int64_t count = 0;
    for (int64_t c = 0; c < cols; ++c)
        count += is_outlier[c];
    return count;
}

/* Row-wise absmax quantization of the non-outlier part.
 * absmax[i] = max over non-outlier columns c of |x[i,c]| (0 for an empty or
 * all-zero row); s = 127 / absmax in fp32; code = round-half-even(x * s) in
 * fp32; outlier columns get code 0. is_outlier may be NULL (no outliers).
 * Returns the number of codes that fell outside [-127, 127] (always 0 when
 * the arithmetic is right). */
int64_t oracle_quantize_rows(const float *X, int64_t rows, int64_t cols,
                             const uint8_t *is_outlier, int8_t *codes, float *absmax)
{
    int64_t bad = 0;
    for (int64_t i = 0; i < rows; ++i) {
        const float *x = X + i * cols;
        float amax = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            if (is_outlier && is_outlier[c])
                continue;
            float a = fabsf(x[c]);
            if (a > amax)
                amax = a;
        }
        absmax[i] = amax;
        float s = 0.0f;
        if (amax > 0.0f)
            s = 127.0f / amax;
        for (int64_t c = 0; c < cols; ++c) {
            int32_t q = 0;
            if (amax > 0.0f && !(is_outlier && is_outlier[c])) {
                float v = x[c] * s;
                q = (int32_t)rintf(v);
            }
            if (q > 127 || q < -127) {
                ++bad;
                q = q > 0 ? 127 : -127;
            }
            codes[i * cols + c] = (int8_t)q;
        }
    }
    return bad;
}

/* The int8 product of the non-outlier part: acc[i,j] = sum_c A[i,c]*B[j,c]
 * with A = [M x K] and B = [N x K] (both row-major, K contiguous), summed
 * exactly in int64. Returns the number of sums that do not fit in int32
 * (those are clamped in the output). */
int64_t oracle_int8_matmul(const int8_t *A, int64_t M, const int8_t *B, int64_t N, int64_t K,
                           int32_t *acc)
{
    int64_t overflow = 0;
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < N; ++j) {
            int64_t s = 0;
            for (int64_t c = 0; c < K; ++c)
                s += (int64_t)A[i * K + c] * (int64_t)B[j * K + c];
            if (s > INT32_MAX || s < INT32_MIN) {
                ++overflow;
                s = s > 0 ? INT32_MAX : INT32_MIN;
            }
            acc[i * N + j] = (int32_t)s;
        }
    }
    return overflow;
}

/* The fp16 side of the decomposition needs W's outlier columns. Either they
 * come from the fp16 weight itself (W non-NULL), or they are recovered from
 * the int8 weight as CB * SCB / 127 with SCB taken per output row j
 * (section "用法"). Wt is [N x n_out]: Wt[j,k] for column cols[k]. */
void oracle_outlier_weight(const float *W, const int8_t *CB, const float *SB, int64_t N, int64_t K,
                           const int64_t *cols, int64_t n_out, float *Wt)
{
    for (int64_t j = 0; j < N; ++j) {
        for (int64_t k = 0; k < n_out; ++k) {
            int64_t c = cols[k];
            float v;
            if (W) {
                v = W[j * K + c];
            } else {
                float prod = (float)CB[j * K + c] * SB[j];
                v = prod / 127.0f;
            }
            Wt[j * n_out + k] = v;
        }
    }
}

/* Steps 2-3 of the decomposition, evaluated in fp64:
 *   Y[i,j] = acc[i,j] * SX[i] * SB[j] / 127^2          (outer-product dequant)
 *          + sum_k X[i, cols[k]] * Wt[j,k]              (the fp16 outlier product)
 * X is [M x K]; Wt is [N x n_out]; Y is [M x N] fp64. */
void oracle_mixed_output(const int32_t *acc, const float *SX, const float *SB, int64_t M, int64_t N,
                         const float *X, int64_t K, const int64_t *cols, int64_t n_out,
                         const float *Wt, double *Y)
{
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < N; ++j) {
            double y = (double)acc[i * N + j] * (double)SX[i] * (double)SB[j] / (127.0 * 127.0);
            double o = 0.0;
            for (int64_t k = 0; k < n_out; ++k)
                o += (double)X[i * K + cols[k]] * (double)Wt[j * n_out + k];
            Y[i * N + j] = y + o;
        }
    }
}

/* The steps after the linear in a transformer block, on the fp64 output:
 * Y[i,j] += bias[j] (nn.Linear's bias, kept by the Linear8bitLt that replaces
 * it: page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
 * accelerate", section "accelerate 就是你需要的一切"), then, for act == 1,
 * BLOOM's GELU in its tanh form (page "优化故事：Bloom 推理", section
 * "唾手可得的优化"): g(y) = y/2 * (1 + tanh(0.79788456 * y * (1 + 0.044715 y^2))).
 * bias may be NULL. */
void oracle_bias_act(double *Y, int64_t M, int64_t N, const float *bias, int act)
{
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < N; ++j) {
            double y = Y[i * N + j];
            if (bias)
                y += (double)bias[j];
            if (act == 1) {
                const double inner = 0.79788456 * y * (1.0 + 0.044715 * y * y);
                y = 0.5 * y * (1.0 + tanh(inner));
            }
            Y[i * N + j] = y;
        }
    }
}

/* The unsigned-int8 / zero-point alternative to absmax quantization (section
 * "模型量化简介": subtract the minimum and scale by the range, close to
 * zero-point quantization, which keeps 0 exactly representable), applied row
 * by row to the non-outlier part. Reading taken: the range of row i is
 * [lo, hi] = [min(0, min x), max(0, max x)] over its non-outlier columns, so
 * that 0 is inside it; s = 255 / (hi - lo) in fp32 (0 for an all-zero or
 * empty row); zero point z = rint(-lo * s) in [0, 255]; code
 * q = clamp(rint(x * s) + z, 0, 255), stored as the int8 value q - 128.
 * Outlier columns get q = z (they then contribute nothing after z is taken
 * off). Dequantization: x ~ (q - z) / s. Returns the number of codes clamped
 * (rint(x * s) and rint(-lo * s) round separately, so the row's extreme
 * values can land one step past [0, 255]; the clamp keeps them in range). */
int64_t oracle_quantize_rows_asym(const float *X, int64_t rows, int64_t cols, const uint8_t *is_outlier,
                                  int8_t *codes, float *scale, int32_t *zero)
{
    int64_t clamped = 0;
    for (int64_t i = 0; i < rows; ++i) {
        const float *x = X + i * cols;
        float lo = 0.0f, hi = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            if (is_outlier && is_outlier[c])
                continue;
            if (x[c] < lo)
                lo = x[c];
            if (x[c] > hi)
                hi = x[c];
        }
        const float range = hi - lo;
        const float s = range > 0.0f ? 255.0f / range : 0.0f;
        const int32_t z = (int32_t)rintf(-lo * s);
        scale[i] = s;
        zero[i] = z;
        for (int64_t c = 0; c < cols; ++c) {
            int32_t q = z;
            if (!(is_outlier && is_outlier[c])) {
                const float v = x[c] * s;
                q = (int32_t)rintf(v) + z;
            }
            if (q < 0 || q > 255) {
                ++clamped;
                q = q < 0 ? 0 : 255;
            }
            codes[i * cols + c] = (int8_t)(q - 128);
        }
    }
    return clamped;
}

/* Row sums of the int8 weight codes, R[j] = sum_c CB[j,c] (exact). */
void oracle_code_row_sums(const int8_t *CB, int64_t N, int64_t K, int64_t *R)
{
    for (int64_t j = 0; j < N; ++j) {
        int64_t s = 0;
        for (int64_t c = 0; c < K; ++c)
            s += CB[j * K + c];
        R[j] = s;
    }
}

/* Steps 2-3 with zero-point codes for X, in fp64: with c = q - 128,
 *   sum_k (q - z_i) CB[j,k] = acc[i,j] + (128 - z_i) * R[j],
 * dequantized by 1 / s_i on the X side and SB[j] / 127 on the weight side:
 *   Y[i,j] = (acc[i,j] + (128 - z_i) R[j]) * SB[j] / (127 s_i)   (0 if s_i = 0)
 *          + sum_k X[i, cols[k]] * Wt[j,k]. */
void oracle_mixed_output_asym(const int32_t *acc, const float *SXs, const int32_t *ZX, const int64_t *R,
                              const float *SB, int64_t M, int64_t N, const float *X, int64_t K,
                              const int64_t *cols, int64_t n_out, const float *Wt, double *Y)
{
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < N; ++j) {
            double y = 0.0;
            if (SXs[i] > 0.0f) {
                const double t = (double)acc[i * N + j] + (double)(128 - ZX[i]) * (double)R[j];
                y = t * (double)SB[j] / (127.0 * (double)SXs[i]);
            }
            double o = 0.0;
            for (int64_t k = 0; k < n_out; ++k)
                o += (double)X[i * K + cols[k]] * (double)Wt[j * n_out + k];
            Y[i * N + j] = y + o;
        }
    }
}
