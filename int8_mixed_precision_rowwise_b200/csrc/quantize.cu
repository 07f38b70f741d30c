// Row-wise absmax quantization with outlier-column decomposition.
//
// Method (page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
// accelerate"): absmax quantization with scale 127 / absmax and rounding
// (section "模型量化简介", Introduction to model quantization); hidden-state
// columns holding any |x| >= threshold go to the fp16 side and the rest is
// quantized per row (sections "LLM.int8() 的简要总结" and "MatMul 内部").
//
// The outlier set O is a property of the whole matrix, yet each row's scale
// must exclude O. K1 reads X exactly once: each CTA keeps a shared-memory copy
// of the columns already known to be outliers (its own discoveries plus the
// global bitmap, refreshed at every row) and takes the row maximum over the
// other columns with |x| < t, recording the column where it sits. That masked
// maximum is never below the true one (known columns are a subset of O, and
// every column outside O has |x| < t), and equals it whenever the recorded
// column is outside the final O. K2 re-quantizes exactly the rows whose
// recorded column ended up in O, zeroes the codes of every column of O, and
// compacts the bitmap into ascending column indices.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"

namespace llmint8 {

namespace {

__device__ __forceinline__ void unpack8(const uint4 &v, float (&x)[8])
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// Quantize one value with the row multiplier s = 127 / absmax (fp32, RN).
__device__ __forceinline__ int quant1(float x, float s)
{
    return __float2int_rn(__fmul_rn(x, s));
}

__device__ __forceinline__ uint2 pack8(const int (&q)[8])
{
    uint2 r;
    r.x = (uint32_t)(q[0] & 0xFF) | ((uint32_t)(q[1] & 0xFF) << 8) | ((uint32_t)(q[2] & 0xFF) << 16) |
          ((uint32_t)(q[3] & 0xFF) << 24);
    r.y = (uint32_t)(q[4] & 0xFF) | ((uint32_t)(q[5] & 0xFF) << 8) | ((uint32_t)(q[6] & 0xFF) << 16) |
          ((uint32_t)(q[7] & 0xFF) << 24);
    return r;
}

template <int NT>
__device__ __forceinline__ unsigned long long block_max_u64(unsigned long long v, unsigned long long *s_red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        s_red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < NT / 32 ? s_red[lane] : 0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
            v = w > v ? w : v;
        }
        if (lane == 0)
            s_red[0] = v;
    }
    __syncthreads();
    v = s_red[0];
    __syncthreads();
    return v;
}

template <int NT>
__device__ __forceinline__ float block_max_f32(float v, float *s_red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        s_red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < NT / 32 ? s_red[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0)
            s_red[0] = v;
    }
    __syncthreads();
    v = s_red[0];
    __syncthreads();
    return v;
}

// Key ordering (value desc, column asc) so a max-reduction returns the
// largest |x| and, among equal values, the smallest column.
__device__ __forceinline__ unsigned long long amax_key(float a, int c)
{
    return ((unsigned long long)__float_as_uint(a) << 32) | (uint32_t)(~(uint32_t)c);
}

// Merge the global outlier bitmap into the CTA's known set.
template <int NT>
__device__ __forceinline__ void refresh_known(uint32_t *s_known, const uint32_t *bitmap, int nwords)
{
    for (int w = threadIdx.x; w < nwords; w += NT) {
        uint32_t g = *reinterpret_cast<const volatile uint32_t *>(bitmap + w);
        if (g & ~s_known[w])
            atomicOr(&s_known[w], g);
    }
}

// Record newly seen outlier columns (bits of word w) in the CTA set and, if
// they were new to this CTA, in the global bitmap.
__device__ __forceinline__ void publish_outliers(uint32_t *s_known, uint32_t *bitmap, int w, uint32_t bits)
{
    uint32_t old = atomicOr(&s_known[w], bits);
    uint32_t fresh = bits & ~old;
    if (fresh)
        atomicOr(&bitmap[w], fresh);
}

// K1, register-resident rows: NT threads per row, V 16-byte vectors each
// (NT * V * 8 >= cols). One CTA walks rows blockIdx.x, +gridDim.x, ...
template <int NT, int V>
__global__ void __launch_bounds__(NT) k_quantize_rows(const uint4 *__restrict__ X, int64_t rows, int cols,
                                                      float t, int8_t *__restrict__ codes,
                                                      float *__restrict__ absmax,
                                                      int32_t *__restrict__ argmax,
                                                      uint32_t *__restrict__ bitmap)
{
    extern __shared__ uint32_t s_known[];
    __shared__ unsigned long long s_red[NT / 32];
    const int tid = threadIdx.x;
    const int nvec = cols >> 3;
    const int nwords = (cols + 31) >> 5;
    const bool thr = t > 0.f;

    if (thr) {
        for (int w = tid; w < nwords; w += NT)
            s_known[w] = 0u;
    }

    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint4 *xr = X + r * (int64_t)nvec;
        uint4 v[V];
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int vi = u * NT + tid;
            v[u] = vi < nvec ? __ldg(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
        }
        uint32_t kbits[V];
#pragma unroll
        for (int u = 0; u < V; ++u)
            kbits[u] = 0u;
        if (thr) {
            __syncthreads(); // s_known initialised / previous row's readers done
            refresh_known<NT>(s_known, bitmap, nwords);
            __syncthreads();
#pragma unroll
            for (int u = 0; u < V; ++u) {
                const int vi = u * NT + tid;
                if (vi < nvec)
                    kbits[u] = (s_known[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
            }
        }

        unsigned long long key = 0ull;
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int vi = u * NT + tid;
            if (vi >= nvec)
                continue;
            float x[8];
            unpack8(v[u], x);
            uint32_t hit = 0u;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = fabsf(x[e]);
                if (thr && a >= t) {
                    hit |= 1u << e;
                } else if (!((kbits[u] >> e) & 1u)) {
                    const unsigned long long k = amax_key(a, vi * 8 + e);
                    key = k > key ? k : key;
                }
            }
            if (hit & ~kbits[u])
                publish_outliers(s_known, bitmap, vi >> 2, (hit & ~kbits[u]) << ((vi & 3) * 8));
            kbits[u] |= hit;
        }

        key = block_max_u64<NT>(key, s_red);
        const float amax = __uint_as_float((uint32_t)(key >> 32));
        const int acol = (int)(~(uint32_t)key);
        const float s = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;

        int8_t *cr = codes + r * (int64_t)cols;
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int vi = u * NT + tid;
            if (vi >= nvec)
                continue;
            float x[8];
            unpack8(v[u], x);
            int q[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                q[e] = ((kbits[u] >> e) & 1u) ? 0 : quant1(x[e], s);
            *reinterpret_cast<uint2 *>(cr + (int64_t)vi * 8) = pack8(q);
        }
        if (tid == 0) {
            absmax[r] = amax;
            argmax[r] = amax > 0.f ? acol : -1;
        }
    }
}

// K1 for rows too long to hold in registers (cols > 65536): the same
// arithmetic, with the row read twice (the second read is served by L2).
template <int NT>
__global__ void __launch_bounds__(NT) k_quantize_rows_loop(const uint4 *__restrict__ X, int64_t rows,
                                                           int cols, float t, int8_t *__restrict__ codes,
                                                           float *__restrict__ absmax,
                                                           int32_t *__restrict__ argmax,
                                                           uint32_t *__restrict__ bitmap)
{
    extern __shared__ uint32_t s_known[];
    __shared__ unsigned long long s_red[NT / 32];
    const int tid = threadIdx.x;
    const int nvec = cols >> 3;
    const int nwords = (cols + 31) >> 5;
    const bool thr = t > 0.f;
    if (thr) {
        for (int w = tid; w < nwords; w += NT)
            s_known[w] = 0u;
    }
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint4 *xr = X + r * (int64_t)nvec;
        if (thr) {
            __syncthreads();
            refresh_known<NT>(s_known, bitmap, nwords);
            __syncthreads();
        }
        unsigned long long key = 0ull;
        for (int vi = tid; vi < nvec; vi += NT) {
            float x[8];
            unpack8(__ldg(xr + vi), x);
            uint32_t kb = thr ? (s_known[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu : 0u;
            uint32_t hit = 0u;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = fabsf(x[e]);
                if (thr && a >= t) {
                    hit |= 1u << e;
                } else if (!((kb >> e) & 1u)) {
                    const unsigned long long k = amax_key(a, vi * 8 + e);
                    key = k > key ? k : key;
                }
            }
            if (hit & ~kb)
                publish_outliers(s_known, bitmap, vi >> 2, (hit & ~kb) << ((vi & 3) * 8));
        }
        key = block_max_u64<NT>(key, s_red);
        const float amax = __uint_as_float((uint32_t)(key >> 32));
        const int acol = (int)(~(uint32_t)key);
        const float s = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        int8_t *cr = codes + r * (int64_t)cols;
        for (int vi = tid; vi < nvec; vi += NT) {
            float x[8];
            unpack8(__ldg(xr + vi), x);
            // Within one row the known set only gains columns whose element in
            // this row is itself >= t, so this mask agrees with the first pass.
            uint32_t kb = thr ? (s_known[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu : 0u;
            int q[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                q[e] = (((kb >> e) & 1u) || (thr && fabsf(x[e]) >= t)) ? 0 : quant1(x[e], s);
            *reinterpret_cast<uint2 *>(cr + (int64_t)vi * 8) = pack8(q);
        }
        if (tid == 0) {
            absmax[r] = amax;
            argmax[r] = amax > 0.f ? acol : -1;
        }
    }
}

// Ascending list of the set bits of s_bm[0..nwords) written by one CTA.
template <int NT>
__device__ void compact_block(const uint32_t *s_bm, int nwords, int32_t *col_idx, int32_t *count)
{
    __shared__ int s_warp[NT / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (nwords + NT - 1) / NT;
    const int w0 = min(tid * per, nwords), w1 = min(w0 + per, nwords);
    int cnt = 0;
    for (int w = w0; w < w1; ++w)
        cnt += __popc(s_bm[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int wv = lane < NT / 32 ? s_warp[lane] : 0;
        int wi = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o)
                wi += y;
        }
        if (lane < NT / 32)
            s_warp[lane] = wi - wv; // exclusive prefix of warp totals
        if (lane == NT / 32 - 1)
            *count = wi;
    }
    __syncthreads();
    int pos = s_warp[warp] + incl - cnt;
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = s_bm[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            col_idx[pos++] = w * 32 + b;
            bits &= bits - 1u;
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(NT) k_compact(const uint32_t *__restrict__ bitmap, int cols,
                                                int32_t *__restrict__ col_idx, int32_t *__restrict__ count)
{
    extern __shared__ uint32_t s_bm[];
    const int nwords = (cols + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += NT)
        s_bm[w] = bitmap[w];
    __syncthreads();
    compact_block<NT>(s_bm, nwords, col_idx, count);
}

// K2: with the final outlier set known, (a) CTA 0 compacts it, (b) rows whose
// masked maximum sat in an outlier column are re-quantized over the
// non-outlier columns, and (c) every other row gets its outlier-column codes
// zeroed.
template <int NT>
__global__ void __launch_bounds__(NT) k_fixup_rows(const uint4 *__restrict__ X, int64_t rows, int cols,
                                                   int8_t *__restrict__ codes, float *__restrict__ absmax,
                                                   const int32_t *__restrict__ argmax,
                                                   const uint32_t *__restrict__ bitmap,
                                                   int32_t *__restrict__ col_idx, int32_t *__restrict__ count)
{
    extern __shared__ uint32_t s_bm[];
    __shared__ float s_red[NT / 32];
    const int tid = threadIdx.x;
    const int nwords = (cols + 31) >> 5;
    const int nvec = cols >> 3;
    for (int w = tid; w < nwords; w += NT)
        s_bm[w] = bitmap[w];
    __syncthreads();
    if (blockIdx.x == 0)
        compact_block<NT>(s_bm, nwords, col_idx, count);

    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int am = argmax[r];
        int8_t *cr = codes + r * (int64_t)cols;
        if (am >= 0 && ((s_bm[am >> 5] >> (am & 31)) & 1u)) {
            const uint4 *xr = X + r * (int64_t)nvec;
            float m = 0.f;
            for (int vi = tid; vi < nvec; vi += NT) {
                float x[8];
                unpack8(__ldg(xr + vi), x);
                const uint32_t kb = (s_bm[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (!((kb >> e) & 1u))
                        m = fmaxf(m, fabsf(x[e]));
            }
            const float amax = block_max_f32<NT>(m, s_red);
            const float s = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
            for (int vi = tid; vi < nvec; vi += NT) {
                float x[8];
                unpack8(__ldg(xr + vi), x);
                const uint32_t kb = (s_bm[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
                int q[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    q[e] = ((kb >> e) & 1u) ? 0 : quant1(x[e], s);
                *reinterpret_cast<uint2 *>(cr + (int64_t)vi * 8) = pack8(q);
            }
            if (tid == 0)
                absmax[r] = amax;
        } else {
            for (int w = tid; w < nwords; w += NT) {
                uint32_t bits = s_bm[w];
                while (bits) {
                    const int b = __ffs(bits) - 1;
                    cr[w * 32 + b] = 0;
                    bits &= bits - 1u;
                }
            }
        }
    }
}

template <int NT, int V>
cudaError_t launch_k1(const void *X, int64_t rows, int cols, float t, int8_t *codes, float *absmax,
                      int32_t *argmax, uint32_t *bitmap, const DeviceInfo &dev, cudaStream_t stream)
{
    const size_t smem = (size_t)((cols + 31) / 32) * 4;
    auto kern = k_quantize_rows<NT, V>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NT, smem);
    if (e != cudaSuccess)
        return e;
    per_sm = std::max(per_sm, 1);
    const int64_t grid = std::min<int64_t>(rows, (int64_t)per_sm * dev.num_sms);
    kern<<<(unsigned)grid, NT, smem, stream>>>(reinterpret_cast<const uint4 *>(X), rows, cols, t, codes,
                                               absmax, argmax, bitmap);
    return cudaGetLastError();
}

template <int NT>
cudaError_t launch_k1_nt(const void *X, int64_t rows, int cols, float t, int8_t *codes, float *absmax,
                         int32_t *argmax, uint32_t *bitmap, const DeviceInfo &dev, cudaStream_t stream,
                         int v)
{
    switch (v) {
    case 1: return launch_k1<NT, 1>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream);
    case 2: return launch_k1<NT, 2>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream);
    case 4: return launch_k1<NT, 4>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream);
    default: return launch_k1<NT, 8>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream);
    }
}

} // namespace

cudaError_t launch_quantize(const void *X, int64_t rows, int64_t cols64, float t, int8_t *codes,
                            float *absmax, uint32_t *bitmap, int32_t *argmax, int32_t *col_idx,
                            int32_t *count, const DeviceInfo &dev, cudaStream_t stream)
{
    if (rows <= 0 || cols64 <= 0)
        return cudaSuccess;
    const int cols = (int)cols64;
    const int nvec = cols / 8;
    const size_t smem = (size_t)((cols + 31) / 32) * 4;
    cudaError_t e;
    // K1: pick the narrowest block whose registers hold a whole row.
    int nt = 0, v = 0;
    for (int cand_nt : {128, 256, 512, 1024}) {
        int need = (nvec + cand_nt - 1) / cand_nt;
        if (need <= 8) {
            nt = cand_nt;
            v = need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : 8;
            break;
        }
    }
    switch (nt) {
    case 128: e = launch_k1_nt<128>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream, v); break;
    case 256: e = launch_k1_nt<256>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream, v); break;
    case 512: e = launch_k1_nt<512>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream, v); break;
    case 1024: e = launch_k1_nt<1024>(X, rows, cols, t, codes, absmax, argmax, bitmap, dev, stream, v); break;
    default: {
        const int64_t grid = std::min<int64_t>(rows, (int64_t)dev.num_sms * 2);
        k_quantize_rows_loop<1024><<<(unsigned)grid, 1024, smem, stream>>>(
            reinterpret_cast<const uint4 *>(X), rows, cols, t, codes, absmax, argmax, bitmap);
        e = cudaGetLastError();
    }
    }
    if (e != cudaSuccess || !(t > 0.f))
        return e;
    // K2: fix-up, zeroing, compaction.
    const int64_t grid2 = std::min<int64_t>(rows, (int64_t)dev.num_sms * 8);
    k_fixup_rows<256><<<(unsigned)grid2, 256, smem, stream>>>(reinterpret_cast<const uint4 *>(X), rows, cols,
                                                             codes, absmax, argmax, bitmap, col_idx, count);
    return cudaGetLastError();
}

cudaError_t launch_compact(const uint32_t *bitmap, int64_t cols, int32_t *col_idx, int32_t *count,
                           cudaStream_t stream)
{
    const size_t smem = (size_t)((cols + 31) / 32) * 4;
    k_compact<1024><<<1, 1024, smem, stream>>>(bitmap, (int)cols, col_idx, count);
    return cudaGetLastError();
}

} // namespace llmint8
