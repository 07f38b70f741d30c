// Row-wise absmax quantization with outlier-column decomposition.
//
// Method (page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
// accelerate"): absmax quantization with scale 127 / absmax and rounding
// (section "模型量化简介", Introduction to model quantization); hidden-state
// columns holding any |x| >= threshold go to the fp16 side and the rest is
// quantized per row (sections "LLM.int8() 的简要总结" and "MatMul 内部").
//
// The outlier set O is a property of the whole matrix, yet each row's scale
// must exclude O. One fused, cooperatively launched kernel does it:
//   seed      a bounded subset of rows (about 2 MB) is read only to find
//             outlier columns; systematic outlier columns show up in most
//             rows, so this almost always finds all of O;
//   quantize  every row zeroes its known outlier columns, takes its maximum
//             |x| and writes its codes (seeded rows come back from L2);
//   finish    compaction of O; only if some column first reached t during
//             the quantize step are the affected rows re-quantized and the
//             new columns' codes zeroed.
// Both paths give exactly the definition's result. The maximum runs on
// packed fp16 pairs, the outlier test compares against the smallest fp16 >= t
// (exact for fp16 inputs), and the codes round with the 1.5 * 2^23 trick,
// which is round-half-even like rintf.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "internal.h"
#include "llmint8.h"
#include "common.cuh"
#include "ptx.cuh"

namespace llmint8 {

namespace {

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
    __syncwarp();
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
    __syncwarp();
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

__device__ __forceinline__ uint32_t known_byte(const uint32_t *s_known, int vi)
{
    return (s_known[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
}

// Record the columns of one vector with |x| >= t16 in the CTA set and the
// global bitmap; returns true if one of them was new to the bitmap.
__device__ __forceinline__ bool publish_vector(const uint4 &v, int vi, __half t16, uint32_t *s_known,
                                               uint32_t *bitmap)
{
    const uint32_t hit = hit_mask8(v, t16);
    if (!hit)
        return false;
    const uint32_t bits = hit << ((vi & 3) * 8);
    const uint32_t old = atomicOr(&s_known[vi >> 2], bits);
    if (!(bits & ~old))
        return false;
    const uint32_t gold = atomicOr(&bitmap[vi >> 2], bits & ~old);
    return ((bits & ~old) & ~gold) != 0u;
}

// Seed: find the outlier columns of one row (no codes). The last chunk read
// stays in `v` (the whole row when it fits in one chunk).
template <int GS, int V, bool FULL>
__device__ __forceinline__ void row_seed(const uint4 *__restrict__ xr, int nvec, int gl, __half t16,
                                         uint32_t *s_known, uint32_t *bitmap, uint4 (&v)[V])
{
    const __half2 t2 = __half2half2(t16);
    for (int c0 = 0; c0 < nvec; c0 += GS * V) {
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int vi = c0 + u * GS + gl;
            v[u] = (FULL || vi < nvec) ? __ldg(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < V; ++u) {
            __half2 a[4];
            const __half2 vm = vec_abs_max(v[u], a);
            if (__hbgt2(t2, vm)) // both halves below t: no outlier in these 8 columns
                continue;
            (void)publish_vector(v[u], c0 + u * GS + gl, t16, s_known, bitmap);
        }
    }
}

// Maximum |x| of one row over the columns not known as outliers, for a group
// of GS threads holding V vectors each per chunk. Known columns are zeroed in
// `v` in place. `kb4` holds this thread's known-column bytes of the first
// chunk (resident rows); longer rows read them from s_known.
template <int GS, int V, bool THR, bool FULL>
__device__ __forceinline__ float row_max(const uint4 *__restrict__ xr, int nvec, int gl, bool resident,
                                         const uint32_t *s_known, const uint32_t (&kb4)[(V + 3) / 4],
                                         uint4 (&v)[V], bool preloaded)
{
    __half2 m2 = __float2half2_rn(0.f);
    for (int c0 = 0; c0 < nvec; c0 += GS * V) {
        if (!(preloaded && resident)) {
#pragma unroll
            for (int u = 0; u < V; ++u) {
                const int vi = c0 + u * GS + gl;
                v[u] = (FULL || vi < nvec) ? __ldg(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < V; ++u) {
            if constexpr (THR) {
                const int vi = c0 + u * GS + gl;
                const uint32_t kbyte = resident ? (kb4[u >> 2] >> ((u & 3) * 8)) & 0xFFu
                                                : ((FULL || vi < nvec) ? known_byte(s_known, vi) : 0u);
                if (kbyte)
                    mask_known(v[u], kbyte);
            }
            __half2 a[4];
            m2 = __hmax2(m2, vec_abs_max(v[u], a));
        }
    }
    return fmaxf(__low2float(m2), __high2float(m2));
}

// Codes of one row with multiplier s: rint(x * s), zero for known outlier
// columns. Uses `v` (already masked) for resident rows, else reads the row
// again and masks it.
template <int GS, int V, bool THR, bool FULL>
__device__ __forceinline__ void row_codes(const uint4 *__restrict__ xr, int nvec, int gl, bool resident,
                                          const uint32_t *s_known, float s, uint4 (&v)[V], int8_t *__restrict__ cr)
{
    for (int c0 = 0; c0 < nvec; c0 += GS * V) {
        if (!resident) {
#pragma unroll
            for (int u = 0; u < V; ++u) {
                const int vi = c0 + u * GS + gl;
                v[u] = (FULL || vi < nvec) ? __ldg(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
                if constexpr (THR) {
                    if (FULL || vi < nvec) {
                        const uint32_t kbyte = known_byte(s_known, vi);
                        if (kbyte)
                            mask_known(v[u], kbyte);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int vi = c0 + u * GS + gl;
            if (FULL || vi < nvec)
                *reinterpret_cast<uint2 *>(cr + (int64_t)vi * 8) = codes8(v[u], s);
        }
    }
}

// Maximum of a float over a row group of WPR warps (WPR = 1: one warp;
// WPR = 8: the whole CTA, through shared memory; `buf` alternates per row so
// one __syncthreads per reduction suffices).
template <int WPR>
__device__ __forceinline__ float group_max_f32(float v, float *buf)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (WPR > 1) {
        if ((threadIdx.x & 31) == 0)
            buf[threadIdx.x >> 5] = v;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < WPR; ++i)
            v = fmaxf(v, buf[i]);
    }
    return v;
}

// Quantize one row with one group of WPR warps: zero its known outlier
// columns, take the maximum |x|, write codes and absmax. With THR, a row that
// holds a column >= t not yet in s_known publishes it, raises *new_flag and
// gets absmax -1 (a marker: the finish step quantizes it again).
template <int WPR, int V, bool THR, bool FULL>
__device__ __forceinline__ void quantize_row(const uint4 *__restrict__ xr, int64_t r, int cols, float t, __half t16,
                                             bool resident, uint32_t *s_known, uint32_t *bitmap, uint32_t *new_flag,
                                             const uint32_t (&kb4)[(V + 3) / 4], uint4 (&v)[V],
                                             int8_t *__restrict__ codes, float *__restrict__ absmax, float *red,
                                             bool preloaded = false)
{
    constexpr int GS = 32 * WPR;
    const int gl = ((threadIdx.x >> 5) % WPR) * 32 + (threadIdx.x & 31);
    const int nvec = cols >> 3;
    float amax = row_max<GS, V, THR, FULL>(xr, nvec, gl, resident, s_known, kb4, v, preloaded);
    amax = group_max_f32<WPR>(amax, red);
    if (THR && amax >= t) {
        for (int vi = gl; vi < nvec; vi += GS)
            if (publish_vector(__ldg(xr + vi), vi, t16, s_known, bitmap))
                atomicOr(new_flag, 1u);
        if (gl == 0) {
            atomicOr(new_flag, 1u);
            absmax[r] = -1.f;
        }
        return;
    }
    const float s = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
    row_codes<GS, V, THR, FULL>(xr, nvec, gl, resident, s_known, s, v, codes + r * (int64_t)cols);
    if (gl == 0)
        absmax[r] = amax;
}

template <int GS, int V>
__device__ __forceinline__ void load_known_bytes(const uint32_t *s_known, int nvec, int gl, bool resident,
                                                 uint32_t (&kb4)[(V + 3) / 4])
{
#pragma unroll
    for (int i = 0; i < (V + 3) / 4; ++i)
        kb4[i] = 0u;
    if (resident) {
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int vi = u * GS + gl;
            if (vi < nvec)
                kb4[u >> 2] |= known_byte(s_known, vi) << ((u & 3) * 8);
        }
    }
}

constexpr int kMaxLate = 64; // late outlier columns handled by the cheap path

// Fused quantizer, one row per group of WPR warps (WPR = 1: a warp per row;
// WPR = 8: the whole CTA per row). With a threshold (THR):
//   seed     - the first row of every group (rows that fit in registers,
//              kept there for the quantize step), or of every
//              `seed_stride`-th group (longer rows, read again from L2 in the
//              next step), is searched for outlier columns (|x| >= t);
//   barrier  - then each CTA loads the outlier set found so far (the "seed
//              set", also kept aside);
//   quantize - every row: maximum over the columns not known as outliers,
//              codes and absmax;
//   barrier  - then CTA 0 compacts the final outlier set. If no column first
//              reached t during the quantize step (flag sync[2]), every row
//              was coded against the final set and the kernel is done.
//              Otherwise, with L = final set minus seed set, each group
//              re-quantizes those of its rows that were marked, or whose
//              maximum equals |x| at a column of L, and zeroes the L-column
//              codes of its other rows (every row, when |L| > kMaxLate).
// Rows that fit in registers: every group seeds its first row, which stays
// in registers from the seed to its codes. When every row is seeded (rows
// <= groups), the set after the first barrier is final: CTA 0 compacts it
// there and the second barrier is skipped.
// Without a threshold only the quantize step runs. FULL: the row length is a
// multiple of the chunk (no bounds checks). A row of at most 32 * WPR * V
// 16-byte vectors stays in registers between its maximum and its codes; a
// longer one is read twice. The next row of a CTA comes in while this one is
// reduced and coded: into a second register set when a thread holds at most
// 16 vectors, else (rows of more than 4096 vectors, one CTA per SM) into a
// shared-memory buffer by bulk copies that one thread issues, from which the
// threads read it into registers when its turn comes.
template <int WPR, int V, bool THR, bool FULL>
__global__ void __launch_bounds__(256) k_quant_fused(const uint4 *__restrict__ X, int64_t rows, int cols, float t,
                                                     __half t16, int8_t *__restrict__ codes,
                                                     float *__restrict__ absmax, uint32_t *__restrict__ bitmap,
                                                     int32_t *__restrict__ col_idx, int32_t *__restrict__ count,
                                                     uint32_t *__restrict__ sync, uint32_t *__restrict__ status,
                                                     int seed_stride, bool all_seeded)
{
    constexpr int GROUPS = 8 / WPR; // row groups per CTA
    constexpr int GS = 32 * WPR;    // threads per group
    extern __shared__ uint32_t s_dyn[];
    __shared__ float s_red[2][8];
    __shared__ __align__(8) uint64_t s_rowbar; // the buffered row has landed
    __shared__ int s_flag, s_nlate;
    __shared__ int s_late[kMaxLate];
    const int tid = threadIdx.x, warp = tid >> 5;
    const int grp = warp / WPR, gl = (warp % WPR) * 32 + (tid & 31);
    const int64_t gid = (int64_t)blockIdx.x * GROUPS + grp;
    const int64_t G = (int64_t)gridDim.x * GROUPS;
    const int nvec = cols >> 3, nwords = (cols + 31) >> 5;
    const bool resident = nvec <= GS * V;
    uint32_t *s_known = s_dyn;         // [nwords]
    uint32_t *s_seed = s_dyn + nwords; // [nwords]
    uint32_t kb4[(V + 3) / 4];
    uint4 v[V];
    // The next row's buffer (rows of more than 16 vectors a thread): after the
    // sets, 128-byte aligned.
    constexpr bool BULK = WPR > 1 && V > 16;
    const bool bulk = BULK && resident;
    const uint32_t row_bytes = (uint32_t)cols * 2u;
    const int buf_off = THR ? ((2 * nwords * 4 + 127) & ~127) : 0;
    const uint4 *rowbuf = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint8_t *>(s_dyn) + buf_off);
    const uint32_t rowbar = smem_u32(&s_rowbar);
    bool row_inflight = false; // (thread 0) a copy into the buffer has not been waited for
    auto issue_row = [&](int64_t r) { // thread 0: row r into the buffer
        mbar_arrive_expect_tx(rowbar, row_bytes);
        const uint8_t *src = reinterpret_cast<const uint8_t *>(X + r * (int64_t)nvec);
        for (uint32_t off = 0; off < row_bytes; off += 32768u)
            bulk_load(smem_u32(rowbuf) + off, src + off, min(32768u, row_bytes - off), rowbar);
        row_inflight = true;
    };
    if (bulk && tid == 0) {
        mbar_init(rowbar, 1);
        fence_barrier_init();
    }
    griddep_wait();    // (a programmatic dependent) the previous kernel is complete
    griddep_release(); // the GEMM may start its weight stream now; it waits for this kernel's output
    if (!THR)
        __syncthreads(); // the buffer's barrier is initialised

    if constexpr (!THR) {
        if (blockIdx.x == 0 && tid == 0 && count)
            *count = 0; // no outlier columns
    }
    if constexpr (THR) {
        for (int w = tid; w < nwords; w += 256)
            s_known[w] = 0u;
        // The late-column flag is raised only after the first barrier: clear
        // it here (before anyone can raise it) instead of before the launch.
        if (blockIdx.x == 0 && tid == 0)
            sync[2] = 0u;
        __syncthreads();
        // A row that fits in registers is read here once and for all: every
        // group seeds its first row and keeps it for the quantize step, so
        // those reads overlap the barrier. Longer rows: every
        // seed_stride-th group reads its first row only to seed.
        if (gid < rows && (resident || gid % seed_stride == 0))
            row_seed<GS, V, FULL>(X + gid * (int64_t)nvec, nvec, gl, t16, s_known, bitmap, v);
        if (bulk && tid == 0 && gid + G < rows)
            issue_row(gid + G); // the group's second row comes in during the barrier
        __syncthreads();
        if (tid == 0) {
            s_flag = grid_barrier(sync, gridDim.x) ? 1 : 0;
            if (!s_flag)
                atomicOr(status, LLMINT8_DEV_TIMEOUT_QUANT);
        }
        __syncthreads();
        if (!s_flag) {
            if (row_inflight)
                mbar_wait(rowbar, 0u); // the copy lands before the CTA exits
            return;
        }
        for (int w = tid; w < nwords; w += 256)
            s_known[w] = s_seed[w] = __ldcg(bitmap + w);
        __syncthreads();
        // Every row seeded (one row per group): the set is final already.
        if (all_seeded && blockIdx.x == 0)
            compact_block<256>(s_known, nwords, col_idx, count);
    }

    load_known_bytes<GS, V>(s_known, nvec, gl, THR && resident, kb4);
    // With the whole CTA on a row that fits in registers (at most 16 vectors
    // a thread), the next row is read into a second register set while this
    // one is reduced and coded: two rows in flight per CTA.
    constexpr bool PREFETCH = WPR > 1 && V <= 16;
    auto load_row = [&](int64_t r, uint4(&dst)[V]) {
        const uint4 *xr = X + r * (int64_t)nvec;
#pragma unroll
        for (int u = 0; u < V; ++u) {
            const int vi = u * GS + gl;
            dst[u] = (FULL || vi < nvec) ? __ldg(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint4 vn[PREFETCH ? V : 1];
    int it = 0;
    bool row_ok = true;
    for (int64_t r = gid; r < rows; r += G, ++it) {
        bool pre = THR && resident && it == 0; // the seed step left the first row in v
        if (BULK && bulk) {
            if (it == 0 && !pre) {
                load_row(r, v);
                pre = true;
            } else if (it > 0) {
                // this row came into the buffer during the previous one
                row_ok = row_ok && mbar_wait(rowbar, (uint32_t)(it - 1) & 1u);
#pragma unroll
                for (int u = 0; u < V; ++u) {
                    const int vi = u * GS + gl;
                    v[u] = (FULL || vi < nvec) ? rowbuf[vi] : make_uint4(0u, 0u, 0u, 0u);
                }
                pre = true;
            }
            __syncthreads(); // every thread has its values: the buffer takes the next row
            if (tid == 0) {
                row_inflight = false;
                if (r + G < rows && !(THR && it == 0)) { // (with a threshold row 1 went out before the barrier)
                    fence_proxy_async_smem();
                    issue_row(r + G);
                }
            }
        }
        if constexpr (PREFETCH) {
            if (resident) {
                if (it == 0 && !pre)
                    load_row(r, v);
                pre = true;
                if (r + G < rows)
                    load_row(r + G, vn);
            }
        }
        quantize_row<WPR, V, THR, FULL>(X + r * (int64_t)nvec, r, cols, t, t16, resident, s_known, bitmap,
                                        sync + 2, kb4, v, codes, absmax, s_red[it & 1], pre);
        if constexpr (PREFETCH) {
            if (resident) {
#pragma unroll
                for (int u = 0; u < V; ++u)
                    v[u] = vn[u];
            }
        }
    }
    if (BULK && bulk && !row_ok && gl == 0)
        atomicOr(status, LLMINT8_DEV_TIMEOUT_QUANT); // a buffered row did not land in time
    if constexpr (!THR)
        return;
    if (all_seeded)
        return; // no row can hold a column the seed did not see

    // ---- finish
    __syncthreads();
    if (tid == 0) {
        s_flag = grid_barrier(sync, gridDim.x) ? 1 : 0;
        if (!s_flag)
            atomicOr(status, LLMINT8_DEV_TIMEOUT_QUANT);
    }
    __syncthreads();
    if (!s_flag)
        return;
    for (int w = tid; w < nwords; w += 256)
        s_known[w] = __ldcg(bitmap + w);
    __syncthreads();
    if (blockIdx.x == 0)
        compact_block<256>(s_known, nwords, col_idx, count);
    if (__ldcg(sync + 2) == 0u)
        return; // every row was coded against the complete outlier set

    // Late columns: in the final set but not in the seed set.
    if (tid == 0)
        s_nlate = 0;
    __syncthreads();
    for (int w = tid; w < nwords; w += 256) {
        uint32_t bits = s_known[w] & ~s_seed[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            const int k = atomicAdd(&s_nlate, 1);
            if (k < kMaxLate)
                s_late[k] = w * 32 + b;
            bits &= bits - 1u;
        }
    }
    __syncthreads();
    const int nlate = s_nlate;
    load_known_bytes<GS, V>(s_known, nvec, gl, resident, kb4);
    it = 0;
    for (int64_t r = gid; r < rows; r += G, ++it) {
        const float a = __ldcg(absmax + r);
        const __half *xh = reinterpret_cast<const __half *>(X + r * (int64_t)nvec);
        bool redo = a < 0.f || nlate > kMaxLate;
        if (!redo) {
            for (int k = gl; k < nlate; k += GS)
                redo |= a > 0.f && __half2float(__habs(xh[s_late[k]])) == a;
        }
        if constexpr (WPR == 1)
            redo = __any_sync(0xffffffffu, redo);
        else
            redo = __syncthreads_or(redo);
        if (redo) {
            quantize_row<WPR, V, true, FULL>(X + r * (int64_t)nvec, r, cols, t, t16, resident, s_known, bitmap,
                                             sync + 2, kb4, v, codes, absmax, s_red[it & 1]);
        } else {
            for (int k = gl; k < nlate; k += GS)
                codes[r * (int64_t)cols + s_late[k]] = 0;
        }
    }
}

template <int WPR, int V, bool THR, bool FULL>
cudaError_t launch_fused(const void *X, int64_t rows, int cols, float t, int8_t *codes, float *absmax,
                         uint32_t *bitmap, int32_t *col_idx, int32_t *count, uint32_t *sync, uint32_t *status,
                         const DeviceInfo &dev, cudaStream_t stream)
{
    constexpr int GROUPS = 8 / WPR;
    const size_t sets = THR ? (size_t)((cols + 31) / 32) * 4 * 2 : 0;
    // rows of more than 16 vectors a thread held in registers: the next row's buffer after the sets
    const bool bulk = WPR > 1 && V > 16 && (cols >> 3) <= 32 * WPR * V;
    const size_t smem = bulk ? ((sets + 127) & ~(size_t)127) + (size_t)cols * 2 : sets;
    auto kern = k_quant_fused<WPR, V, THR, FULL>;
    if (smem > 48 * 1024) {
        static std::mutex amu;
        static int attr_dev = -1;
        std::lock_guard<std::mutex> lock(amu);
        if (attr_dev != dev.device) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, kern);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dev.max_smem_optin - (int)fa.sharedSizeBytes);
            if (e != cudaSuccess)
                return e;
            attr_dev = dev.device;
        }
    }
    // Resident CTAs per SM, cached per (kernel, device, shared memory in 1 KB steps).
    static std::mutex mu;
    static std::map<std::pair<int, size_t>, int> occ;
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        const auto key = std::make_pair(dev.device, (smem + 1023) / 1024);
        auto it = occ.find(key);
        if (it != occ.end()) {
            per_sm = it->second;
        } else {
            cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, key.second * 1024);
            if (e != cudaSuccess)
                return e;
            occ[key] = per_sm;
        }
    }
    if (per_sm < 1)
        return cudaErrorInvalidConfiguration;
    const int64_t want = (rows + GROUPS - 1) / GROUPS;
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)per_sm * dev.num_sms);
    // Seed about 2 MB of rows (at least 64 rows, all rows when fewer): every
    // seed_stride-th row group seeds its first row. A column that misses the
    // seed is still handled exactly, by the finish step.
    const int64_t groups = std::min<int64_t>(rows, (int64_t)grid * GROUPS);
    const int64_t row_bytes = (int64_t)cols * 2;
    const int64_t seed_rows = std::min<int64_t>(groups, std::max<int64_t>(64, (2ll << 20) / row_bytes));
    const int seed_stride = (int)std::max<int64_t>(1, groups / std::max<int64_t>(1, seed_rows));
    const __half t16 = threshold_fp16(t);
    const uint4 *xp = reinterpret_cast<const uint4 *>(X);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative; // the barriers need every CTA resident
    attr[0].val.cooperative = THR ? 1 : 0;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization; // launch overlaps the previous tail
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const bool resident = (cols >> 3) <= 32 * WPR * V;
    const bool all_seeded = rows <= groups && (resident || seed_stride == 1);
    return cudaLaunchKernelEx(&cfg, kern, xp, rows, cols, t, t16, codes, absmax, bitmap, col_idx, count, sync,
                              status, seed_stride, all_seeded);
}

template <int WPR, int V>
cudaError_t launch_fused_v(const void *X, int64_t rows, int cols, float t, int8_t *codes, float *absmax,
                           uint32_t *bitmap, int32_t *col_idx, int32_t *count, uint32_t *sync, uint32_t *status,
                           const DeviceInfo &dev, cudaStream_t stream)
{
    const bool thr = t > 0.f;
    const bool full = ((cols >> 3) % (32 * WPR * V)) == 0;
    if (thr)
        return full ? launch_fused<WPR, V, true, true>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count,
                                                       sync, status, dev, stream)
                    : launch_fused<WPR, V, true, false>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count,
                                                        sync, status, dev, stream);
    return full ? launch_fused<WPR, V, false, true>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count, sync,
                                                    status, dev, stream)
                : launch_fused<WPR, V, false, false>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count, sync,
                                                     status, dev, stream);
}

// The quantizer for an X that fits in the shared memory of one CTA per SM,
// with rows of up to 4096 columns. Each CTA holds its block of rows
// (contiguous in X) for the whole call. The block arrives as chunks of whole
// rows, each bulk-copied into shared memory on an mbarrier of its own (a few
// chunks in flight at a time), and each of 15 worker warps takes rows
// w, w + 15, ... as they land, a row in the warp's registers. Per row
// (threshold on):
//   detect - the row's outlier columns (|x| >= t16) join the CTA's set s_bm;
//            a column new to it is counted in s_cnt;
//   c      - the size of the set the row is quantized against: each lane
//            caches the set bytes of its vectors, read after reading c, and
//            reads them again when s_cnt has moved or the row added to it;
//   row    - maximum over the columns outside the set, codes
//            rint(x * 127 / absmax) (set columns 0) and absmax.
// A control warp, once every row is detected, ORs the CTA's set into this
// call's global bitmap, passes the grid barrier and reads the complete set
// back. (The workers never wait for global memory: they start on the first
// rows as soon as those land.) Sets only grow and every column counted in c
// was in s_bm before the row read it, so a row whose c equals the size of
// the complete set used exactly that set; the others (a column that only a
// later row, or another CTA, saw) are quantized again from shared memory.
// A short seed step (the first rows of the block detected before any row
// goes on) makes that rare. The result is the definition's after a single
// read of X from HBM, with the codes written while the block still arrives
// and the grid barrier's latency behind the last rows.
//
// The global bitmap is one of two in the workspace: call n (the workspace's
// call counter) ORs into set[n & 1], and CTA 0 clears set[(n + 1) & 1],
// which no CTA of this call reads, for call n + 1.
constexpr int kQsWorkers = 480;                 // 15 worker warps (16 warps in all: 128 registers a thread)
constexpr int kQsWarps = kQsWorkers / 32;
constexpr int kQsThreads = kQsWorkers + 32;     // + the control warp
constexpr int kQsMaxChunks = 64;
constexpr int kQsChunkBytes = 4096;
constexpr int kQsSeedRows = 4;
constexpr int kQsInFlight = 8;                  // chunks of one CTA requested ahead
constexpr int kQsRegVec = 16;                   // rows of up to 32 * 16 vectors stay in registers

// Rows of one CTA per chunk: at least kQsChunkBytes, at most kQsMaxChunks chunks.
__host__ __device__ inline int qs_rows_per_chunk(int nr, int cols)
{
    const int by_size = (kQsChunkBytes + cols * 2 - 1) / (cols * 2);
    return max(max(by_size, 1), (nr + kQsMaxChunks - 1) / kQsMaxChunks);
}

__device__ __forceinline__ uint32_t set_byte(const uint32_t *bm, int v)
{
    return (bm[v >> 2] >> ((v & 3) * 8)) & 0xFFu;
}

struct QsRow {
    const uint4 *xr; // the row in shared memory
    int nvec;
    __half t16;
    uint32_t *s_bm;  // the CTA's set (detection adds to it)
    int *s_cnt;      // its size
    int8_t *cr;      // the row's codes
    float *am;       // the row's absmax (zero-point codes: its scale s)
    int32_t *zp;     // zero-point codes: the row's zero point
    int lane;
};

// Add the outlier columns of vector v (x) to the CTA's set, then count the
// ones new to it. (The control warp ORs the CTA's whole set into this call's
// global bitmap once every row is detected.) Returns true if it added any.
// Out of line: it runs for the few vectors holding an outlier, and inlined
// into every unrolled step it would crowd the instruction cache that the
// common path runs from.
__device__ __noinline__ bool qs_publish(uint4 x, int v, __half t16, uint32_t *s_bm, int *s_cnt)
{
    const uint32_t bits = hit_mask8(x, t16) << ((v & 3) * 8);
    const int w = v >> 2;
    const uint32_t nb = bits & ~atomicOr(&s_bm[w], bits);
    if (!nb)
        return false;
    __threadfence_block(); // the bits are in s_bm before the count says so
    atomicAdd(s_cnt, __popc(nb));
    return true;
}

// |x| maximum of the vector; if it reaches t16, the vector's outlier
// columns not among `known` (bits of the vector's columns already seen in
// the CTA's set) are published (pub set when any was new to the CTA).
__device__ __forceinline__ __half2 qs_detect_vec(const QsRow &q, int v, const uint4 &x, uint32_t known, bool &pub)
{
    __half2 a[4];
    const __half2 m = vec_abs_max(x, a);
    if (__hge(__hmax(__low2half(m), __high2half(m)), q.t16) && (hit_mask8(x, q.t16) & ~known))
        pub |= qs_publish(x, v, q.t16, q.s_bm, q.s_cnt);
    return m;
}

// Size of the CTA's set, read by lane 0 after the warp's detection and
// ordered before every later read of s_bm by the warp.
__device__ __forceinline__ int qs_count(const QsRow &q)
{
    __syncwarp();
    int c = 0;
    if (q.lane == 0)
        c = *reinterpret_cast<volatile int *>(q.s_cnt);
    __threadfence_block();
    c = __shfl_sync(0xffffffffu, c, 0);
    __syncwarp();
    return c;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float qs_scale(float amax) { return amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f; }

// Set bytes of one lane's vectors (lane + 32 k), four to a word, and the
// count c they were read after.
struct QsSetCache {
    uint32_t b[kQsRegVec / 4];
    int count;
};

__device__ __forceinline__ void qs_load_set(QsSetCache &sc, const uint32_t *bm, int nvec, int lane, int count)
{
#pragma unroll
    for (int j = 0; j < kQsRegVec / 4; ++j) {
        uint32_t w = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int v = lane + 32 * (4 * j + i);
            if (v < nvec)
                w |= set_byte(bm, v) << (8 * i);
        }
        sc.b[j] = w;
    }
    sc.count = count;
}

// The warp's last arrival at the detection barrier (its rows' columns are in
// the CTA's set; the barrier orders them before the control warp reads it).
__device__ __forceinline__ void qs_arrive_detected(bool pub)
{
    (void)pub;
    named_barrier_arrive(2, kQsThreads);
}

// One row held in registers (nvec <= 32 * kQsRegVec), against the CTA's set
// through the lane's cache sc (or, fixed, against the set sc already holds:
// no detection, no count). Known outlier columns are masked first; a vector
// whose remaining maximum still reaches t16 holds a column the cache did not
// have, and only then is the row's new part of the set published and the
// maximum taken again against the set read afresh. Returns the count the
// row's set was read after (0 when !THR or fixed).
// ASYM: zero-point codes instead (page "Hugging Face 将 LLM.int8() 8-bit 量化
// 集成进 transformers 与 accelerate", section "模型量化简介"): over the row's
// values with the known columns zeroed, [lo, hi] = [min(0, min x),
// max(0, max x)] on packed fp16, s = 255 / (hi - lo) in fp32 (0 for an
// all-zero row), z = rint(-lo * s), q = clamp(rint(x * s) + z, 0, 255)
// stored as q - 128 (a zeroed column gets q = z). rint is the 1.5 * 2^23
// addition in round-to-nearest-even, exact here: |x * s| <= 255 (+ rounding).
template <bool THR, bool FULL, bool ASYM>
__device__ int qs_row_reg(const QsRow &q, QsSetCache &sc, bool fixed, bool &pub, bool arrive)
{
    uint4 x[kQsRegVec];
#pragma unroll
    for (int k = 0; k < kQsRegVec; ++k) {
        const int v = q.lane + 32 * k;
        x[k] = (FULL || v < q.nvec) ? q.xr[v] : make_uint4(0u, 0u, 0u, 0u);
    }
    if (THR && !fixed) { // the set grew since the cache was read: read it again
        int now = 0;
        if (q.lane == 0)
            now = *reinterpret_cast<volatile int *>(q.s_cnt);
        if (__shfl_sync(0xffffffffu, now, 0) != sc.count)
            qs_load_set(sc, q.s_bm, q.nvec, q.lane, qs_count(q));
    }
    __half2 rm = __float2half2_rn(0.f);
#pragma unroll
    for (int k = 0; k < kQsRegVec; ++k) {
        if (THR) {
            const uint32_t kb = (sc.b[k >> 2] >> (8 * (k & 3))) & 0xFFu;
            if (kb)
                mask_known(x[k], kb);
        }
        __half2 a[4];
        rm = __hmax2(rm, vec_abs_max(x[k], a));
    }
    // The maximum over the columns left reaches t16 exactly when one of
    // them is an outlier column the cache did not have.
    if (THR && !fixed && __any_sync(0xffffffffu, __hge(__hmax(__low2half(rm), __high2half(rm)), q.t16))) {
        // columns new to this lane's cache: into the CTA's set, then the
        // maximum again against the set read afresh
#pragma unroll
        for (int k = 0; k < kQsRegVec; ++k) {
            __half2 a[4];
            const __half2 mk = vec_abs_max(x[k], a);
            if (__hge(__hmax(__low2half(mk), __high2half(mk)), q.t16))
                pub |= qs_publish(x[k], q.lane + 32 * k, q.t16, q.s_bm, q.s_cnt);
        }
        qs_load_set(sc, q.s_bm, q.nvec, q.lane, qs_count(q));
        rm = __float2half2_rn(0.f);
#pragma unroll
        for (int k = 0; k < kQsRegVec; ++k) {
            const uint32_t kb = (sc.b[k >> 2] >> (8 * (k & 3))) & 0xFFu;
            if (kb)
                mask_known(x[k], kb);
            __half2 a[4];
            rm = __hmax2(rm, vec_abs_max(x[k], a));
        }
    }
    if (THR && arrive)
        qs_arrive_detected(pub);
    if constexpr (ASYM) {
        __half2 lo2 = __float2half2_rn(0.f), hi2 = __float2half2_rn(0.f);
#pragma unroll
        for (int k = 0; k < kQsRegVec; ++k) {
            const __half2 *h = reinterpret_cast<const __half2 *>(&x[k]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lo2 = __hmin2(lo2, h[i]);
                hi2 = __hmax2(hi2, h[i]);
            }
        }
        float lo = fminf(__low2float(lo2), __high2float(lo2));
        float hi = fmaxf(__low2float(hi2), __high2float(hi2));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const float range = __fsub_rn(hi, lo);
        const float s = range > 0.f ? __fdiv_rn(255.0f, range) : 0.f;
        const int z = (int)(__float_as_uint(__fadd_rn(__fmul_rn(-lo, s), 12582912.0f)) - 0x4B400000u);
        // rint(x s) + z = (bits of x s + 1.5 * 2^23) - 0x4B400000 + z
        const int zoff = z - (int)0x4B400000u;
#pragma unroll
        for (int k = 0; k < kQsRegVec; ++k) {
            const int v = q.lane + 32 * k;
            if (FULL || v < q.nvec) {
                const __half2 *h = reinterpret_cast<const __half2 *>(&x[k]);
                uint32_t b[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __half22float2(h[i]);
                    const int q0 = (int)__float_as_uint(__fadd_rn(__fmul_rn(f.x, s), 12582912.0f)) + zoff;
                    const int q1 = (int)__float_as_uint(__fadd_rn(__fmul_rn(f.y, s), 12582912.0f)) + zoff;
                    b[2 * i] = (uint32_t)(min(max(q0, 0), 255) - 128) & 0xFFu;
                    b[2 * i + 1] = (uint32_t)(min(max(q1, 0), 255) - 128) & 0xFFu;
                }
                *reinterpret_cast<uint2 *>(q.cr + (int64_t)v * 8) =
                    make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                               b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
            }
        }
        if (q.lane == 0) {
            *q.am = s;
            *q.zp = z;
        }
    } else {
        const float amax = warp_max(fmaxf(__low2float(rm), __high2float(rm)));
        const float s = qs_scale(amax);
#pragma unroll
        for (int k = 0; k < kQsRegVec; ++k) {
            const int v = q.lane + 32 * k;
            if (FULL || v < q.nvec)
                *reinterpret_cast<uint2 *>(q.cr + (int64_t)v * 8) = codes8(x[k], s);
        }
        if (q.lane == 0)
            *q.am = amax;
    }
    return (THR && !fixed) ? sc.count : 0;
}

template <bool THR, bool FULL, bool ASYM>
__global__ void __launch_bounds__(kQsThreads, 1)
    k_quant_smem(const uint4 *__restrict__ X, int rows, int cols, __half t16, int8_t *__restrict__ codes,
                 float *__restrict__ absmax, int32_t *__restrict__ zero, uint32_t *__restrict__ bitmap_out,
                 uint32_t *sets, uint32_t *calls, unsigned long long *arrivals, int32_t *__restrict__ col_idx,
                 int32_t *__restrict__ count, uint32_t *__restrict__ status)
{
    extern __shared__ __align__(1024) uint8_t q_smem[];
    __shared__ uint64_t s_bars[kQsMaxChunks];
    __shared__ int s_cnt, s_gcount, s_fail, s_flag;
    __shared__ uint32_t s_call;
    __shared__ unsigned long long s_target;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nvec = cols >> 3, nwords = (cols + 31) >> 5;
    const int G = gridDim.x, c = blockIdx.x;
    const int r0 = (int)((int64_t)c * rows / G), r1 = (int)((int64_t)(c + 1) * rows / G);
    const int nr = r1 - r0;
    const int rpc = qs_rows_per_chunk(max(nr, 1), cols);
    const int nch = (nr + rpc - 1) / rpc;
    const uint4 *sx = reinterpret_cast<const uint4 *>(q_smem);
    const uint32_t xbytes = (uint32_t)nr * (uint32_t)cols * 2u;
    uint32_t *s_bm = reinterpret_cast<uint32_t *>(q_smem + ((xbytes + 15u) & ~15u)); // the CTA's set
    uint32_t *s_gbm = s_bm + nwords;                                                  // the complete set
    // Launched as a programmatic dependent: the kernel before this one may
    // still be finishing; nothing here touches global memory before it has.
    griddep_wait();
    griddep_release();

    if (warp == kQsWarps) {
        // ------------------------------------------------ control warp
        if (lane == 0) {
            for (int j = 0; j < nch; ++j)
                mbar_init(smem_u32(&s_bars[j]), 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            s_call = 0u;
            s_cnt = 0;
            s_gcount = 0;
            s_fail = 0;
            s_flag = 1;
        }
        __syncwarp();
        __syncthreads();
        // At most kQsInFlight chunks of this CTA in flight: the next is
        // requested when the oldest lands, so that every CTA's rows arrive as
        // a steady stream from the start (with all of them requested at once,
        // the order HBM serves them in left some CTAs without their first
        // rows until most of X had arrived). Lane 0 issues.
        const uint8_t *src = reinterpret_cast<const uint8_t *>(X + (int64_t)r0 * nvec);
        auto issue = [&](int j) {
            const uint32_t b0 = (uint32_t)(j * rpc) * (uint32_t)cols * 2u;
            const uint32_t b1 = min(xbytes, (uint32_t)((j + 1) * rpc) * (uint32_t)cols * 2u);
            const uint32_t bar = smem_u32(&s_bars[j]);
            mbar_arrive_expect_tx(bar, b1 - b0);
            for (uint32_t off = b0; off < b1; off += 32768u)
                bulk_load(smem_u32(q_smem) + off, src + off, min(32768u, b1 - off), bar);
        };
        if (lane == 0) {
            for (int j = 0; j < min(nch, kQsInFlight); ++j)
                issue(j);
            if (THR) {
                // The counters only after the first copies are on their way
                // (each read is a global round trip): which global bitmap this
                // call uses, and the arrival count its barrier opens at (the
                // next multiple of the grid; CTAs that arrived already are
                // below it).
                s_call = *reinterpret_cast<volatile uint32_t *>(calls);
                unsigned long long a;
                asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(a) : "l"(arrivals) : "memory");
                s_target = a - a % (unsigned long long)G + (unsigned long long)G;
            }
        }
        if (lane == 0) {
            for (int j = kQsInFlight; j < nch; ++j) {
                if (!mbar_wait(smem_u32(&s_bars[j - kQsInFlight]), 0u))
                    s_fail = 1; // the workers' wait on that chunk fails too
                issue(j);
            }
        }
        if (THR) {
            named_barrier_sync(2, kQsThreads); // every row detected, its columns in s_bm
            __syncwarp();
            const uint32_t call = __shfl_sync(0xffffffffu, s_call, 0);
            // The CTA's set into this call's global bitmap (nonzero words only);
            // CTA 0 also clears the other bitmap for the next call, which no
            // CTA of this call reads.
            uint32_t *myset = sets + (call & 1u) * kSetWords;
            for (int w = lane; w < nwords; w += 32) {
                const uint32_t b = s_bm[w];
                if (b)
                    atomicOr(myset + w, b);
            }
            if (c == 0) {
                uint32_t *next = sets + ((call + 1u) & 1u) * kSetWords;
                for (int w = lane; w < (int)kSetWords; w += 32)
                    next[w] = 0u;
            }
            __threadfence(); // this lane's ORs (and clears) before lane 0's release below
            __syncwarp();
            bool passed = true;
            if (lane == 0) {
                // Grid barrier: one posted add per CTA (release: the CTA's
                // bits, made visible by its workers' fences, come first),
                // then wait for the count to reach this call's target.
                asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(arrivals) : "memory");
                const uint64_t t0 = global_timer_ns();
                for (;;) {
                    unsigned long long a;
                    asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(a) : "l"(arrivals) : "memory");
                    if ((long long)(a - s_target) >= 0)
                        break;
                    if (global_timer_ns() - t0 > kWaitLimitNs) {
                        passed = false;
                        break;
                    }
                }
            }
            passed = __shfl_sync(0xffffffffu, passed, 0);
            const uint32_t *gset = sets + (s_call & 1u) * kSetWords;
            int n = 0;
            for (int w = lane; w < nwords; w += 32) {
                const uint32_t g = __ldcg(gset + w);
                s_gbm[w] = g;
                n += __popc(g);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                n += __shfl_xor_sync(0xffffffffu, n, o);
            if (lane == 0) {
                s_gcount = n;
                if (!passed)
                    s_flag = 0;
                if (c == 0) // every CTA read the counter before the barrier
                    *reinterpret_cast<volatile uint32_t *>(calls) = s_call + 1u;
            }
            named_barrier_arrive(3, kQsThreads); // the complete set is in s_gbm
        }
    } else {
        // ------------------------------------------------ worker warps
        for (int w = tid; w < nwords; w += kQsWorkers)
            s_bm[w] = 0u;
        __syncthreads();
        QsRow q;
        q.nvec = nvec;
        q.t16 = t16;
        q.s_bm = s_bm;
        q.s_cnt = &s_cnt;
        q.lane = lane;
        QsSetCache sc;
        sc.count = -1;
        bool ok = true, pub = false;
        // seed: the first rows of the block, spread over every worker, are
        // detected before any row is quantized
        const int nseed = THR ? min(nr, kQsSeedRows) : 0;
        if (THR) {
            for (int j = 0; j * rpc < nseed; ++j)
                if (!mbar_wait(smem_u32(&s_bars[j]), 0u))
                    ok = false;
            if (ok) {
                const int n = nseed * nvec;
                int i = tid, v = tid % nvec;
                const int step = kQsWorkers % nvec;
                for (; i < n; i += kQsWorkers) {
                    qs_detect_vec(q, v, sx[i], set_byte(s_bm, v), pub);
                    v += step;
                    if (v >= nvec)
                        v -= nvec;
                }
            }
            named_barrier_sync(1, kQsWorkers);
        }
        int cmin = INT_MAX;
        if (THR && warp >= nr)
            qs_arrive_detected(pub); // no rows: nothing to detect
        for (int r = warp; r < nr; r += kQsWarps) {
            const bool last = r + kQsWarps >= nr;
            if (!mbar_wait(smem_u32(&s_bars[r / rpc]), 0u)) {
                ok = false;
                if (THR && last)
                    qs_arrive_detected(pub);
                continue;
            }
            q.xr = sx + (int64_t)r * nvec;
            q.cr = codes + (int64_t)(r0 + r) * cols;
            q.am = absmax + r0 + r;
            q.zp = zero + r0 + r;
            cmin = min(cmin, qs_row_reg<THR, FULL, ASYM>(q, sc, false, pub, last));
        }
        if (THR) {
            named_barrier_sync(3, kQsThreads);
            if (s_flag && __all_sync(0xffffffffu, ok)) {
                const int total = s_gcount;
                if (cmin != INT_MAX && cmin != total) { // a row saw only part of the set: this warp's rows again
                    qs_load_set(sc, s_gbm, nvec, lane, total);
                    for (int r = warp; r < nr; r += kQsWarps) {
                        q.xr = sx + (int64_t)r * nvec;
                        q.cr = codes + (int64_t)(r0 + r) * cols;
                        q.am = absmax + r0 + r;
                        q.zp = zero + r0 + r;
                        qs_row_reg<THR, FULL, ASYM>(q, sc, true, pub, false);
                    }
                }
            }
        }
        if (!__all_sync(0xffffffffu, ok) && lane == 0)
            s_fail = 1;
    }
    __syncwarp();
    __syncthreads();
    if (tid == 0 && (s_fail || !s_flag))
        atomicOr(status, LLMINT8_DEV_TIMEOUT_QUANT);
    if (c == 0) {
        const uint32_t *fin = THR ? s_gbm : s_bm;
        if (bitmap_out)
            for (int w = tid; w < nwords; w += kQsThreads)
                bitmap_out[w] = fin[w];
        if (THR)
            compact_block<kQsThreads>(fin, nwords, col_idx, count);
        else if (tid == 0)
            *count = 0;
    }
}

} // namespace

// The smallest fp16 value >= t, so that for fp16 x, |x| >= t exactly when
// |x| >= t16 (t above the fp16 range: no finite value qualifies).
__half threshold_fp16(float t)
{
    if (!(t > 0.f))
        return __float2half(0.f);
    if (t > 65504.f)
        return __ushort_as_half((unsigned short)0x7C00u); // +inf
    __half h = __float2half_rn(t);
    if (__half2float(h) < t)
        h = __ushort_as_half((unsigned short)(__half_as_ushort(h) + 1u));
    return h;
}

cudaError_t launch_quantize(const void *X, int64_t rows, int64_t cols64, float t, int8_t *codes,
                            float *absmax, uint32_t *bitmap, int32_t *col_idx, int32_t *count, uint32_t *sync,
                            uint32_t *status, const DeviceInfo &dev, cudaStream_t stream)
{
    if (rows <= 0 || cols64 <= 0)
        return cudaSuccess;
    const int cols = (int)cols64;
    const int nvec = cols / 8;
    // Many rows of up to 4096 columns: one warp per row, the row in registers
    // (16 vectors a thread). Otherwise the whole CTA on each row, with 8, 16
    // or 32 vectors a thread, so that rows of up to 65536 columns stay in
    // registers and are read from HBM once; longer rows are read twice.
    if (rows >= (int64_t)dev.num_sms * 8 && nvec <= 32 * 16)
        return launch_fused_v<1, 16>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count, sync, status, dev,
                                     stream);
    if (nvec <= 256 * 16 && nvec > 256 * 8)
        return launch_fused_v<8, 16>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count, sync, status, dev,
                                     stream);
    if (nvec <= 256 * 32 && nvec > 256 * 16)
        return launch_fused_v<8, 32>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count, sync, status, dev,
                                     stream);
    // Rows of exactly 7 vectors a thread (14336 columns, BLOOM-176B's hidden
    // width): no empty eighth vector and no bounds checks (measured on B200:
    // 2048 x 14336 in 27.0 instead of 28.7 us).
    if (nvec == 256 * 7)
        return launch_fused_v<8, 7>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count, sync, status, dev,
                                    stream);
    return launch_fused_v<8, 8>(X, rows, cols, t, codes, absmax, bitmap, col_idx, count, sync, status, dev, stream);
}

namespace {

size_t quant_smem_bytes(int64_t rows, int64_t cols, int num_sms)
{
    // the block of rows, then the CTA's set and the complete set
    const int64_t per = (rows + num_sms - 1) / num_sms;
    return (size_t)((per * cols * 2 + 15) & ~15ll) + (size_t)((cols + 31) / 32) * 8;
}

} // namespace

bool quantize_smem_fits(int64_t rows, int64_t cols, const DeviceInfo &dev)
{
    // Rows that a warp holds in registers, and room for the block of rows and
    // the two bitmaps under the opt-in limit, with a margin for the kernel's
    // static shared memory. (Longer rows go to the streaming quantizer, which
    // keeps a row of up to 65536 columns in the registers of one CTA.)
    return rows >= 1 && cols >= 8 && cols % 8 == 0 && cols <= 8 * 32 * kQsRegVec && rows <= INT32_MAX &&
           quant_smem_bytes(rows, cols, dev.num_sms) + 2048 <= (size_t)dev.max_smem_optin;
}

cudaError_t launch_quantize_smem(const void *X, int64_t rows, int64_t cols, float t, int8_t *codes, float *absmax,
                                 uint32_t *bitmap_out, uint32_t *sets, uint32_t *calls,
                                 unsigned long long *arrivals, int32_t *col_idx, int32_t *count,
                                 uint32_t *status, const DeviceInfo &dev, cudaStream_t stream, int32_t *zero)
{
    const bool thr = t > 0.f;
    const bool full = cols / 8 == 32 * kQsRegVec;
    const bool asym = zero != nullptr;
    auto kern = asym ? (thr ? (full ? k_quant_smem<true, true, true> : k_quant_smem<true, false, true>)
                            : (full ? k_quant_smem<false, true, true> : k_quant_smem<false, false, true>))
                     : (thr ? (full ? k_quant_smem<true, true, false> : k_quant_smem<true, false, false>)
                            : (full ? k_quant_smem<false, true, false> : k_quant_smem<false, false, false>));
    const size_t smem = quant_smem_bytes(rows, cols, dev.num_sms);
    static std::mutex mu;
    static std::map<std::pair<int, int>, size_t> configured; // (device, variant) -> bytes set
    {
        std::lock_guard<std::mutex> lock(mu);
        size_t &have = configured[std::make_pair(dev.device, (thr ? 1 : 0) + (full ? 2 : 0) + (asym ? 4 : 0))];
        if (have < smem) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 dev.max_smem_optin - 1024);
            if (e != cudaSuccess)
                return e;
            have = (size_t)dev.max_smem_optin - 1024;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)dev.num_sms);
    cfg.blockDim = dim3(kQsThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative; // the grid barrier needs every CTA resident
    attr[0].val.cooperative = 1;
    // the launch itself may overlap the previous kernel's tail (the kernel
    // waits for it before reading anything): ~1 us a call on B200
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const uint4 *>(X), (int)rows, (int)cols,
                              threshold_fp16(t), codes, absmax, zero, bitmap_out, sets, calls, arrivals, col_idx, count,
                              status);
}

namespace {

// Zero-point quantization of the rows: the unsigned-int8 alternative to
// absmax (page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
// accelerate", section "模型量化简介": subtract the minimum, scale by the
// range, with 0 exactly representable), one warp per row. Over the columns
// not in `bitmap` (null: every column): range [lo, hi] = [min(0, min x),
// max(0, max x)], s = 255 / (hi - lo) in fp32 (0 for an all-zero row), zero
// point z = rint(-lo * s), code q = clamp(rint(x * s) + z, 0, 255) stored as
// the int8 value q - 128; columns in `bitmap` get q = z, so that they drop
// out once z is taken off. Outlier columns are zeroed before the range is
// taken (0 lies inside it anyway).
__global__ void __launch_bounds__(256) k_quant_asym(const uint4 *__restrict__ X, int64_t rows, int cols,
                                                    const uint32_t *__restrict__ bitmap, int8_t *__restrict__ codes,
                                                    float *__restrict__ scale, int32_t *__restrict__ zero)
{
    extern __shared__ uint32_t s_abm[];
    const int nvec = cols >> 3, nwords = (cols + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += blockDim.x)
        s_abm[w] = bitmap ? bitmap[w] : 0u;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nwarps) {
        const uint4 *xr = X + r * nvec;
        __half2 lo2 = __float2half2_rn(0.f), hi2 = __float2half2_rn(0.f);
        for (int vi = lane; vi < nvec; vi += 32) {
            uint4 v = __ldg(xr + vi);
            const uint32_t kb = (s_abm[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
            if (kb)
                mask_known(v, kb);
            const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lo2 = __hmin2(lo2, h[i]);
                hi2 = __hmax2(hi2, h[i]);
            }
        }
        float lo = fminf(__low2float(lo2), __high2float(lo2));
        float hi = fmaxf(__low2float(hi2), __high2float(hi2));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const float range = __fsub_rn(hi, lo);
        const float sc = range > 0.f ? __fdiv_rn(255.0f, range) : 0.f;
        const int z = __float2int_rn(__fmul_rn(-lo, sc));
        int8_t *cr = codes + r * (int64_t)cols;
        for (int vi = lane; vi < nvec; vi += 32) {
            const uint4 v = __ldg(xr + vi);
            const uint32_t kb = (s_abm[vi >> 2] >> ((vi & 3) * 8)) & 0xFFu;
            const __half *h = reinterpret_cast<const __half *>(&v);
            uint32_t b[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                int q = z;
                if (!((kb >> e) & 1u))
                    q = __float2int_rn(__fmul_rn(__half2float(h[e]), sc)) + z;
                q = min(max(q, 0), 255);
                b[e] = (uint32_t)(q - 128) & 0xFFu;
            }
            *reinterpret_cast<uint2 *>(cr + (int64_t)vi * 8) =
                make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                           b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
        }
        if (lane == 0) {
            scale[r] = sc;
            zero[r] = z;
        }
    }
}

// R[j] = sum over K of the int8 codes of row j (one warp per row, four codes
// per __dp4a).
__global__ void __launch_bounds__(256) k_code_row_sums(const uint4 *__restrict__ CB, int64_t N, int K,
                                                       int32_t *__restrict__ R)
{
    const int lane = threadIdx.x & 31;
    const int nv = K >> 4;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t j = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < N; j += nwarps) {
        const uint4 *row = CB + j * nv;
        int acc = 0;
        for (int vi = lane; vi < nv; vi += 32) {
            const uint4 v = __ldg(row + vi);
            acc = __dp4a((int)v.x, 0x01010101, acc);
            acc = __dp4a((int)v.y, 0x01010101, acc);
            acc = __dp4a((int)v.z, 0x01010101, acc);
            acc = __dp4a((int)v.w, 0x01010101, acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0)
            R[j] = acc;
    }
}

} // namespace

cudaError_t launch_quantize_asym(const void *X, int64_t rows, int64_t cols, const uint32_t *bitmap, int8_t *codes,
                                 float *scale, int32_t *zero, const DeviceInfo &dev, cudaStream_t stream)
{
    if (rows <= 0)
        return cudaSuccess;
    const size_t smem = (size_t)((cols + 31) / 32) * 4;
    const int64_t want = (rows + 7) / 8;
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)dev.num_sms * 8);
    k_quant_asym<<<grid, 256, smem, stream>>>(reinterpret_cast<const uint4 *>(X), rows, (int)cols, bitmap, codes,
                                              scale, zero);
    return cudaGetLastError();
}

cudaError_t launch_code_row_sums(const int8_t *CB, int64_t N, int64_t K, int32_t *R, const DeviceInfo &dev,
                                 cudaStream_t stream)
{
    if (N <= 0)
        return cudaSuccess;
    const int64_t want = (N + 7) / 8;
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)dev.num_sms * 8);
    k_code_row_sums<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4 *>(CB), N, (int)K, R);
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
