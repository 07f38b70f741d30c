// The LLM.int8() linear for a few tokens (decode), fused into one kernel.
//
// Method (page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
// accelerate"): hidden-state columns holding any |x| >= threshold stay in fp16
// (sections "LLM.int8() 的简要总结" and "MatMul 内部"), the other columns are
// absmax-quantized per token row with scale 127 / absmax (section
// "模型量化简介"), multiplied in int8 against the per-row quantized weight and
// dequantized by the outer product of the two absmax vectors; the fp16
// outlier product is added.
//
// With at most 32 tokens the layer is a stream of the int8 weight (N x K
// bytes) past a tiny activation, so the kernel is built around that stream:
//   - every CTA (one per SM, cooperative launch) owns an equal share of the
//     (128-row weight tile, 128-byte K slice) units, so all SMs pull weight
//     bytes at once;
//   - its four helper warps first read one slice of columns of X across all
//     tokens (before the weight flood starts: behind it these few reads
//     would wait for it), so each CTA knows exactly which of its columns are
//     outliers; per-row partial maxima meet after a grid barrier, the codes
//     of each slice are written and a second grid barrier makes them
//     visible; meanwhile the TMA producer fills its ring with weight tiles;
//   - the MMA then runs with both operands TMA-loaded per unit; the weight
//     is read with an evict-first L2 policy (it is used once), so X, the
//     partial buffers and this kernel's own instructions stay in L2;
//   - a tile whose K range is split between CTAs is summed exactly in int32:
//     every CTA processes its segments from the last to the first, so the
//     head of a tile (the end of one CTA's range) is done early and parked
//     with a flag tagged with this call's barrier generation; the CTA that
//     holds the tile's tail finishes it at the end of its stream.
// The MMA is the swapped form: the weight tile is the M = 128 side, tokens
// the N = 16 or 32 side. The code that runs once per launch (scales, codes,
// epilogue) is written as short loops over the M real tokens rather than
// unrolled over BN: it runs from a cold instruction cache on every launch,
// and on B200 its instruction fetches, not its arithmetic, set its time.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>

#include "internal.h"
#include "llmint8.h"
#include "common.cuh"
#include "ptx.cuh"

namespace llmint8 {

namespace {

constexpr int TM = 128;       // weight rows per tile (MMA M)
constexpr int SK = 128;       // K bytes per slice (one 128-byte swizzle row, one TMA box)
constexpr int UK = 32;        // K per tcgen05.mma kind::i8
constexpr int OC = 32;        // outlier columns staged per chunk in the epilogue
constexpr int NTHREADS = 192; // warp 0 producer, warp 1 MMA, warps 2..5 quantizer + epilogue
constexpr int NHELP = 128;    // threads of warps 2..5
constexpr int kMaxVecPerCta = 128; // 8-column vectors of X per CTA (K <= 133143 needs at most 113)
constexpr int kL2Ahead = 8;        // weight units per CTA prefetched into L2 beyond the ring
constexpr float kInv127Sq = 1.0f / 16129.0f;

struct DParams {
    const uint4 *X;          // [M x K] fp16, as 16-byte vectors
    int M, N, K;
    int num_tiles, num_kb;   // 128-row weight tiles, K units of KS slices
    int num_slices;          // 128-byte K slices
    int64_t units;           // num_tiles * num_kb
    float t;
    __half t16;              // smallest fp16 >= t (+inf when there is no threshold)
    const int8_t *CB;
    const float *sb;
    const __half *W16;
    const __half *bias;      // fp16 [N] or null
    int act;                 // LLMINT8_ACT_*
    __half *Y;
    int32_t *acc_out;        // [M x N] int32 products, or null
    uint8_t *hitmask;        // [K/8] outlier mask per 8 columns
    float *prow;             // [32 x kDecodeMaxCtas] partial row maxima, one row per token
    int8_t *cx;              // [M x K] codes (each CTA writes its column slice)
    float *sx;               // [M] row absmax
    int32_t *col_idx;        // ascending outlier columns, written by CTA 0
    int32_t *count;
    uint32_t *sync;          // grid-barrier counter, generation, outlier-list flag
    int32_t *slots;          // [gridDim.x x 32 x 128] partial accumulators, token-major
    uint32_t *pflags;        // [gridDim.x] partial ready: set to the call's barrier generation
    uint32_t *status;
};

template <int BN, int STAGES, int KS>
struct DSmem {
    static constexpr int W_SUB = TM * SK;
    static constexpr int X_SUB = BN * SK;
    static constexpr int W_BYTES = KS * W_SUB;
    static constexpr int X_BYTES = KS * X_SUB;
    static constexpr int W_OFF = 0;
    static constexpr int X_OFF = W_OFF + STAGES * W_BYTES;
    static constexpr int SIDE_OFF = X_OFF + STAGES * X_BYTES;        // float [OC][BN]
    static constexpr int SCALE_OFF = SIDE_OFF + OC * BN * 4;         // float [32]: token absmax
    static constexpr int MULT_OFF = SCALE_OFF + 32 * 4;              // float [32]: 127 / absmax
    static constexpr int RMAX_OFF = MULT_OFF + 32 * 4;               // uint32 [32]: CTA row maxima
    static constexpr int HIT_OFF = RMAX_OFF + 32 * 4;                // uint32 [kMaxVecPerCta / 4]
    static constexpr int CPFX_OFF = HIT_OFF + kMaxVecPerCta;         // int [NHELP / 32]: compaction
    static constexpr int COLS_OFF = CPFX_OFF + 64;                   // int [OC]: first outlier columns
    static constexpr int ACC_OFF = COLS_OFF + OC * 4;                // int32 [TM][BN + 1]: accumulator rows
    static constexpr int WV_OFF = ACC_OFF + TM * (BN + 1) * 4;       // float [OC][TM]: outlier weights
    static constexpr int BAR_OFF = WV_OFF + OC * TM * 4;             // uint64 barriers
    static constexpr int NBARS = 2 * STAGES + 7;                     // full, empty, tfull[2], tempty[2], drain, xloaded, ready
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;             // tmem base, abort, last, grid flag, generation, outlier count
    static constexpr int BYTES = MISC_OFF + 32;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * BN <= 32 ? 32 : 64;
    static_assert(ALLOC <= 232448, "shared memory over the 227 KB per-CTA limit");
    static_assert(W_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "swizzle atoms need 1024-byte alignment");
    // The accumulator rows and outlier weights double as the scratch of the
    // outlier-mask compaction (K / 8 bytes, at most kMaxVecPerCta per CTA).
    static_assert(WV_OFF + OC * TM * 4 - ACC_OFF >= kMaxVecPerCta * kDecodeMaxCtas + 16 && ACC_OFF % 16 == 0,
                  "mask scratch");
};

__device__ __forceinline__ void report(const DParams &p, volatile int *s_abort, uint32_t bit)
{
    atomicOr(p.status, bit);
    *s_abort = 1;
}

// W's outlier column value: the fp16 weight if given, else CB * SCB / 127 per
// output row (page section "用法", Usage), in fp32.
__device__ __forceinline__ float wtilde(const DParams &p, int j, int c)
{
    if (p.W16)
        return __half2float(p.W16[(int64_t)j * p.K + c]);
    return __fdiv_rn(__fmul_rn((float)p.CB[(int64_t)j * p.K + c], p.sb[j]), 127.0f);
}

// First unit of CTA c when `units` units are split over G CTAs.
__device__ __forceinline__ int64_t unit_begin(int64_t c, int64_t units, int64_t G) { return c * units / G; }

// The CTA whose unit range holds unit u.
__device__ __forceinline__ int owner_of(int64_t u, int64_t units, int64_t G)
{
    int64_t c = u * G / units;
    while (c + 1 < G && unit_begin(c + 1, units, G) <= u)
        ++c;
    while (c > 0 && unit_begin(c, units, G) > u)
        --c;
    return (int)c;
}

// The i-th unit a CTA with units [u0, u1) processes: its segments (maximal
// runs of units in one tile) from the last to the first, the units of each
// in ascending order. The last segment of a range is a tile's head, whose
// tile is finished by another CTA; processing it first lets that partial be
// parked early.
__device__ __forceinline__ int64_t unit_order(int64_t u0, int64_t u1, int KB, int64_t i)
{
    int64_t se = u1;
    for (;;) {
        const int64_t ts = ((se - 1) / KB) * KB;
        const int64_t su = ts > u0 ? ts : u0;
        if (i < se - su)
            return su + i;
        i -= se - su;
        se = su;
    }
}

// Ascending list of the outlier columns from the per-8-column masks
// hitmask[0 .. nvec), by the NHELP helper threads of one CTA: the first `cap`
// columns into s_cols and their number into *s_count; with g_idx non-null
// the whole list and its length also into g_idx / *g_count. The masks are
// read once into s_scratch with 16-byte loads, all in flight together (each
// dependent global round trip costs microseconds behind the weight stream);
// the workspace region of the masks is padded to 256 bytes, and the bytes
// at or past nvec are never counted.
__device__ void compact_masks(const uint8_t *hitmask, int nvec, uint8_t *s_scratch, int *s_cols, int32_t *s_count,
                              int cap, int32_t *g_idx, int32_t *g_count, int et, int *s_pfx)
{
    const int nq = (nvec + 15) >> 4;
    for (int q0 = et; q0 < nq; q0 += 4 * NHELP) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (q0 + u * NHELP < nq)
                v[u] = __ldcg(reinterpret_cast<const uint4 *>(hitmask) + q0 + u * NHELP);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (q0 + u * NHELP < nq)
                reinterpret_cast<uint4 *>(s_scratch)[q0 + u * NHELP] = v[u];
    }
    named_barrier_sync(1, NHELP);
    const int lane = et & 31, w = et >> 5;
    const int per = (nvec + NHELP - 1) / NHELP;
    const int b0 = min(et * per, nvec), b1 = min(b0 + per, nvec);
    int cnt = 0;
    for (int b = b0; b < b1; ++b)
        cnt += __popc((uint32_t)s_scratch[b]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        s_pfx[w] = incl;
    named_barrier_sync(1, NHELP);
    int base = 0;
    for (int i = 0; i < w; ++i)
        base += s_pfx[i];
    if (et == NHELP - 1) {
        *s_count = base + incl;
        if (g_idx)
            *g_count = base + incl;
    }
    int pos = base + incl - cnt;
    for (int b = b0; b < b1; ++b) {
        uint32_t bits = s_scratch[b];
        while (bits) {
            const int e = __ffs(bits) - 1;
            if (pos < cap)
                s_cols[pos] = b * 8 + e;
            if (g_idx)
                g_idx[pos] = b * 8 + e;
            ++pos;
            bits &= bits - 1u;
        }
    }
    if (g_idx)
        __threadfence();
    named_barrier_sync(1, NHELP);
}


// Outlier columns of one 16-byte vector of X (slice vector v) into s_hit.
__device__ __forceinline__ void mark_outliers(const DParams &p, const uint4 &x, int v, uint32_t *s_hit)
{
    const uint32_t h = hit_mask8(x, p.t16);
    if (h)
        atomicOr(&s_hit[v >> 2], h << ((v & 3) * 8));
}

// Maximum |x| of one 16-byte vector of row r over its non-outlier columns
// into s_rmax[r].
__device__ __forceinline__ void row_max_into(uint4 x, int r, int v, const uint32_t *s_hit, uint32_t *s_rmax)
{
    const uint32_t kb = (s_hit[v >> 2] >> ((v & 3) * 8)) & 0xFFu;
    if (kb)
        mask_known(x, kb);
    __half2 a[4];
    const __half2 m2 = vec_abs_max(x, a);
    const float m = fmaxf(__low2float(m2), __high2float(m2));
    if (m > 0.f)
        atomicMax(&s_rmax[r], __float_as_uint(m)); // non-negative floats order like their bits
}

// Codes of one 16-byte vector of row r (global vector index gv, slice
// vector v) into p.cx, outlier columns zeroed.
__device__ __forceinline__ void store_codes(const DParams &p, uint4 x, int r, int gv, int v, const uint32_t *s_hit,
                                            const float *s_mult)
{
    const uint32_t kb = (s_hit[v >> 2] >> ((v & 3) * 8)) & 0xFFu;
    if (kb)
        mask_known(x, kb);
    *reinterpret_cast<uint2 *>(p.cx + (int64_t)r * p.K + (int64_t)gv * 8) = codes8(x, s_mult[r]);
}

// Row scales and codes of the M token rows, by the helper warps of every
// CTA. CTA c holds the 8-column vectors [v0, v1) of all rows, so the outlier
// test of its columns is complete without the other CTAs:
//   1. mark the slice's outlier columns; maximum |x| per row over the
//      slice's other columns; publish the mask bytes and one partial maximum
//      per row;
//   grid barrier (it also yields *gen), then arrive on `xloaded_bar` (the
//   weight stream may start);
//   2. absmax per row = maximum of the partial maxima (s_amax) and the
//      multiplier 127 / absmax; the slice's codes go to p.cx; CTA 0 writes SX;
//   grid barrier (codes complete before any CTA's TMA reads them).
// Each thread keeps its first PC vectors of X in registers; the rest is read
// again (from L2). Returns false if a grid barrier gave up.
template <bool THR>
__device__ bool row_scales(const DParams &p, int et, uint32_t xloaded_bar, uint32_t *s_hit, uint32_t *s_rmax,
                           float *s_amax, float *s_mult, int *s_pfx, volatile int *s_flag, volatile uint32_t *s_gen,
                           uint32_t *gen)
{
    const int G = gridDim.x, c = blockIdx.x;
    const int nvec = p.K >> 3;
    const int v0 = (int)((int64_t)c * nvec / G), v1 = (int)((int64_t)(c + 1) * nvec / G);
    const int nv = v1 - v0;
    const int npairs = p.M * nv;
    for (int i = et; i < kMaxVecPerCta / 4; i += NHELP)
        s_hit[i] = 0u;
    if (et < 32)
        s_rmax[et] = 0u;
    // This CTA's partial-ready flag and (CTA 0) the outlier-list flag are read
    // only after the second grid barrier: clearing them here, before the
    // first one, keeps whatever an earlier call (or other data) left there
    // from ever matching this call's generation.
    if (et == 0) {
        p.pflags[c] = 0u;
        if (c == 0)
            p.sync[3] = 0u;
    }
    named_barrier_sync(1, NHELP);
    // The first PC vectors of each thread stay in registers for the maxima.
    constexpr int PC = 4;
    uint4 xs[PC];
#pragma unroll
    for (int k = 0; k < PC; ++k) {
        const int i = et + k * NHELP;
        xs[k] = make_uint4(0u, 0u, 0u, 0u);
        if (i < npairs) {
            const int r = i / nv, v = i - r * nv;
            xs[k] = __ldg(p.X + (int64_t)r * nvec + v0 + v);
        }
    }
    if constexpr (THR) {
#pragma unroll
        for (int k = 0; k < PC; ++k)
            if (et + k * NHELP < npairs)
                mark_outliers(p, xs[k], (et + k * NHELP) % nv, s_hit);
        for (int i = et + PC * NHELP; i < npairs; i += NHELP)
            mark_outliers(p, __ldg(p.X + (int64_t)(i / nv) * nvec + v0 + i % nv), i % nv, s_hit);
    }
    named_barrier_sync(1, NHELP);
#pragma unroll
    for (int k = 0; k < PC; ++k)
        if (et + k * NHELP < npairs)
            row_max_into(xs[k], (et + k * NHELP) / nv, (et + k * NHELP) % nv, s_hit, s_rmax);
    for (int i = et + PC * NHELP; i < npairs; i += NHELP)
        row_max_into(__ldg(p.X + (int64_t)(i / nv) * nvec + v0 + i % nv), i / nv, i % nv, s_hit, s_rmax);
    named_barrier_sync(1, NHELP);
    if (et < 32) {
        p.prow[(int64_t)et * kDecodeMaxCtas + c] = __uint_as_float(s_rmax[et]);
        s_rmax[et] = 0u; // reused for the final maxima
    }
    for (int v = et; v < nv; v += NHELP)
        p.hitmask[v0 + v] = (uint8_t)((s_hit[v >> 2] >> ((v & 3) * 8)) & 0xFFu);
    named_barrier_sync(1, NHELP);
    if (et == 0) {
        uint32_t g = 0;
        *s_flag = grid_barrier(p.sync, (uint32_t)G, &g) ? 1 : 0;
        *s_gen = g;
    }
    named_barrier_sync(1, NHELP);
    if (!*s_flag)
        return false;
    *gen = *s_gen;
    // The weight stream may start now: the first step's global round trips
    // are done (behind the stream each of them would wait for it).
    if (et == 0)
        mbar_arrive(xloaded_bar);

    // Row maxima over the G partial maxima (16-byte loads; entries of CTAs
    // >= G are left over from other calls and skipped).
    const int nq = (G + 3) >> 2;
    for (int i = et; i < p.M * nq; i += NHELP) {
        const int r = i / nq, q = i - r * nq;
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.prow + (int64_t)r * kDecodeMaxCtas) + q);
        float m = v.x;
        if (4 * q + 1 < G)
            m = fmaxf(m, v.y);
        if (4 * q + 2 < G)
            m = fmaxf(m, v.z);
        if (4 * q + 3 < G)
            m = fmaxf(m, v.w);
        if (m > 0.f)
            atomicMax(&s_rmax[r], __float_as_uint(m));
    }
    named_barrier_sync(1, NHELP);
    if (et < 32) {
        const float amax = et < p.M ? __uint_as_float(s_rmax[et]) : 0.f;
        s_amax[et] = amax;
        s_mult[et] = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        if (c == 0 && et < p.M)
            p.sx[et] = amax;
    }
    named_barrier_sync(1, NHELP);
#pragma unroll
    for (int k = 0; k < PC; ++k)
        if (et + k * NHELP < npairs)
            store_codes(p, xs[k], (et + k * NHELP) / nv, v0 + (et + k * NHELP) % nv, (et + k * NHELP) % nv, s_hit,
                        s_mult);
    for (int i = et + PC * NHELP; i < npairs; i += NHELP)
        store_codes(p, __ldg(p.X + (int64_t)(i / nv) * nvec + v0 + i % nv), i / nv, v0 + i % nv, i % nv, s_hit,
                    s_mult);
    // The codes are read next by TMA (the async proxy) in every CTA; the
    // barrier's release and acquire carry them across CTAs.
    asm volatile("fence.proxy.async.global;" ::: "memory");
    named_barrier_sync(1, NHELP);
    if (et == 0)
        *s_flag = grid_barrier(p.sync, (uint32_t)G) ? 1 : 0;
    named_barrier_sync(1, NHELP);
    return *s_flag != 0;
}

// Outlier weights W~[j, cols[k]] of this thread's weight row j for k < nk
// into s_wv[k][r], eight loads in flight at a time.
__device__ __forceinline__ void load_wv(const DParams &p, int j, int r, const int *cols, int nk, float *s_wv)
{
    for (int k0 = 0; k0 < nk; k0 += 8) {
        float w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            w[u] = (k0 + u < nk && j < p.N) ? wtilde(p, j, cols[k0 + u]) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (k0 + u < nk)
                s_wv[(k0 + u) * TM + r] = w[u];
    }
}

// y[0..8) += W~[j, col k] * X[c0 + u, col k] over the staged outlier columns
// k < nk, k ascending: s_wv points at this row's first weight, side at token
// c0 of column 0. One weight load and two broadcast loads of X per column
// feed eight independent FMA chains (one chain per token would wait on the
// shared-memory latency at every column); each token's sum keeps the column
// order.
template <int BN>
__device__ __forceinline__ void outlier_fma8(float (&y)[8], const float *s_wv, const float *side, int nk)
{
#pragma unroll 2
    for (int k = 0; k < nk; ++k) {
        const float w = s_wv[k * TM];
        const float4 a = *reinterpret_cast<const float4 *>(side + k * BN);
        const float4 b = *reinterpret_cast<const float4 *>(side + k * BN + 4);
        y[0] = fmaf(w, a.x, y[0]);
        y[1] = fmaf(w, a.y, y[1]);
        y[2] = fmaf(w, a.z, y[2]);
        y[3] = fmaf(w, a.w, y[3]);
        y[4] = fmaf(w, b.x, y[4]);
        y[5] = fmaf(w, b.y, y[5]);
        y[6] = fmaf(w, b.z, y[6]);
        y[7] = fmaf(w, b.w, y[7]);
    }
}

// Dequantize this thread's accumulator row acc[0..M) (weight row j), add the
// outlier product and store Y (and the raw products when asked). All NHELP
// helper threads call it together: with more than OC outlier columns the
// columns are staged in chunks behind named barriers. The row's outputs are
// kept in place of the accumulators (fp32) until the final stores.
template <int BN>
__device__ void finalize_row(const DParams &p, int j, int r, int32_t *acc, const float *s_amax, float *s_side,
                             int *s_cols, float *s_wv, int cnt, int et)
{
    static_assert(BN % 8 == 0, "tokens are processed in groups of eight");
    const int M = p.M;
    if (p.acc_out && j < p.N)
        for (int c = 0; c < M; ++c)
            p.acc_out[(int64_t)c * p.N + j] = acc[c];
    const float sbj = j < p.N ? p.sb[j] : 0.f;
    const float bj = (p.bias && j < p.N) ? __half2float(p.bias[j]) : 0.f;
    float *yr = reinterpret_cast<float *>(acc); // in place: one float per token
    // With at most OC outlier columns s_side holds X at all of them for every
    // token (staged once per CTA) and s_wv this row's outlier weights (loaded
    // before the accumulator).
    const int nk0 = cnt <= OC ? cnt : 0;
    for (int c0 = 0; c0 < M; c0 += 8) {
        float y[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            y[u] = c0 + u < M ? (float)acc[c0 + u] * (sbj * s_amax[c0 + u]) * kInv127Sq : 0.f;
        outlier_fma8<BN>(y, s_wv + r, s_side + c0, nk0);
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (c0 + u < M)
                yr[c0 + u] = y[u];
    }
    for (int ch = 0; cnt > OC && ch < cnt; ch += OC) {
        const int nk = min(OC, cnt - ch);
        named_barrier_sync(1, NHELP);
        if (et < nk)
            s_cols[et] = __ldcg(p.col_idx + ch + et);
        named_barrier_sync(1, NHELP);
        for (int idx = et; idx < nk * BN; idx += NHELP) {
            const int k = idx / BN, c = idx - k * BN;
            s_side[idx] = c < M ? __half2float(reinterpret_cast<const __half *>(p.X)[(int64_t)c * p.K + s_cols[k]])
                                : 0.f;
        }
        load_wv(p, j, r, s_cols, nk, s_wv);
        named_barrier_sync(1, NHELP);
        for (int c0 = 0; c0 < M; c0 += 8) {
            float y[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                y[u] = c0 + u < M ? yr[c0 + u] : 0.f;
            outlier_fma8<BN>(y, s_wv + r, s_side + c0, nk);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (c0 + u < M)
                    yr[c0 + u] = y[u];
        }
    }
    if (j < p.N)
        for (int c = 0; c < M; ++c)
            p.Y[(int64_t)c * p.N + j] = __float2half_rn(bias_act(yr[c], bj, p.act));
}

// Epilogue of one segment [su, se) of tile t = su / num_kb, held in TMEM
// accumulator buffer seg & 1. A whole tile is finished here. A split tile is
// finished by the CTA holding its last unit, c_hi: the tile is that CTA's
// first segment, which it processes last, and before its own accumulator is
// complete it reads the partials that the tile's other CTAs parked (after
// their ready flags). For each other CTA the tile is its last segment, which
// it processes first and parks in its slot before raising its flag to
// `gen`. All NHELP helper threads call it together; returns false on a
// timeout (nothing written).
template <int BN>
__device__ bool epilogue_segment(const DParams &p, int et, int warp, int lane, int64_t u0, int64_t u1, int64_t su,
                                 int64_t se,
                                 int seg, uint32_t tmem_base, uint32_t tfull_b, uint32_t tempty_b, uint32_t &tph_b,
                                 const float *s_amax, float *s_side, int *s_cols, int32_t *s_acc, float *s_wv,
                                 int cnt, bool wv_loaded, uint32_t gen, volatile int *s_abort, volatile int *s_last)
{
    const int64_t G = gridDim.x, cta = blockIdx.x;
    const int KB = p.num_kb, M = p.M;
    const int t = (int)(su / KB);
    const int64_t tile_u0 = (int64_t)t * KB;
    const bool whole = su == tile_u0 && se == tile_u0 + KB;
    const int c_lo = whole ? (int)cta : owner_of(tile_u0, p.units, G);
    const int c_hi = whole ? (int)cta : owner_of(tile_u0 + KB - 1, p.units, G);
    const bool finisher = cta == c_hi;
    (void)u0;
    (void)u1;
    const int q = warp & 3;      // TMEM lane quarter this warp may read
    const int r = q * 32 + lane; // weight row within the tile
    const int j = t * TM + r;
    int32_t *acc = s_acc + r * (BN + 1);
    if (finisher) {
        // Everything that does not need this CTA's accumulator first, while
        // its last MMAs run: this row's outlier weights and the partial sums
        // the tile's other CTAs parked (normally long ready).
        if (cnt <= OC && !wv_loaded)
            load_wv(p, j, r, s_cols, cnt, s_wv);
        for (int c = 0; c < M; ++c)
            acc[c] = 0;
        if (c_hi > c_lo) {
            if (et == 0) {
                bool all = true;
                const uint64_t t0 = global_timer_ns();
                for (int cc = c_lo; cc < c_hi; ++cc) {
                    uint32_t f;
                    for (;;) {
                        asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(f) : "l"(p.pflags + cc) : "memory");
                        if (f == gen || global_timer_ns() - t0 > kWaitLimitNs)
                            break;
                        __nanosleep(64);
                    }
                    all = all && f == gen;
                }
                *s_last = all ? 1 : 0;
            }
            named_barrier_sync(1, NHELP);
            if (!*s_last) {
                if (et == 0)
                    report(p, s_abort, LLMINT8_DEV_TIMEOUT_EPILOGUE);
                return false;
            }
            for (int cc = c_lo; cc < c_hi; ++cc) {
                const int32_t *src = p.slots + ((int64_t)cc * kDecodeMaxM) * TM + r;
                int32_t v[BN];
#pragma unroll
                for (int c = 0; c < BN; ++c) // every load in flight at once
                    v[c] = c < M ? __ldcg(src + c * TM) : 0;
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c < M)
                        acc[c] += v[c];
            }
        }
    }
    const bool got = mbar_wait(tfull_b, tph_b);
    if (named_barrier_or(1, NHELP, !got)) {
        if (!got)
            report(p, s_abort, LLMINT8_DEV_TIMEOUT_EPILOGUE);
        return false;
    }
    tph_b ^= 1u;
    tc_fence_after();
    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)((seg & 1) * BN);
    uint32_t raw[BN];
    if constexpr (BN == 32)
        tmem_ld_32x32b_x32(taddr, raw);
    else
        tmem_ld_32x32b_x16(taddr, raw);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
        mbar_arrive(tempty_b); // the accumulator is in registers now
    if (!finisher) {
        // This tile is this CTA's last segment (processed first): park it
        // for the finisher.
        int32_t *dst = p.slots + (cta * kDecodeMaxM) * TM + r;
#pragma unroll
        for (int c = 0; c < BN; ++c)
            if (c < M)
                dst[c * TM] = (int32_t)raw[c];
        named_barrier_sync(1, NHELP); // the release below covers the CTA's stores
        if (et == 0)
            asm volatile("st.release.gpu.u32 [%0], %1;" ::"l"(p.pflags + cta), "r"(gen) : "memory");
        return true;
    }
#pragma unroll
    for (int c = 0; c < BN; ++c)
        if (c < M)
            acc[c] += (int32_t)raw[c];
    finalize_row<BN>(p, j, r, acc, s_amax, s_side, s_cols, s_wv, cnt, et);
    return true;
}

template <int BN, int STAGES, int KS, bool THR>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_decode(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const DParams p)
{
    using L = DSmem<BN, STAGES, KS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *s_side = reinterpret_cast<float *>(smem + L::SIDE_OFF);
    float *s_amax = reinterpret_cast<float *>(smem + L::SCALE_OFF);
    float *s_mult = reinterpret_cast<float *>(smem + L::MULT_OFF);
    uint32_t *s_rmax = reinterpret_cast<uint32_t *>(smem + L::RMAX_OFF);
    uint32_t *s_hit = reinterpret_cast<uint32_t *>(smem + L::HIT_OFF);
    int *s_pfx = reinterpret_cast<int *>(smem + L::CPFX_OFF);
    int *s_cols = reinterpret_cast<int *>(smem + L::COLS_OFF);
    int32_t *s_acc = reinterpret_cast<int32_t *>(smem + L::ACC_OFF);
    float *s_wv = reinterpret_cast<float *>(smem + L::WV_OFF);
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    const uint32_t xloaded_bar = bar0 + 8u * (2 * STAGES + 5);
    const uint32_t ready_bar = bar0 + 8u * (2 * STAGES + 6);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);
    volatile int *s_last = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 8);
    volatile int *s_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 12);
    volatile uint32_t *s_gen = reinterpret_cast<volatile uint32_t *>(smem + L::MISC_OFF + 16);
    int32_t *s_cnt = reinterpret_cast<int32_t *>(smem + L::MISC_OFF + 20);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4); // one arrival per helper warp
        }
        mbar_init(drain_bar, 1);
        mbar_init(xloaded_bar, 1); // X's reads of this CTA are back
        mbar_init(ready_bar, 1);   // the codes of X are complete in every CTA
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(s_tmem), L::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    // Launched as a programmatic dependent: the set-up above overlapped the
    // previous kernel's tail; nothing below reads or writes global memory
    // before that kernel is complete.
    griddep_wait();
    const int64_t G = gridDim.x, cta = blockIdx.x;
    const int64_t u0 = unit_begin(cta, p.units, G), u1 = unit_begin(cta + 1, p.units, G);
    const int64_t n = u1 - u0;
    const int KB = p.num_kb;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_phase = 0;
            // Slices in unit kb (the last unit along K may hold fewer) and
            // the bytes they bring.
            auto slices = [&](int kb) { return min(KS, p.num_slices - kb * KS); };
            auto tx = [&](int ns) { return (uint32_t)ns * (uint32_t)(L::W_SUB + L::X_SUB); };
            const int pre = (int)(n < STAGES ? n : STAGES);
            const uint64_t evict_first = l2_evict_first_policy(); // the weight is read once
            // X's few reads first (behind the weight flood they would wait for
            // it), then fill the ring with weight tiles while X is quantized.
            // Only the ring's first units go to L2 at once: HBM is otherwise
            // idle until then, and this little does not hold up those reads
            // (measured on B200: these 4 units gain 0.5-1 us at M = 1, 8 and
            // 32; the ring plus 8 more, 12 units, cost 2 us at M = 32).
            for (int s = 0; s < pre; ++s) {
                const int64_t u = unit_order(u0, u1, KB, s);
                const int t = (int)(u / KB), kb = (int)(u - (int64_t)t * KB);
                for (int j = 0; j < slices(kb); ++j)
                    tma_prefetch_l2_2d(&tmW, (kb * KS + j) * SK, t * TM);
            }
            if (!mbar_wait(xloaded_bar, 0u))
                report(p, s_abort, LLMINT8_DEV_TIMEOUT_PRODUCER);
            for (int s = 0; s < pre; ++s) {
                const int64_t u = unit_order(u0, u1, KB, s);
                const int t = (int)(u / KB), kb = (int)(u - (int64_t)t * KB);
                const int ns = slices(kb);
                mbar_arrive_expect_tx(full_bar(s), tx(ns));
                for (int j = 0; j < ns; ++j)
                    tma_load_2d_hint(sbase + L::W_OFF + s * L::W_BYTES + j * L::W_SUB, &tmW, full_bar(s),
                                     (kb * KS + j) * SK, t * TM, evict_first);
                armed |= 1u << s; // phase 0
            }
            // The next units into L2, so that HBM stays busy until the codes
            // are ready and the ring turns over.
            for (int64_t i = pre; i < n && i < pre + kL2Ahead; ++i) {
                const int64_t u = unit_order(u0, u1, KB, i);
                const int t = (int)(u / KB), kb = (int)(u - (int64_t)t * KB);
                for (int j = 0; j < slices(kb); ++j)
                    tma_prefetch_l2_2d(&tmW, (kb * KS + j) * SK, t * TM);
            }
            if (!mbar_wait(ready_bar, 0u))
                report(p, s_abort, LLMINT8_DEV_TIMEOUT_PRODUCER);
            asm volatile("fence.proxy.async.global;" ::: "memory"); // codes written by other CTAs
            for (int64_t i = 0; i < n; ++i) {
                const int64_t u = unit_order(u0, u1, KB, i);
                const int t = (int)(u / KB), kb = (int)(u - (int64_t)t * KB);
                const int ns = slices(kb);
                if (i < pre) {
                    // The stage's weight bytes are in flight; add the codes
                    // (also after a failure, so that every armed stage completes).
                    for (int j = 0; j < ns; ++j)
                        tma_load_2d(sbase + L::X_OFF + stage * L::X_BYTES + j * L::X_SUB, &tmX, full_bar(stage),
                                    (kb * KS + j) * SK, 0);
                } else {
                    if (*s_abort)
                        break;
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u)) {
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_PRODUCER);
                        break;
                    }
                    if (*s_abort)
                        break;
                    mbar_arrive_expect_tx(full_bar(stage), tx(ns));
                    for (int j = 0; j < ns; ++j) {
                        tma_load_2d_hint(sbase + L::W_OFF + stage * L::W_BYTES + j * L::W_SUB, &tmW, full_bar(stage),
                                         (kb * KS + j) * SK, t * TM, evict_first);
                        tma_load_2d(sbase + L::X_OFF + stage * L::X_BYTES + j * L::X_SUB, &tmX, full_bar(stage),
                                    (kb * KS + j) * SK, 0);
                    }
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (*s_abort) {
                // Let every copy this thread started land before the CTA exits.
                for (int s = 0; s < STAGES; ++s)
                    if ((armed >> s) & 1u)
                        mbar_wait(full_bar(s), (armed_phase >> s) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t tph[2] = {0u, 0u};
            constexpr uint32_t IDESC = idesc_i8(TM, BN);
            int seg = 0;
            int64_t seg_end = u1; // segments from the last to the first
            while (seg_end > u0 && !*s_abort) {
                const int64_t u = max(u0, ((seg_end - 1) / KB) * KB);
                const int b = seg & 1;
                if (!mbar_wait(tempty_bar(b), tph[b] ^ 1u)) {
                    report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
                    break;
                }
                tph[b] ^= 1u;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                bool ok = true;
                for (int64_t v = u; v < seg_end; ++v) {
                    if (!mbar_wait_poll(full_bar(stage), phase)) {
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int ns = min(KS, p.num_slices - (int)(v % KB) * KS);
                    for (int j = 0; j < ns; ++j) {
                        const uint32_t a0 = sbase + L::W_OFF + stage * L::W_BYTES + j * L::W_SUB;
                        const uint32_t b0 = sbase + L::X_OFF + stage * L::X_BYTES + j * L::X_SUB;
#pragma unroll
                        for (int k = 0; k < SK / UK; ++k)
                            mma_i8(d_tmem, smem_desc_k128(a0 + k * UK), smem_desc_k128(b0 + k * UK), IDESC,
                                   (v != u || j != 0 || k != 0) ? 1u : 0u);
                    }
                    mma_commit(empty_bar(stage)); // stage free once these MMAs have read it
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                mma_commit(tfull_bar(b)); // this segment's product is complete
                seg_end = u;
                ++seg;
            }
            // Wait for every MMA this thread issued before TMEM is released.
            mma_commit(drain_bar);
            if (!mbar_wait(drain_bar, 0u))
                report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ helpers: scales and codes, then epilogue
        const int et = threadIdx.x - 64;
        uint32_t gen = 0;
        const bool ok =
            row_scales<THR>(p, et, xloaded_bar, s_hit, s_rmax, s_amax, s_mult, s_pfx, s_flag, s_gen, &gen);
        if (et == 0) {
            if (!ok)
                report(p, s_abort, LLMINT8_DEV_TIMEOUT_QUANT);
            mbar_arrive(ready_bar); // the producer may add the codes to its stages
        }
        int cnt = 0;
        bool go = ok;
        if (ok) {
            // This CTA's own copy of the first OC outlier columns and their
            // number, from the masks that every CTA published before the
            // first grid barrier (no wait on another CTA). CTA 0 also writes
            // the whole list and its length to the workspace and then sets
            // the list flag sync[3] to `gen`; only with more than OC columns
            // do the epilogues read that list.
            const bool publish = blockIdx.x == 0;
            if constexpr (THR) {
                compact_masks(p.hitmask, p.K >> 3, reinterpret_cast<uint8_t *>(s_acc), s_cols, s_cnt, OC,
                              publish ? p.col_idx : nullptr, p.count, et, s_pfx);
            } else if (et == 0) {
                *s_cnt = 0;
                if (publish)
                    *p.count = 0;
            }
            if (publish && et == 0) {
                __threadfence();
                asm volatile("st.release.gpu.u32 [%0], %1;" ::"l"(p.sync + 3), "r"(gen) : "memory");
            }
            named_barrier_sync(1, NHELP);
            cnt = *s_cnt;
            if (cnt > OC) {
                // More columns than one staging chunk: the epilogues read the
                // whole list, CTA 0's.
                if (et == 0) {
                    const uint64_t t0 = global_timer_ns();
                    uint32_t f;
                    for (;;) {
                        asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(f) : "l"(p.sync + 3) : "memory");
                        if (f == gen || global_timer_ns() - t0 > kWaitLimitNs)
                            break;
                        __nanosleep(200);
                    }
                    *s_flag = f == gen ? 1 : 0;
                    if (f != gen)
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_EPILOGUE);
                }
                named_barrier_sync(1, NHELP);
                go = *s_flag != 0;
            } else {
                // X at the outlier columns, for every tile of this CTA.
                for (int idx = et; idx < cnt * BN; idx += NHELP) {
                    const int k = idx / BN, c = idx - k * BN;
                    s_side[idx] =
                        c < p.M ? __half2float(reinterpret_cast<const __half *>(p.X)[(int64_t)c * p.K + s_cols[k]])
                                : 0.f;
                }
            }
            named_barrier_sync(1, NHELP);
        }
        if (go) {
            uint32_t tph[2] = {0u, 0u};
            int seg = 0;
            bool wv_loaded = false; // s_wv holds the outlier weights of the segment processed next
            for (int64_t seg_end = u1; seg_end > u0; ++seg) { // segments from the last to the first
                const int64_t su = max(u0, ((seg_end - 1) / KB) * KB);
                const int b = seg & 1;
                const bool wv_now = wv_loaded;
                wv_loaded = false;
                // Only the first segment processed can be a parked one (a tile
                // head); every segment after it ends at a tile end and is
                // finished here. Its outlier weights (a round trip to HBM) are
                // fetched before the parked segment's epilogue, off the path
                // that follows the last MMA.
                const int64_t tile_u0 = (su / KB) * KB;
                const bool parks = seg_end % KB != 0 && owner_of(tile_u0 + KB - 1, p.units, G) != (int)cta;
                if (parks && su > u0 && cnt <= OC) {
                    const int r = (warp & 3) * 32 + lane;
                    load_wv(p, (int)((su - 1) / KB) * TM + r, r, s_cols, cnt, s_wv);
                    wv_loaded = true;
                }
                if (!epilogue_segment<BN>(p, et, warp, lane, u0, u1, su, seg_end, seg, tmem_base, tfull_bar(b),
                                          tempty_bar(b), tph[b], s_amax, s_side, s_cols, s_acc, s_wv, cnt, wv_now,
                                          gen, s_abort, s_last))
                    break;
                seg_end = su;
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

// CTAs of the decode kernel: one per SM, at most one per unit.
int decode_grid(int64_t N, int64_t K, int ks, const DeviceInfo &dev)
{
    const int64_t units = ((N + TM - 1) / TM) * ((K + SK * ks - 1) / (SK * ks));
    return (int)std::min<int64_t>(std::min<int64_t>(dev.num_sms, kDecodeMaxCtas), units);
}

template <int BN, int STAGES, int KS, bool THR>
cudaError_t run_decode(const DecodeArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    using L = DSmem<BN, STAGES, KS>;
    auto kern = k_decode<BN, STAGES, KS, THR>;
    static std::atomic<uint64_t> configured{0};
    const uint64_t bit = 1ull << (dev.device & 63);
    if (!(configured.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
        if (e != cudaSuccess)
            return e;
        configured.fetch_or(bit);
    }
    CUtensorMap tw, tx;
    if (!make_map_i8(&tw, dev.device, a.CB, a.N, a.K, TM) || !make_map_i8(&tx, dev.device, a.ws.cx, a.M, a.K, BN))
        return cudaErrorInvalidValue;
    DParams p{};
    p.X = reinterpret_cast<const uint4 *>(a.X);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.num_tiles = (int)((a.N + TM - 1) / TM);
    p.num_slices = (int)((a.K + SK - 1) / SK);
    p.num_kb = (p.num_slices + KS - 1) / KS;
    p.units = (int64_t)p.num_tiles * p.num_kb;
    p.t = a.t;
    p.t16 = threshold_fp16(a.t);
    p.CB = a.CB;
    p.sb = a.sb;
    p.W16 = reinterpret_cast<const __half *>(a.W16);
    p.bias = reinterpret_cast<const __half *>(a.bias);
    p.act = a.act;
    p.Y = reinterpret_cast<__half *>(a.Y);
    p.acc_out = a.acc_out;
    p.hitmask = a.ws.hitmask;
    p.prow = a.ws.prow;
    p.cx = a.ws.cx;
    p.sx = a.ws.sx;
    p.col_idx = a.ws.col_idx;
    p.count = a.ws.count;
    p.sync = a.ws.sync;
    p.slots = a.ws.slots;
    p.pflags = a.ws.pflags;
    p.status = a.ws.status;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)decode_grid(a.N, a.K, KS, dev));
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = L::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative; // the grid barrier needs every CTA resident
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization; // launch overlaps the previous tail
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tw, tx, p);
}

} // namespace

bool decode_fused_fits(int64_t M, int64_t N, int64_t K, const DeviceInfo &dev)
{
    if (!decode_shape(M, N) || K < 16)
        return false;
    const int G = decode_grid(N, K, 2, dev);
    return G >= 1 && (K / 8 + G - 1) / G <= kMaxVecPerCta;
}

cudaError_t launch_decode(const DecodeArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    const bool thr = a.t > 0.f;
    // Units of two 128-byte slices: each TMA load pair then reads 256
    // contiguous bytes of every weight row, which the HBM serves much better
    // than 128 (measured on B200: 7.6 vs 5.4 TB/s for the stream alone).
    if (a.M <= 16)
        return thr ? run_decode<16, 4, 2, true>(a, dev, stream) : run_decode<16, 4, 2, false>(a, dev, stream);
    return thr ? run_decode<32, 4, 2, true>(a, dev, stream) : run_decode<32, 4, 2, false>(a, dev, stream);
}

} // namespace llmint8
