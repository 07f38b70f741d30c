// int8 x int8 -> int32 GEMM on the 5th-generation tensor cores (tcgen05,
// kind::i8) with the LLM.int8() epilogue fused in.
//
// The int8 product of the non-outlier part is the vector-wise quantized
// matmul of page "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与
// accelerate", section "模型量化简介" (Introduction to model quantization):
// rows of X and output rows of W are quantized separately and the int32
// result is dequantized by the outer product of their absmax vectors. The
// epilogue adds the fp16 outlier product of section "LLM.int8() 的简要总结"
// (step 2: outlier columns in fp16; step 3: dequantize and add).
//
// Structure (one CTA per SM, 192 threads, persistent over output tiles):
//   warp 0      TMA producer: 128x128-byte K-major int8 tiles of both
//               operands into a STAGES-deep shared-memory ring (128B swizzle).
//   warp 1      allocates TMEM; one thread issues tcgen05.mma kind::i8
//               (M=128, N=BN, K=32 per instruction) into one of two TMEM
//               int32 accumulators and commits stage releases / tile done.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, dequant
//               acc * SX[i] * SB[j] / 127^2, plus sum over outlier columns
//               c of X[i,c] * Wt[j,c] in fp32 FMAs, fp16 store. The outlier
//               operands for the next tile are staged while the tensor cores
//               run its main loop.
// SWAP=true is the decode form (few tokens): W takes the MMA M side (128
// output features per tile) and the tokens the N side (BN = 16 or 32).
// From 256 rows of X the CTA-pair form runs instead (k_gemm_i8_pair: 256-row
// tiles over two CTAs of a cluster, tcgen05.mma.cta_group::2); when its tiles
// do not fill the last round, the last tiles are split over the pairs by K
// stages (stream-K, work lists in sched.h) and the int32 parts summed exactly.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "llmint8.h"
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "sched.h"

namespace llmint8 {

namespace {

constexpr int BM = 128;       // MMA M: rows of the A operand per tile
constexpr int BK = 128;       // K bytes per pipeline stage (one 128-byte swizzle row)
static_assert(2 * BM == kPairRows && BK == kSliceBytes, "the pair plan's tile and slice sizes");
constexpr int UK = 32;        // K per tcgen05.mma kind::i8
constexpr int OC = 32;        // outlier columns staged per chunk in the epilogue
constexpr int kStoreStage = 16384; // bytes at the end of s_side for the TMA-store staging (4 warps x 4 KB)
static_assert(OC == kGatherCols, "the gathered staging fills s_side for up to OC columns");
constexpr int NTHREADS = 192; // 6 warps
constexpr float kInv127Sq = 1.0f / 16129.0f;

struct KParams {
    int rows_a, rows_b, K;     // operand rows (A on the MMA M side), K in bytes
    int num_m_blk, num_n_blk, num_kb;
    int M, N;                  // problem sizes: tokens, output features
    const float *sx, *sb;
    const __half *X16, *W16;
    const int8_t *CB;
    const int32_t *col_idx, *count;
    const __half *bias;        // fp16 [N] or null
    int act;                   // LLMINT8_ACT_*
    void *Y;
    uint32_t *status;
    // Zero-point codes of X (null: absmax codes): sx holds the scale s per
    // row, zx the zero point, rsum the code row sums of W.
    const int32_t *zx, *rsum;
    int out_f32;               // MixedFp16 epilogue: store fp32 (1) instead of fp16 (0)
    // Gathered outlier operands (null: gathered in place): W's outlier columns
    // [kGatherCols x np] and SB [np] (staged per tile by bulk copies), X's
    // outlier columns [kGatherCols x mp] (read per row).
    const float *wt_t, *sb_p, *xo_t;
    int np, mp;
    int y_tma;                 // Y (fp16) has a TMA store map (tmY): 32-row x 64-column boxes
    // Stream-K (CTA-pair kernel only; 0: none): the last sk_tiles tiles are
    // split over the pairs by K stages. A split tile's first part parks its
    // int32 partial accumulator in the parking pair's slot of sk_part
    // ([pairs][2 CTAs][BN/32][8][128 rows][4]) and raises that pair's flag in
    // sk_flag ([pairs][2]); the pair holding the tile's last stage adds it.
    int sk_tiles;
    int32_t *sk_part;
    uint32_t *sk_flag;
};

template <int BN, int STAGES>
struct Smem {
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int SIDE_OFF = B_OFF + STAGES * B_BYTES;          // float [OC][BN]
    static constexpr int SCALE_OFF = SIDE_OFF + OC * BN * 4;           // float [BN]
    static constexpr int COLS_OFF = SCALE_OFF + BN * 4;                // int [OC] outlier columns
    static constexpr int BAR_OFF = COLS_OFF + OC * 4;                  // uint64 barriers
    static constexpr int NBARS = 2 * STAGES + 6; // full, empty, tfull[2], tempty[2], drain, staging
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;               // tmem base, abort flag
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;                         // slack for 1024-byte alignment
    static constexpr uint32_t TMEM_COLS = (2 * BN) <= 32 ? 32 : (2 * BN) <= 64 ? 64 : (2 * BN) <= 128 ? 128
                                         : (2 * BN) <= 256 ? 256 : 512;
    static_assert(ALLOC <= 232448, "shared memory over the 227 KB per-CTA limit");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms need 1024-byte alignment");
};

__device__ __forceinline__ float wtilde(const KParams &p, int j, int c)
{
    // W's outlier column value: the fp16 weight if given, else CB * SCB / 127
    // per output row (page section "用法", Usage), in fp32.
    if (p.W16)
        return __half2float(p.W16[(int64_t)j * p.K + c]);
    return __fdiv_rn(__fmul_rn((float)p.CB[(int64_t)j * p.K + c], p.sb[j]), 127.0f);
}

__device__ __forceinline__ void report(const KParams &p, volatile int *s_abort, uint32_t bit)
{
    atomicOr(p.status, bit);
    *s_abort = 1;
}

// Epilogue of one CTA (warps 2..5): for each of its output tiles, stage the
// outlier operands and scales while the tile's MMAs run, wait for the
// accumulator, then dequantize, add the outlier product and store (or store
// the raw int32 accumulators), and hand the TMEM buffer back to the MMA
// issuer. Its work items are those of `sc` (whole tiles, and for CTA pairs
// the parts of stream-K tiles: a parked part only stores its int32 partials
// for the next pair; the part holding a tile's last stage adds the parked
// partials, copied into `sk_buf`, before the usual epilogue); this CTA's
// accumulator rows are a_row_off .. a_row_off + 127 of each a_tile_rows-row
// A tile.
// One tile's staging loads held in registers as they arrive (raw: no
// arithmetic on them, so issuing them does not wait for them): the scales of
// the thread's entries of s_scale, its row's SX and outlier values of X, and
// up to 2 x 128 x 8 gathered outlier values of W (fp16 bits, or the int8
// code and its row's SB).
constexpr int kPipeCols = 8;   // outlier columns the pipelined staging covers
constexpr int kPipeGather = 16; // gathers per thread it covers
template <int BN>
struct StageRegs {
    float sc[(BN + 127) / 128];
    float own_scale;
    uint32_t own_side[kPipeCols]; // fp16 bits of X[i, col_k]
    uint32_t g[kPipeGather];      // fp16 bits of W[r, col] or the int8 code of CB[r, col]
    float gsb[kPipeGather];       // SB[r] (code form only)
};

template <int BN>
__device__ __forceinline__ void stage_issue(const KParams &p, const int *s_cols, int cnt, int tile, int a_tile_rows,
                                            int a_row_off, int r_in_tile, int et, StageRegs<BN> &st)
{
    const int mb = tile % p.num_m_blk, nb = tile / p.num_m_blk;
    const int arow = mb * a_tile_rows + a_row_off + r_in_tile;
    const int brow0 = nb * BN;
#pragma unroll
    for (int u = 0; u < (BN + 127) / 128; ++u) {
        const int idx = et + u * 128, r = brow0 + idx;
        st.sc[u] = (idx < BN && r < p.N) ? p.sb[r] : 0.f;
    }
    st.own_scale = arow < p.M ? p.sx[arow] : 0.f;
    const unsigned short *x16 = reinterpret_cast<const unsigned short *>(p.X16);
#pragma unroll
    for (int k = 0; k < kPipeCols; ++k)
        st.own_side[k] = (k < cnt && arow < p.M) ? x16[(int64_t)arow * p.K + s_cols[k]] : 0u;
    const unsigned short *w16 = reinterpret_cast<const unsigned short *>(p.W16);
#pragma unroll
    for (int u = 0; u < kPipeGather; ++u) {
        const int idx = u * 128 + et;
        uint32_t v = 0u;
        float sbv = 0.f;
        if (idx < cnt * BN) {
            const int k = idx / BN, r = brow0 + (idx - k * BN);
            if (r < p.N) {
                const int64_t off = (int64_t)r * p.K + s_cols[k];
                if (p.W16) {
                    v = w16[off];
                } else {
                    v = (uint32_t)(uint8_t)p.CB[off];
                    sbv = p.sb[r];
                }
            }
        }
        st.g[u] = v;
        st.gsb[u] = sbv;
    }
}

template <int BN, bool SWAP, bool RAW, bool PAIR>
__device__ __forceinline__ void run_epilogue(const KParams &p, const CUtensorMap *tmY, int warp, int lane,
                                             float *s_side, float *s_scale, int *s_cols,
                                             uint32_t tfull0, uint32_t tempty0, uint32_t sbar, volatile int *s_abort,
                                             uint32_t tmem_base, const Sched &sc, int a_tile_rows, int a_row_off,
                                             uint8_t *sk_buf)
{
    auto tfull_bar = [&](int b) { return tfull0 + 8u * b; };
    auto tempty_bar = [&](int b) { return tempty0 + 8u * b; };
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int et = threadIdx.x - 64;        // 0..127
    const int r_in_tile = q * 32 + lane;    // accumulator row (A-side row in the tile)
    const int cnt = RAW ? 0 : min(*p.count, p.K);
    const bool fast = cnt <= OC;
    if (!RAW && fast) {
        // The outlier columns, the same for every tile, once into shared memory.
        for (int k = et; k < cnt; k += 128)
            s_cols[k] = p.col_idx[k];
        named_barrier_sync(1, 128);
    }
    uint32_t tph[2] = {0u, 0u};
    int local = 0;
    // Few outlier columns: the next tile's staging loads go out before this
    // tile's epilogue and land while it runs (under the TMA stream a round of
    // them takes several microseconds, longer than a K = 4096 tile's MMAs).
    static_assert(RAW || SWAP || OC * BN >= (kPipeGather + kPipeCols) * 128,
                  "the pipelined staging keeps W's values and X's values in s_side");
    // Gathered operands (a kernel before this one copied W's and X's outlier
    // columns into contiguous arrays): the tile's slice of W's columns and of
    // SB arrive by bulk copies on `sbar`, issued by one thread as soon as the
    // previous tile's epilogue is done with s_side; no per-thread gathers run
    // next to the MMAs.
    const bool gathered = !RAW && !SWAP && p.wt_t != nullptr && fast;
    // X's values of the CTA's 128 rows follow W's in s_side when both fit
    const bool x_in_smem = gathered && cnt * (BN + 128) <= OC * BN;
    const bool pipe = !gathered && !RAW && !SWAP && fast && cnt <= kPipeCols && cnt * BN <= kPipeGather * 128;
    // Output through shared memory and TMA stores (coalesced, async) when the
    // staged operands leave the last 16 KB of s_side (OC * BN floats) free:
    // each warp stages its 32 rows x 64 columns (fp16, 128-byte swizzle,
    // 4 KB, 1024-byte aligned) there.
    constexpr int kSideBytes = OC * BN * 4;
    const bool tma_st = x_in_smem && p.y_tma && !p.out_f32 && cnt * (BN + 128) * 4 + kStoreStage <= kSideBytes;
    uint8_t *obuf = reinterpret_cast<uint8_t *>(s_side) + (kSideBytes - kStoreStage) + q * 4096;
    bool stores_pending = false; // (lane 0) TMA stores of this warp not yet complete
    uint32_t sph = 0u;
    bool staged_pending = false; // (thread et == 0) a staging copy is in flight
    auto issue_staging = [&](int tile) {
        const int brow0 = (tile / p.num_m_blk) * BN;
        const int arow0 = (tile % p.num_m_blk) * a_tile_rows + a_row_off;
        mbar_arrive_expect_tx(sbar, (uint32_t)(cnt + 1) * BN * 4u + (x_in_smem ? (uint32_t)cnt * 512u : 0u));
        for (int k = 0; k < cnt; ++k)
            bulk_load(smem_u32(s_side + k * BN), p.wt_t + (int64_t)k * p.np + brow0, BN * 4u, sbar);
        if (x_in_smem)
            for (int k = 0; k < cnt; ++k)
                bulk_load(smem_u32(s_side + cnt * BN + k * 128), p.xo_t + (int64_t)k * p.mp + arow0, 512u, sbar);
        bulk_load(smem_u32(s_scale), p.sb_p + brow0, BN * 4u, sbar);
        staged_pending = true;
    };
    const int nwork = sc.count();
    if (gathered && et == 0 && nwork > 0)
        issue_staging(sc.item(0).tile);
    StageRegs<BN> nx;
    if (pipe && nwork > 0)
        stage_issue<BN>(p, s_cols, cnt, sc.item(0).tile, a_tile_rows, a_row_off, r_in_tile, et, nx);
    // Stream-K slots of this CTA (rank a_row_off / BM of its pair) and of the
    // previous pair's CTA of the same rank, 128 rows x BN int32 each.
    constexpr int kSlotVec = (BN >= 32 ? BN / 32 : 1) * 8 * 128; // int4 vectors per CTA slot
    const int rank = a_row_off / BM;
    for (int w = 0; w < nwork; ++w, ++local) {
        const Seg it = sc.item(w);
        const int tile = it.tile;
        const bool park = PAIR && it.st1 < sc.S;             // K stages [0, st1): parked for the next pair
        const bool owner = PAIR && !park && it.st0 > 0;      // the previous pair parked stages [0, st0)
        const int b = local & 1;
        const int mb = tile % p.num_m_blk, nb = tile / p.num_m_blk;
        const int arow = mb * a_tile_rows + a_row_off + r_in_tile; // A-operand row of this thread
        const int brow0 = nb * BN;               // first B-operand row of the tile
        float own_scale = 0.f;
        const int own_z = (!RAW && !SWAP && p.zx && arow < p.M) ? __ldg(p.zx + arow) : 128;
        float own_side[OC];
#pragma unroll
        for (int k = 0; k < OC; ++k)
            own_side[k] = 0.f;
        if (gathered) {
            own_scale = arow < p.M ? p.sx[arow] : 0.f;
            if (!x_in_smem) {
                // too many columns for s_side: this row's outlier values into
                // registers, one coalesced load per column
#pragma unroll
                for (int k = 0; k < OC; ++k)
                    own_side[k] = (k < cnt && arow < p.M) ? __ldg(p.xo_t + (int64_t)k * p.mp + arow) : 0.f;
            }
            const bool landed = mbar_wait(sbar, sph);
            if (named_barrier_or(1, 128, !landed)) {
                if (!landed)
                    report(p, s_abort, LLMINT8_DEV_TIMEOUT_EPILOGUE);
                break;
            }
            sph ^= 1u;
            staged_pending = false;
        } else if (pipe) {
            named_barrier_sync(1, 128); // the previous tile's readers are done with s_side / s_scale
#pragma unroll
            for (int u = 0; u < (BN + 127) / 128; ++u)
                if (et + u * 128 < BN)
                    s_scale[et + u * 128] = nx.sc[u];
#pragma unroll
            for (int u = 0; u < kPipeGather; ++u) {
                const int idx = u * 128 + et;
                if (idx < cnt * BN)
                    s_side[idx] = p.W16 ? __half2float(__ushort_as_half((unsigned short)nx.g[u]))
                                        : __fdiv_rn(__fmul_rn((float)(int8_t)(uint8_t)nx.g[u], nx.gsb[u]), 127.0f);
            }
            own_scale = nx.own_scale;
            // The row's outlier values of X go to this thread's slots after
            // the staged W values (s_side holds OC * BN floats, the pipelined
            // case fills at most kPipeCols * BN + kPipeCols * 128 of them),
            // so that the outlier loop below can run over the actual count.
            float *s_own = s_side + cnt * BN;
#pragma unroll
            for (int k = 0; k < kPipeCols; ++k)
                if (k < cnt)
                    s_own[k * 128 + et] = __half2float(__ushort_as_half((unsigned short)nx.own_side[k]));
            named_barrier_sync(1, 128);
            if (w + 1 < nwork)
                stage_issue<BN>(p, s_cols, cnt, sc.item(w + 1).tile, a_tile_rows, a_row_off, r_in_tile, et, nx);
        } else if (!RAW) {
            // Stage the tile's scales and outlier operands while the MMAs run.
            // Every load of the first round goes out before any is used (with
            // the column list in shared memory, nothing here waits on a load
            // to find its address): under the TMA stream each global round
            // trip costs a microsecond or more, and at K = 4096 a tile's MMAs
            // last only about 10 us.
            named_barrier_sync(1, 128);
            constexpr int NSC = (BN + 127) / 128;
            float sc[NSC];
#pragma unroll
            for (int u = 0; u < NSC; ++u) {
                const int idx = et + u * 128, r = brow0 + idx;
                sc[u] = 0.f;
                if (idx < BN)
                    sc[u] = SWAP ? (r < p.M ? p.sx[r] : 0.f) : (r < p.N ? p.sb[r] : 0.f);
            }
            if (SWAP) {
                if (arow < p.N) {
                    own_scale = p.sb[arow];
                    if (fast) {
#pragma unroll
                        for (int k = 0; k < OC; ++k)
                            if (k < cnt)
                                own_side[k] = wtilde(p, arow, s_cols[k]);
                    }
                }
            } else {
                if (arow < p.M) {
                    own_scale = p.sx[arow];
                    if (fast) {
#pragma unroll
                        for (int k = 0; k < OC; ++k)
                            if (k < cnt)
                                own_side[k] = __half2float(p.X16[(int64_t)arow * p.K + s_cols[k]]);
                    }
                }
            }
            if (fast) {
                // Eight independent gathers in flight per thread, then the stores.
                for (int base = 0; base < cnt * BN; base += 8 * 128) {
                    float vals[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int idx = base + u * 128 + et;
                        float v = 0.f;
                        if (idx < cnt * BN) {
                            const int k = idx / BN, c = idx - k * BN;
                            const int r = brow0 + c;
                            const int col = s_cols[k];
                            if (SWAP) {
                                if (r < p.M)
                                    v = __half2float(p.X16[(int64_t)r * p.K + col]);
                            } else {
                                if (r < p.N)
                                    v = wtilde(p, r, col);
                            }
                        }
                        vals[u] = v;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int idx = base + u * 128 + et;
                        if (idx < cnt * BN)
                            s_side[idx] = vals[u];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < NSC; ++u)
                if (et + u * 128 < BN)
                    s_scale[et + u * 128] = sc[u];
            named_barrier_sync(1, 128);
        }

        // All 128 epilogue threads leave together if any of them gave up,
        // so no thread is left waiting at a named barrier.
        const bool got = mbar_wait(tfull_bar(b), tph[b]);
        if (named_barrier_or(1, 128, !got)) {
            if (!got)
                report(p, s_abort, LLMINT8_DEV_TIMEOUT_EPILOGUE);
            break;
        }
        tph[b] ^= 1u;
        tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN);

        if (park) {
            // The tile's first stages: this row's int32 partials to the
            // pair's slot (a warp stores 512 contiguous bytes per vector).
            int4 *dst = reinterpret_cast<int4 *>(p.sk_part) + (size_t)(sc.first * 2 + rank) * kSlotVec + r_in_tile;
#pragma unroll 1
            for (int g = 0; g < BN / 32; ++g) {
                uint32_t acc[32];
                tmem_ld_32x32b_x32(tbase + g * 32, acc);
                tmem_wait_ld();
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4)
                    dst[(g * 8 + c4) * 128] = make_int4((int)acc[4 * c4], (int)acc[4 * c4 + 1], (int)acc[4 * c4 + 2],
                                                        (int)acc[4 * c4 + 3]);
            }
        } else {
            if (PAIR && owner) {
                // The tile's last stages: the partials the previous pair parked
                // (normally long ready) into this CTA's pipeline buffers, free
                // now that its last MMAs are complete, by bulk copies.
                bool ok = true;
                if (et == 0) {
                    uint32_t *flag = p.sk_flag + (sc.first - 1) * 2 + rank;
                    uint32_t f = 0u;
                    const uint64_t t0 = global_timer_ns();
                    for (;;) {
                        asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(f) : "l"(flag) : "memory");
                        if (f == 1u || global_timer_ns() - t0 > kWaitLimitNs)
                            break;
                        __nanosleep(64);
                    }
                    ok = f == 1u;
                    if (ok) {
                        *flag = 0u; // ready for the next call
                        fence_proxy_async_global();
                        const uint8_t *src = reinterpret_cast<const uint8_t *>(
                            reinterpret_cast<const int4 *>(p.sk_part) + (size_t)((sc.first - 1) * 2 + rank) * kSlotVec);
                        constexpr uint32_t bytes = (uint32_t)kSlotVec * 16u;
                        mbar_arrive_expect_tx(sbar, bytes);
                        for (uint32_t off = 0; off < bytes; off += 32768u)
                            bulk_load(smem_u32(sk_buf) + off, src + off, min(32768u, bytes - off), sbar);
                        staged_pending = true;
                    }
                }
                if (named_barrier_or(1, 128, !ok)) {
                    if (!ok)
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_EPILOGUE);
                    break;
                }
                const bool landed = mbar_wait(sbar, sph);
                if (named_barrier_or(1, 128, !landed)) {
                    if (!landed)
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_EPILOGUE);
                    break;
                }
                sph ^= 1u;
                staged_pending = false;
            }

            if constexpr (!SWAP) {
                const int i = arow;
                // More outlier columns than s_side holds at once: the columns go
                // in chunks of OC, outermost. Each chunk's W values are staged
                // for the whole tile (one round of gathers, eight in flight per
                // thread) and this row's X values go to registers once; between
                // chunks the partial sums wait in the tile's own TMEM accumulator
                // (fp32 bits in place of the int32 products), so each output
                // still adds its outlier products in ascending column order.
                const int nch = (RAW || fast) ? 1 : (cnt + OC - 1) / OC;
                for (int ch = 0; ch < nch; ++ch) {
                const int nk = min(OC, cnt - ch * OC);
                if (!RAW && !fast) {
                    named_barrier_sync(1, 128); // the previous chunk's readers are done with s_side / s_cols
                    if (et < nk)
                        s_cols[et] = p.col_idx[ch * OC + et];
                    named_barrier_sync(1, 128);
                    for (int base = 0; base < nk * BN; base += 32 * 128) { // 32 gathers in flight per thread
                        float vals[32];
#pragma unroll
                        for (int u = 0; u < 32; ++u) {
                            const int idx = base + u * 128 + et;
                            float v = 0.f;
                            if (idx < nk * BN) {
                                const int k = idx / BN, r = brow0 + (idx - k * BN);
                                if (r < p.N)
                                    v = wtilde(p, r, s_cols[k]);
                            }
                            vals[u] = v;
                        }
#pragma unroll
                        for (int u = 0; u < 32; ++u) {
                            const int idx = base + u * 128 + et;
                            if (idx < nk * BN)
                                s_side[idx] = vals[u];
                        }
                    }
#pragma unroll
                    for (int k = 0; k < OC; ++k)
                        own_side[k] =
                            (k < nk && arow < p.M) ? __half2float(p.X16[(int64_t)arow * p.K + s_cols[k]]) : 0.f;
                    named_barrier_sync(1, 128);
                }
                const bool last_chunk = ch == nch - 1;
#pragma unroll 1
                for (int g = 0; g < BN / 32; ++g) {
                    uint32_t acc[32];
                    tmem_ld_32x32b_x32(tbase + g * 32, acc);
                    tmem_wait_ld();
                    if (owner && ch == 0) {
                        // the parked partial products of this row's 32 columns
                        const int4 *pp = reinterpret_cast<const int4 *>(sk_buf) + g * 8 * 128 + r_in_tile;
#pragma unroll
                        for (int c4 = 0; c4 < 8; ++c4) {
                            const int4 v = pp[c4 * 128];
                            acc[4 * c4] += (uint32_t)v.x;
                            acc[4 * c4 + 1] += (uint32_t)v.y;
                            acc[4 * c4 + 2] += (uint32_t)v.z;
                            acc[4 * c4 + 3] += (uint32_t)v.w;
                        }
                    }
                    const int j0 = brow0 + g * 32;
                    if constexpr (RAW) {
                        int32_t *Yr = reinterpret_cast<int32_t *>(p.Y) + (int64_t)i * p.N;
                        if (i < p.M) {
                            if (j0 + 32 <= p.N && (p.N & 3) == 0) {
#pragma unroll
                                for (int c = 0; c < 32; c += 4)
                                    *reinterpret_cast<uint4 *>(Yr + j0 + c) =
                                        make_uint4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
                            } else {
                                for (int c = 0; c < 32; ++c)
                                    if (j0 + c < p.N)
                                        Yr[j0 + c] = (int32_t)acc[c];
                            }
                        }
                        continue;
                    }
                    float y[32];
                    if (ch > 0) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            y[c] = __uint_as_float(acc[c]); // the partial sums the previous chunk left
                    } else if (p.zx) {
                        // Zero-point codes: sum_k (q - z_i) CB[j,k] = acc + (128 - z_i) R[j],
                        // dequantized by SB[j] / (127 s_i) (s_i = 0: an all-zero row).
                        const float zc = (float)(128 - own_z);
                        const float inv = own_scale > 0.f ? __frcp_rn(127.0f * own_scale) : 0.f;
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int j = j0 + c;
                            const float rj = j < p.N ? (float)__ldg(p.rsum + j) : 0.f;
                            y[c] = fmaf(zc, rj, (float)(int32_t)acc[c]) * (s_scale[g * 32 + c] * inv);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            y[c] = (float)(int32_t)acc[c] * (own_scale * s_scale[g * 32 + c]) * kInv127Sq;
                    }
                    if (gathered && x_in_smem) {
                        // X's outlier values of this row, staged in s_side after W's
                        const float *xs = s_side + cnt * BN + r_in_tile; // staged in row order
#pragma unroll 1
                        for (int k = 0; k < cnt; ++k) {
                            const float xv = xs[k * 128];
                            const float4 *wrow = reinterpret_cast<const float4 *>(s_side + k * BN + g * 32);
#pragma unroll
                            for (int c4 = 0; c4 < 8; ++c4) {
                                const float4 w = wrow[c4];
                                y[4 * c4 + 0] = fmaf(xv, w.x, y[4 * c4 + 0]);
                                y[4 * c4 + 1] = fmaf(xv, w.y, y[4 * c4 + 1]);
                                y[4 * c4 + 2] = fmaf(xv, w.z, y[4 * c4 + 2]);
                                y[4 * c4 + 3] = fmaf(xv, w.w, y[4 * c4 + 3]);
                            }
                        }
                    } else if (pipe) {
                        // A loop over the actual columns: the form unrolled over
                        // OC below is about 1300 instructions per chunk, more
                        // than the instruction cache keeps next to the rest.
                        const float *s_own = s_side + cnt * BN;
#pragma unroll 1
                        for (int k = 0; k < cnt; ++k) {
                            const float xv = s_own[k * 128 + et];
                            const float4 *wrow = reinterpret_cast<const float4 *>(s_side + k * BN + g * 32);
#pragma unroll
                            for (int c4 = 0; c4 < 8; ++c4) {
                                const float4 w = wrow[c4];
                                y[4 * c4 + 0] = fmaf(xv, w.x, y[4 * c4 + 0]);
                                y[4 * c4 + 1] = fmaf(xv, w.y, y[4 * c4 + 1]);
                                y[4 * c4 + 2] = fmaf(xv, w.z, y[4 * c4 + 2]);
                                y[4 * c4 + 3] = fmaf(xv, w.w, y[4 * c4 + 3]);
                            }
                        }
                    } else if (fast) { // (gathered with X's values in registers, or gathered in place)
#pragma unroll
                        for (int k = 0; k < OC; ++k) {
                            if (k < cnt) {
                                const float xv = own_side[k];
                                const float4 *wrow = reinterpret_cast<const float4 *>(s_side + k * BN + g * 32);
#pragma unroll
                                for (int c4 = 0; c4 < 8; ++c4) {
                                    const float4 w = wrow[c4];
                                    y[4 * c4 + 0] = fmaf(xv, w.x, y[4 * c4 + 0]);
                                    y[4 * c4 + 1] = fmaf(xv, w.y, y[4 * c4 + 1]);
                                    y[4 * c4 + 2] = fmaf(xv, w.z, y[4 * c4 + 2]);
                                    y[4 * c4 + 3] = fmaf(xv, w.w, y[4 * c4 + 3]);
                                }
                            }
                        }
                    } else {
                        // chunk ch of the outlier columns (staged above; unrolled
                        // over the OC slots so that own_side stays in registers)
#pragma unroll
                        for (int k = 0; k < OC; ++k) {
                            if (k < nk) {
                                const float xv = own_side[k];
                                const float4 *wrow = reinterpret_cast<const float4 *>(s_side + k * BN + g * 32);
#pragma unroll
                                for (int c4 = 0; c4 < 8; ++c4) {
                                    const float4 w = wrow[c4];
                                    y[4 * c4 + 0] = fmaf(xv, w.x, y[4 * c4 + 0]);
                                    y[4 * c4 + 1] = fmaf(xv, w.y, y[4 * c4 + 1]);
                                    y[4 * c4 + 2] = fmaf(xv, w.z, y[4 * c4 + 2]);
                                    y[4 * c4 + 3] = fmaf(xv, w.w, y[4 * c4 + 3]);
                                }
                            }
                        }
                        if (!last_chunk) {
                            uint32_t part[32];
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                part[c] = __float_as_uint(y[c]);
                            tmem_st_32x32b_x32(tbase + g * 32, part);
                            continue;
                        }
                    }
                    if (p.bias || p.act) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int j = j0 + c;
                            const float bv = (p.bias && j < p.N) ? __half2float(__ldg(p.bias + j)) : 0.f;
                            y[c] = bias_act(y[c], bv, p.act);
                        }
                    }
                    if (i < p.M && p.out_f32) {
                        // fp32 partial output (tensor-parallel row split: summed across ranks afterwards)
                        float *Yr = reinterpret_cast<float *>(p.Y) + (int64_t)i * p.N;
                        if (j0 + 32 <= p.N && (p.N & 3) == 0) {
#pragma unroll
                            for (int c = 0; c < 32; c += 4)
                                *reinterpret_cast<float4 *>(Yr + j0 + c) =
                                    make_float4(y[c], y[c + 1], y[c + 2], y[c + 3]);
                        } else {
                            for (int c = 0; c < 32; ++c)
                                if (j0 + c < p.N)
                                    Yr[j0 + c] = y[c];
                        }
                    } else if (tma_st && (g | 1) < BN / 32) {
                        // chunk g is half of a full 64-column group: into this
                        // warp's staging buffer (row = lane, 16-byte pieces
                        // swizzled by row), and the group out by one TMA store
                        if ((g & 1) == 0) {
                            if (lane == 0 && stores_pending)
                                bulk_wait_group_read0(); // the previous group has left obuf
                            __syncwarp();
                        }
#pragma unroll
                        for (int c8 = 0; c8 < 4; ++c8) {
                            uint4 pk;
                            __half2 *h = reinterpret_cast<__half2 *>(&pk);
                            h[0] = __floats2half2_rn(y[8 * c8 + 0], y[8 * c8 + 1]);
                            h[1] = __floats2half2_rn(y[8 * c8 + 2], y[8 * c8 + 3]);
                            h[2] = __floats2half2_rn(y[8 * c8 + 4], y[8 * c8 + 5]);
                            h[3] = __floats2half2_rn(y[8 * c8 + 6], y[8 * c8 + 7]);
                            const int piece = ((g & 1) * 4 + c8) ^ (lane & 7);
                            *reinterpret_cast<uint4 *>(obuf + lane * 128 + piece * 16) = pk;
                        }
                        if (g & 1) {
                            fence_proxy_async_smem(); // this lane's pieces, before the async proxy reads them
                            __syncwarp();
                            // (a box entirely past M or N has nothing to write; a
                            // staging buffer off its 1024-byte alignment or outside
                            // s_side, or a column not on a 16-byte boundary, is
                            // reported and not stored)
                            const int x0 = brow0 + (g - 1) * 32, y0 = arow - lane;
                            const uint32_t ob = smem_u32(obuf), sb0 = smem_u32(s_side);
                            const bool sane = (ob & 1023u) == 0 && ob >= sb0 && ob + 4096u <= sb0 + kSideBytes &&
                                              (x0 & 7) == 0 && x0 >= 0 && y0 >= 0;
                            if (lane == 0 && !sane)
                                atomicOr(p.status, LLMINT8_DEV_BAD_STORE);
                            if (lane == 0 && sane && y0 < p.M && x0 < p.N) {
                                tma_store_2d(tmY, ob, x0, y0);
                                bulk_commit_group();
                                stores_pending = true;
                            }
                        }
                    } else if (i < p.M) {
                        __half *Yr = reinterpret_cast<__half *>(p.Y) + (int64_t)i * p.N;
                        if (j0 + 32 <= p.N && (p.N & 7) == 0) {
#pragma unroll
                            for (int c = 0; c < 32; c += 8) {
                                uint4 pk;
                                __half2 *h = reinterpret_cast<__half2 *>(&pk);
                                h[0] = __floats2half2_rn(y[c + 0], y[c + 1]);
                                h[1] = __floats2half2_rn(y[c + 2], y[c + 3]);
                                h[2] = __floats2half2_rn(y[c + 4], y[c + 5]);
                                h[3] = __floats2half2_rn(y[c + 6], y[c + 7]);
                                *reinterpret_cast<uint4 *>(Yr + j0 + c) = pk;
                            }
                        } else {
                            for (int c = 0; c < 32; ++c)
                                if (j0 + c < p.N)
                                    Yr[j0 + c] = __float2half_rn(y[c]);
                        }
                    }
                }
                if (!last_chunk)
                    tmem_wait_st(); // the partial sums are in TMEM before the next chunk reads them
                }
            } else {
                // Decode form: this thread owns output feature j = arow; the
                // accumulator columns are tokens brow0 .. brow0 + BN - 1.
                const int j = arow;
                uint32_t acc[BN];
                if constexpr (BN == 32) {
                    tmem_ld_32x32b_x32(tbase, acc);
                } else {
                    tmem_ld_32x32b_x16(tbase, acc);
                }
                tmem_wait_ld();
                if constexpr (RAW) {
                    if (j < p.N) {
                        int32_t *Yc = reinterpret_cast<int32_t *>(p.Y) + j;
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (brow0 + c < p.M)
                                Yc[(int64_t)(brow0 + c) * p.N] = (int32_t)acc[c];
                    }
                } else {
                    float y[BN];
                    if (p.zx) {
                        // Zero-point codes (see the other form): token c = brow0 + c.
                        const float rj = j < p.N ? (float)__ldg(p.rsum + j) : 0.f;
#pragma unroll
                        for (int c = 0; c < BN; ++c) {
                            const int r = brow0 + c;
                            const float zc = r < p.M ? (float)(128 - __ldg(p.zx + r)) : 0.f;
                            const float sc = s_scale[c];
                            const float inv = sc > 0.f ? __frcp_rn(127.0f * sc) : 0.f;
                            y[c] = fmaf(zc, rj, (float)(int32_t)acc[c]) * (own_scale * inv);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            y[c] = (float)(int32_t)acc[c] * (own_scale * s_scale[c]) * kInv127Sq;
                    }
                    if (fast) {
#pragma unroll
                        for (int k = 0; k < OC; ++k) {
                            if (k < cnt) {
                                const float wv = own_side[k];
#pragma unroll
                                for (int c = 0; c < BN; ++c)
                                    y[c] = fmaf(wv, s_side[k * BN + c], y[c]);
                            }
                        }
                    } else {
                        for (int ch = 0; ch < cnt; ch += OC) {
                            const int nk = min(OC, cnt - ch);
                            named_barrier_sync(1, 128);
                            for (int idx = et; idx < nk * BN; idx += 128) {
                                const int k = idx / BN, c = idx - k * BN;
                                const int r = brow0 + c;
                                s_side[idx] =
                                    r < p.M ? __half2float(p.X16[(int64_t)r * p.K + p.col_idx[ch + k]]) : 0.f;
                            }
                            named_barrier_sync(1, 128);
                            for (int k = 0; k < nk; ++k) {
                                const float wv = j < p.N ? wtilde(p, j, p.col_idx[ch + k]) : 0.f;
#pragma unroll
                                for (int c = 0; c < BN; ++c)
                                    y[c] = fmaf(wv, s_side[k * BN + c], y[c]);
                            }
                        }
                    }
                    if (p.bias || p.act) {
                        const float bv = (p.bias && j < p.N) ? __half2float(__ldg(p.bias + j)) : 0.f;
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            y[c] = bias_act(y[c], bv, p.act);
                    }
                    if (j < p.N && p.out_f32) {
                        float *Yc = reinterpret_cast<float *>(p.Y) + j;
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (brow0 + c < p.M)
                                Yc[(int64_t)(brow0 + c) * p.N] = y[c];
                    } else if (j < p.N) {
                        __half *Yc = reinterpret_cast<__half *>(p.Y) + j;
#pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (brow0 + c < p.M)
                                Yc[(int64_t)(brow0 + c) * p.N] = __float2half_rn(y[c]);
                    }
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            if constexpr (PAIR)
                mbar_arrive_cluster(tempty_bar(b), 0); // the pair's MMA runs in CTA 0
            else
                mbar_arrive(tempty_bar(b));
        }
        if (park) {
            // every row of the CTA stored, then the flag (release)
            __threadfence();
            named_barrier_sync(1, 128);
            if (et == 0)
                asm volatile("st.release.gpu.u32 [%0], %1;" ::"l"(p.sk_flag + sc.first * 2 + rank), "r"(1u) : "memory");
        }
        if (gathered) {
            // every reader of s_side / s_scale is done: stage the next tile
            named_barrier_sync(1, 128);
            if (et == 0 && w + 1 < nwork) {
                fence_proxy_async_smem();
                issue_staging(sc.item(w + 1).tile);
            }
        }
    }
    // A staging or stream-K copy still in flight (the loop was left early)
    // lands, and this warp's TMA stores complete, before the CTA may exit.
    if (et == 0 && staged_pending)
        mbar_wait(sbar, sph);
    if (lane == 0 && stores_pending)
        bulk_wait_group0();
}

template <int BN, int STAGES, bool SWAP, bool RAW>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_gemm_i8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmY, const KParams p)
{
    using L = Smem<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *s_side = reinterpret_cast<float *>(smem + L::SIDE_OFF);
    float *s_scale = reinterpret_cast<float *>(smem + L::SCALE_OFF);
    int *s_cols = reinterpret_cast<int *>(smem + L::COLS_OFF);
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    const uint32_t stage_bar = bar0 + 8u * (2 * STAGES + 5);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4); // one arrival per epilogue warp
        }
        mbar_init(drain_bar, 1);
        mbar_init(stage_bar, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(s_tmem), L::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (p.y_tma)
            tma_prefetch_desc(&tmY);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int num_tiles = p.num_m_blk * p.num_n_blk;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_phase = 0;
            constexpr uint32_t TX = (uint32_t)(L::A_BYTES + L::B_BYTES);
            // The weight operand (A when SWAP, else B) does not depend on the
            // kernel before this one: start streaming the first tile's weight
            // tiles before waiting for the quantizer's output. (Hinting more of
            // them into L2 here was measured to slow the quantizer down by
            // queueing its few reads behind the flood.)
            const CUtensorMap *wmap = SWAP ? &tmA : &tmB;
            int pre = 0;
            if ((int)blockIdx.x < num_tiles) {
                const int mb = (int)blockIdx.x % p.num_m_blk, nb = (int)blockIdx.x / p.num_m_blk;
                const int wrow = SWAP ? mb * BM : nb * BN;
                const uint32_t woff = SWAP ? L::A_OFF : L::B_OFF;
                const uint32_t wbytes = SWAP ? L::A_BYTES : L::B_BYTES;
                pre = min(STAGES, p.num_kb);
                for (int s = 0; s < pre; ++s) {
                    mbar_arrive_expect_tx(full_bar(s), TX);
                    tma_load_2d(sbase + woff + s * wbytes, wmap, full_bar(s), s * BK, wrow);
                    armed |= 1u << s; // phase 0
                }
            }
            griddep_wait();
            for (int tile = blockIdx.x; tile < num_tiles && !*s_abort; tile += gridDim.x) {
                const int mb = tile % p.num_m_blk, nb = tile / p.num_m_blk;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (tile == (int)blockIdx.x && kb < pre) {
                        // Weight tile already in flight on this stage's barrier.
                        if (SWAP)
                            tma_load_2d(sbase + L::B_OFF + stage * L::B_BYTES, &tmB, full_bar(stage), kb * BK,
                                        nb * BN);
                        else
                            tma_load_2d(sbase + L::A_OFF + stage * L::A_BYTES, &tmA, full_bar(stage), kb * BK,
                                        mb * BM);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        continue;
                    }
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u)) {
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_PRODUCER);
                        break;
                    }
                    if (*s_abort)
                        break;
                    mbar_arrive_expect_tx(full_bar(stage), TX);
                    tma_load_2d(sbase + L::A_OFF + stage * L::A_BYTES, &tmA, full_bar(stage), kb * BK, mb * BM);
                    tma_load_2d(sbase + L::B_OFF + stage * L::B_BYTES, &tmB, full_bar(stage), kb * BK, nb * BN);
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
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
            constexpr uint32_t IDESC = idesc_i8(BM, BN);
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*s_abort; tile += gridDim.x, ++local) {
                const int b = local & 1;
                if (!mbar_wait(tempty_bar(b), tph[b] ^ 1u)) {
                    report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
                    break;
                }
                tph[b] ^= 1u;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                bool ok = true;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait_poll(full_bar(stage), phase)) {
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = sbase + L::A_OFF + stage * L::A_BYTES;
                    const uint32_t b0 = sbase + L::B_OFF + stage * L::B_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / UK; ++k)
                        mma_i8(d_tmem, smem_desc_k128(a0 + k * UK), smem_desc_k128(b0 + k * UK), IDESC,
                               (kb | k) != 0 ? 1u : 0u);
                    mma_commit(empty_bar(stage)); // stage free once these MMAs have read it
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                mma_commit(tfull_bar(b)); // accumulator b complete
            }
            // Wait for every MMA this thread issued before TMEM is released.
            mma_commit(drain_bar);
            if (!mbar_wait(drain_bar, 0u))
                report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
        }
        __syncwarp();
    } else {
        griddep_wait(); // SX, |O| and the outlier columns come from the quantizer
        const Sched sc = make_sched(num_tiles, 0, blockIdx.x, gridDim.x, p.num_kb);
        run_epilogue<BN, SWAP, RAW, false>(p, &tmY, warp, lane, s_side, s_scale, s_cols, tfull_bar(0), tempty_bar(0),
                                           stage_bar, s_abort, tmem_base, sc, BM, 0, nullptr);
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

// Shared-memory layout of one CTA of a pair: A holds this CTA's 128 rows,
// B its BN/2 rows, per stage; a stage spans KS 128-byte K slices (one TMA
// box and one swizzle atom column each), so the pair synchronises once per
// KS * 128 bytes of K.
template <int BN, int STAGES, int KS>
struct SmemPair {
    static constexpr int A_SUB = BM * BK;
    static constexpr int B_SUB = (BN / 2) * BK;
    static constexpr int A_BYTES = A_SUB * KS;
    static constexpr int B_BYTES = B_SUB * KS;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int SIDE_OFF = B_OFF + STAGES * B_BYTES;
    static constexpr int SCALE_OFF = SIDE_OFF + OC * BN * 4;
    static constexpr int COLS_OFF = SCALE_OFF + BN * 4;
    static constexpr int BAR_OFF = COLS_OFF + OC * 4;
    static constexpr int NBARS = 2 * STAGES + 6;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = (2 * BN) <= 256 ? 256 : 512;
    static_assert(ALLOC <= 232448, "shared memory over the 227 KB per-CTA limit");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms need 1024-byte alignment");
    static_assert(BN % 32 == 0 && BN <= 256, "pair MMA needs N a multiple of 32, at most 256");
    static_assert(BM * BN * 4 <= SIDE_OFF, "a parked stream-K partial fits in the pipeline buffers");
};

// The prefill GEMM on CTA pairs (a cluster of two CTAs on one TPC). Each pair
// computes 256 x BN output tiles with tcgen05.mma.cta_group::2 (M = 256):
// every CTA TMA-loads its own 128 A rows and BN/2 B rows per stage (no
// multicast) and counts the bytes on the even CTA's barrier; the even CTA's
// MMA thread waits there, issues the MMAs for the pair, and multicasts its
// commits (stage free, accumulator ready) to both CTAs. Each CTA's epilogue
// reads its own 128 accumulator rows from its TMEM and reports back to the
// even CTA. Per MAC this moves half the operand bytes of the single-CTA form.
// A stage holds KS K slices of 128 bytes: fewer, larger stages cut the
// barrier round trips between producer and MMA issuer per byte of K (on
// B200, KS = 2 with 3 stages runs 7-15% faster than KS = 1 with 6 stages).
template <int BN, int STAGES, int KS, bool RAW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    k_gemm_i8_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const KParams p)
{
    using L = SmemPair<BN, STAGES, KS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    float *s_side = reinterpret_cast<float *>(smem + L::SIDE_OFF);
    float *s_scale = reinterpret_cast<float *>(smem + L::SCALE_OFF);
    int *s_cols = reinterpret_cast<int *>(smem + L::COLS_OFF);
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    const uint32_t stage_bar = bar0 + 8u * (2 * STAGES + 5);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);  // the even CTA's producer arms it for both CTAs' bytes
            mbar_init(empty_bar(s), 1); // the pair's MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 8); // 4 epilogue warps in each CTA
        }
        mbar_init(drain_bar, 1);
        mbar_init(stage_bar, 1);         // this CTA's epilogue staging copies
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(s_tmem), L::TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (p.y_tma)
            tma_prefetch_desc(&tmY);
    }
    tc_fence_before();
    cluster_sync_all(); // barriers and TMEM of both CTAs ready before any cross-CTA traffic
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int num_tiles = p.num_m_blk * p.num_n_blk;
    const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int num_st = (p.num_kb + KS - 1) / KS; // stages per tile
    // K slices in stage `st` of a tile (the last one may hold fewer).
    auto slices = [&](int st) { return min(KS, p.num_kb - st * KS); };
    // Whole tiles pair_id, pair_id + num_pairs, ..., then this pair's share
    // of the stream-K tiles' stages; every role walks the same list.
    const Sched sc = make_sched(num_tiles, p.sk_tiles, pair_id, num_pairs, num_st);
    const int nwork = sc.count();

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            // Bytes both CTAs bring into one stage of `ns` slices.
            auto tx = [](int ns) { return 2u * (uint32_t)ns * (uint32_t)(L::A_SUB + L::B_SUB); };
            // The weight half (B) of the first stages goes out before the wait
            // for the quantizer's codes (A).
            int pre = 0;
            if (nwork > 0) {
                const Seg f = sc.item(0);
                const int nb = f.tile / p.num_m_blk;
                const int b_row = nb * BN + (int)rank * (BN / 2);
                pre = min(STAGES, f.st1 - f.st0);
                for (int s = 0; s < pre; ++s) {
                    const int ns = slices(f.st0 + s);
                    if (leader)
                        mbar_arrive_expect_tx(full_bar(s), tx(ns));
                    for (int j = 0; j < ns; ++j)
                        tma_load_2d_pair(sbase + L::B_OFF + s * L::B_BYTES + j * L::B_SUB, &tmB, full_bar(s),
                                         ((f.st0 + s) * KS + j) * BK, b_row);
                }
            }
            griddep_wait();
            for (int w = 0; w < nwork && !*s_abort; ++w) {
                const Seg it = sc.item(w);
                const int mb = it.tile % p.num_m_blk, nb = it.tile / p.num_m_blk;
                const int a_row = mb * 2 * BM + (int)rank * BM;
                const int b_row = nb * BN + (int)rank * (BN / 2);
                for (int st = it.st0; st < it.st1; ++st) {
                    const int ns = slices(st);
                    const uint32_t a_dst = sbase + L::A_OFF + stage * L::A_BYTES;
                    const uint32_t b_dst = sbase + L::B_OFF + stage * L::B_BYTES;
                    if (w == 0 && st - it.st0 < pre) {
                        for (int j = 0; j < ns; ++j)
                            tma_load_2d_pair(a_dst + j * L::A_SUB, &tmA, full_bar(stage), (st * KS + j) * BK, a_row);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        continue;
                    }
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u)) {
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_PRODUCER);
                        break;
                    }
                    if (*s_abort)
                        break;
                    if (leader)
                        mbar_arrive_expect_tx(full_bar(stage), tx(ns));
                    for (int j = 0; j < ns; ++j) {
                        tma_load_2d_pair(a_dst + j * L::A_SUB, &tmA, full_bar(stage), (st * KS + j) * BK, a_row);
                        tma_load_2d_pair(b_dst + j * L::B_SUB, &tmB, full_bar(stage), (st * KS + j) * BK, b_row);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (leader && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t tph[2] = {0u, 0u};
            constexpr uint32_t IDESC = idesc_i8(2 * BM, BN);
            int local = 0;
            for (int w = 0; w < nwork && !*s_abort; ++w, ++local) {
                const Seg it = sc.item(w);
                const int b = local & 1;
                if (!mbar_wait_cluster(tempty_bar(b), tph[b] ^ 1u)) {
                    report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
                    break;
                }
                tph[b] ^= 1u;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                bool ok = true;
                for (int st = it.st0; st < it.st1; ++st) {
                    if (!mbar_wait_poll(full_bar(stage), phase)) {
                        report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int ns = slices(st);
#pragma unroll
                    for (int j = 0; j < KS; ++j) {
                        if (j < ns) {
                            const uint32_t a0 = sbase + L::A_OFF + stage * L::A_BYTES + j * L::A_SUB;
                            const uint32_t b0 = sbase + L::B_OFF + stage * L::B_BYTES + j * L::B_SUB;
#pragma unroll
                            for (int k = 0; k < BK / UK; ++k)
                                mma_i8_pair(d_tmem, smem_desc_k128(a0 + k * UK), smem_desc_k128(b0 + k * UK), IDESC,
                                            (st != it.st0 || j != 0 || k != 0) ? 1u : 0u);
                        }
                    }
                    mma_commit_pair_mc(empty_bar(stage), 0x3); // both CTAs' stage is free
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                mma_commit_pair_mc(tfull_bar(b), 0x3); // both halves of accumulator b are ready
            }
            mma_commit_pair(drain_bar);
            if (!mbar_wait(drain_bar, 0u))
                report(p, s_abort, LLMINT8_DEV_TIMEOUT_MMA);
        }
        __syncwarp();
    } else {
        griddep_wait(); // SX, |O| and the outlier columns come from the quantizer
        run_epilogue<BN, false, RAW, true>(p, &tmY, warp, lane, s_side, s_scale, s_cols, tfull_bar(0), tempty_bar(0),
                                           stage_bar, s_abort, tmem_base, sc, 2 * BM, (int)rank * BM,
                                           smem + L::A_OFF);
    }

    tc_fence_before();
    cluster_sync_all(); // both CTAs done with TMEM and with each other's barriers
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
    }
}

// The epilogue's outlier operands, gathered once per call (launch_gather_outliers):
// wt_t[k][j] = Wt[j, col_k] (the fp16 weight, or CB * SB / 127 per output row,
// in fp32), xo_t[k][i] = X[i, col_k], sb_p[j] = SB[j], zero past N, for the
// first |O| <= kGatherCols outlier columns (none written for more: the
// epilogue then gathers in place). One element a thread, so that every
// scattered read is in flight at once.
__global__ void __launch_bounds__(256)
    k_gather_outliers(const KParams p, float *__restrict__ wt_t, float *__restrict__ sb_p, float *__restrict__ xo_t)
{
    __shared__ int s_c[kGatherCols];
    griddep_wait(); // the quantizer's outlier list
    griddep_release();
    const int cnt = min(*p.count, p.K);
    const int kk = cnt <= kGatherCols ? cnt : 0;
    if ((int)threadIdx.x < kGatherCols)
        s_c[threadIdx.x] = (int)threadIdx.x < kk ? p.col_idx[threadIdx.x] : 0;
    __syncthreads();
    const int64_t per = (int64_t)p.np + p.mp; // items of one outlier column
    const int64_t total = (int64_t)(kk > 0 ? kk : 1) * per;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int k = (int)(t / per);
        const int64_t r = t - (int64_t)k * per;
        if (r < p.np) {
            const int j = (int)r;
            const bool in = j < p.N;
            if (k == 0)
                sb_p[j] = in ? p.sb[j] : 0.f;
            if (kk > 0)
                wt_t[(int64_t)k * p.np + j] = in ? wtilde(p, j, s_c[k]) : 0.f;
        } else if (kk > 0) {
            const int i = (int)(r - p.np);
            if (i < p.M)
                xo_t[(int64_t)k * p.mp + i] = __half2float(p.X16[(int64_t)i * p.K + s_c[k]]);
        }
    }
}

// ---------------------------------------------------------------- host side

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream finishes (it waits with griddep_wait()
// before reading that kernel's output).
template <typename Kern>
cudaError_t launch_dependent(Kern kern, int grid, int smem, cudaStream_t stream, const CUtensorMap &ta,
                             const CUtensorMap &tb, const CUtensorMap &ty, const KParams &p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p);
}

} // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Row-major int8 [rows x K] as a 2-D tensor map with a 128-byte x box_rows box.
// Encoded maps are cached (keyed on device, address, shape and box) so that
// repeated calls on the same buffers skip the driver call between launches.
bool encode_map_i8(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_map_i8(CUtensorMap *map, int device, const void *base, int64_t rows, int64_t K, int box_rows)
{
    struct Entry {
        int device;
        const void *base;
        int64_t rows, K;
        int box_rows;
        CUtensorMap map;
    };
    constexpr int kCache = 32;
    static std::mutex mu;
    static Entry cache[kCache];
    static int used = 0, next = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i) {
            const Entry &e = cache[i];
            if (e.device == device && e.base == base && e.rows == rows && e.K == K && e.box_rows == box_rows) {
                *map = e.map;
                return true;
            }
        }
    }
    if (!encode_map_i8(map, base, rows, K, box_rows))
        return false;
    std::lock_guard<std::mutex> lock(mu);
    Entry &e = cache[next];
    e = Entry{device, base, rows, K, box_rows, *map};
    next = (next + 1) % kCache;
    used = used < kCache ? used + 1 : kCache;
    return true;
}

// Y fp16 [rows x cols] as a 2-D TMA map for the epilogue's stores: 64-column
// (128-byte) x 32-row boxes, 128-byte swizzle; cached like the operand maps.
bool make_map_y16(CUtensorMap *map, int device, const void *base, int64_t rows, int64_t cols)
{
    struct Entry {
        int device;
        const void *base;
        int64_t rows, cols;
        CUtensorMap map;
    };
    constexpr int kCache = 16;
    static std::mutex mu;
    static Entry cache[kCache];
    static int used = 0, next = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i) {
            const Entry &e = cache[i];
            if (e.device == device && e.base == base && e.rows == rows && e.cols == cols) {
                *map = e.map;
                return true;
            }
        }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, 32};
    cuuint32_t estr[2] = {1, 1};
    if (enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    Entry &e = cache[next];
    e = Entry{device, base, rows, cols, *map};
    next = (next + 1) % kCache;
    used = used < kCache ? used + 1 : kCache;
    return true;
}

namespace {

// The fp16 output goes out by TMA stores when the epilogue produces fp16 and
// Y's rows are 16-byte multiples (the map then describes it exactly).
bool y_map(const GemmArgs &a, bool swap, const DeviceInfo &dev, CUtensorMap *ty)
{
    *ty = CUtensorMap{};
    if (swap || a.epi != Epilogue::MixedFp16 || a.out_f32 || a.N % 8 != 0)
        return false;
    return make_map_y16(ty, dev.device, a.Y, a.M, a.N);
}

template <int BN, int STAGES, bool SWAP, bool RAW>
cudaError_t run(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    using L = Smem<BN, STAGES>;
    auto kern = k_gemm_i8<BN, STAGES, SWAP, RAW>;
    static std::atomic<uint64_t> configured{0};
    const uint64_t bit = 1ull << (dev.device & 63);
    if (!(configured.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
        if (e != cudaSuccess)
            return e;
        configured.fetch_or(bit);
    }
    // A operand rides the MMA M side (128 rows per tile).
    const int8_t *Aop = SWAP ? a.B : a.A;
    const int8_t *Bop = SWAP ? a.A : a.B;
    const int64_t rows_a = SWAP ? a.N : a.M;
    const int64_t rows_b = SWAP ? a.M : a.N;
    CUtensorMap ta, tb;
    if (!make_map_i8(&ta, dev.device, Aop, rows_a, a.K, BM) || !make_map_i8(&tb, dev.device, Bop, rows_b, a.K, BN))
        return cudaErrorInvalidValue;
    KParams p{};
    p.rows_a = (int)rows_a;
    p.rows_b = (int)rows_b;
    p.K = (int)a.K;
    p.num_m_blk = (int)((rows_a + BM - 1) / BM);
    p.num_n_blk = (int)((rows_b + BN - 1) / BN);
    p.num_kb = (int)((a.K + BK - 1) / BK);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.sx = a.sx;
    p.sb = a.sb;
    p.X16 = reinterpret_cast<const __half *>(a.X16);
    p.W16 = reinterpret_cast<const __half *>(a.W16);
    p.CB = a.B;
    p.col_idx = a.col_idx;
    p.count = a.count;
    p.bias = reinterpret_cast<const __half *>(a.bias);
    p.act = a.act;
    p.Y = a.Y;
    p.status = a.status;
    p.zx = a.zx;
    p.rsum = a.rsum;
    p.out_f32 = a.out_f32;
    p.wt_t = SWAP ? nullptr : a.wt_t;
    p.sb_p = a.sb_p;
    p.xo_t = a.xo_t;
    p.np = (int)a.np;
    p.mp = (int)a.mp;
    CUtensorMap ty;
    p.y_tma = y_map(a, SWAP, dev, &ty) ? 1 : 0;
    const int tiles = p.num_m_blk * p.num_n_blk;
    const int grid = std::min(tiles, dev.num_sms);
    return launch_dependent(kern, grid, L::ALLOC, stream, ta, tb, ty, p);
}

template <int BN, int STAGES, int KS, bool RAW>
cudaError_t run_pair(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream, bool stream_k)
{
    using L = SmemPair<BN, STAGES, KS>;
    auto kern = k_gemm_i8_pair<BN, STAGES, KS, RAW>;
    static std::atomic<uint64_t> configured{0};
    const uint64_t bit = 1ull << (dev.device & 63);
    if (!(configured.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
        if (e != cudaSuccess)
            return e;
        configured.fetch_or(bit);
    }
    CUtensorMap ta, tb;
    if (!make_map_i8(&ta, dev.device, a.A, a.M, a.K, BM) || !make_map_i8(&tb, dev.device, a.B, a.N, a.K, BN / 2))
        return cudaErrorInvalidValue;
    KParams p{};
    p.rows_a = (int)a.M;
    p.rows_b = (int)a.N;
    p.K = (int)a.K;
    p.num_m_blk = (int)((a.M + 2 * BM - 1) / (2 * BM));
    p.num_n_blk = (int)((a.N + BN - 1) / BN);
    p.num_kb = (int)((a.K + BK - 1) / BK);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.sx = a.sx;
    p.sb = a.sb;
    p.X16 = reinterpret_cast<const __half *>(a.X16);
    p.W16 = reinterpret_cast<const __half *>(a.W16);
    p.CB = a.B;
    p.col_idx = a.col_idx;
    p.count = a.count;
    p.bias = reinterpret_cast<const __half *>(a.bias);
    p.act = a.act;
    p.Y = a.Y;
    p.status = a.status;
    p.zx = a.zx;
    p.rsum = a.rsum;
    p.out_f32 = a.out_f32;
    p.wt_t = a.wt_t;
    p.sb_p = a.sb_p;
    p.xo_t = a.xo_t;
    p.np = (int)a.np;
    p.mp = (int)a.mp;
    CUtensorMap ty;
    p.y_tma = y_map(a, false, dev, &ty) ? 1 : 0;
    const int tiles = p.num_m_blk * p.num_n_blk;
    const int pairs = std::min(tiles, dev.num_sms / 2);
    // Stream-K: the last one to two rounds' worth of tiles (at least one tile
    // per pair) split evenly over the pairs by K stages.
    p.sk_tiles = 0;
    p.sk_part = a.sk_part;
    p.sk_flag = a.sk_flag;
    if (stream_k) {
        if (!a.sk_part || !a.sk_flag || pairs > kSkMaxPairs || tiles <= pairs || KS != kStageSlices)
            return cudaErrorInvalidValue;
        p.sk_tiles = sk_tile_count(tiles, pairs);
    }
    return launch_dependent(kern, 2 * pairs, L::ALLOC, stream, ta, tb, ty, p);
}

// Tile width for the persistent prefill GEMM: the one that minimises the
// number of tile waves times the tile width (a tile's main loop is
// proportional to its width), preferring wider tiles on ties. 224 divides
// 14336, 43008 and 57344 exactly, which removes the ragged last wave.
int pick_bn(int64_t M, int64_t N, int num_sms)
{
    static const int cands[] = {256, 224, 192, 128};
    int best = 256;
    int64_t best_cost = INT64_MAX;
    for (int bn : cands) {
        const int64_t tiles = ((M + BM - 1) / BM) * ((N + bn - 1) / bn);
        const int64_t waves = (tiles + num_sms - 1) / num_sms;
        const int64_t cost = waves * bn;
        if (cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

template <bool RAW>
cudaError_t run_prefill(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    if (a.M >= 2 * BM && dev.num_sms >= 2) {
        const PairPlan plan = pick_pair_plan(a.M, a.N, a.K, dev.num_sms / 2, a.sk_part && a.sk_flag, kSkMaxPairs);
        switch (plan.bn) {
        case 224: return run_pair<224, 3, 2, RAW>(a, dev, stream, false);
        case 192: return run_pair<192, 3, 2, RAW>(a, dev, stream, false);
        case 128: return run_pair<128, 4, 2, RAW>(a, dev, stream, false);
        default: return run_pair<256, 3, 2, RAW>(a, dev, stream, plan.stream_k);
        }
    }
    switch (pick_bn(a.M, a.N, dev.num_sms)) {
    case 224: return run<224, 4, false, RAW>(a, dev, stream);
    case 192: return run<192, 5, false, RAW>(a, dev, stream);
    case 128: return run<128, 6, false, RAW>(a, dev, stream);
    default: return run<256, 4, false, RAW>(a, dev, stream);
    }
}

} // namespace

cudaError_t launch_gather_outliers(const GemmArgs &a, float *wt_t, float *sb_p, float *xo_t, int64_t np, int64_t mp,
                                   const DeviceInfo &dev, cudaStream_t stream)
{
    KParams p{};
    p.K = (int)a.K;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.sb = a.sb;
    p.X16 = reinterpret_cast<const __half *>(a.X16);
    p.W16 = reinterpret_cast<const __half *>(a.W16);
    p.CB = a.B;
    p.col_idx = a.col_idx;
    p.count = a.count;
    p.np = (int)np;
    p.mp = (int)mp;
    const int64_t total = (int64_t)kGatherCols * (np + mp);
    const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)dev.num_sms * 8);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_gather_outliers, p, wt_t, sb_p, xo_t);
}

cudaError_t launch_gemm(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    if (a.M <= 0 || a.N <= 0)
        return cudaSuccess;
    const bool raw = a.epi == Epilogue::RawInt32;
    if (a.M <= 16)
        return raw ? run<16, 12, true, true>(a, dev, stream) : run<16, 12, true, false>(a, dev, stream);
    if (a.M <= 32)
        return raw ? run<32, 10, true, true>(a, dev, stream) : run<32, 10, true, false>(a, dev, stream);
    return raw ? run_prefill<true>(a, dev, stream) : run_prefill<false>(a, dev, stream);
}

} // namespace llmint8
