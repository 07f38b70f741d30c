// Work lists of the persistent CTA-pair GEMM and its tile plan. Host and
// device code both use them: the kernel's three roles (TMA producer, MMA
// issuer, epilogue) walk the same list, and a CPU test checks the lists'
// invariants over many shapes.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define LLMINT8_HD __host__ __device__ __forceinline__
#else
#define LLMINT8_HD inline
#endif

namespace llmint8 {

// Pair tiles are kPairRows rows of A (two CTAs of 128) by BN rows of B; a
// K stage is kStageSlices slices of kSliceBytes bytes of K.
constexpr int kPairRows = 256;
constexpr int kSliceBytes = 128;
constexpr int kStageSlices = 2;

// One unit of a pair's work: K stages [st0, st1) of a tile.
struct Seg {
    int tile, st0, st1;
};

// The work of one CTA (or pair) `first` of `step`, in processing order:
// whole tiles first, first + step, ... below the stream-K tiles; then its
// share of the stream-K tiles' stages, a contiguous range of the stages of
// those tiles in order, cut at tile boundaries and taken from its end to its
// start. Each range spans at least one tile's stages and fewer than three
// tiles (the stream-K tiles number between one and two per pair), so a
// range is at most three segments: the part of a tile it ends in (parked
// for the pair that holds the tile's last stage, and processed first, so
// that no pair waits for one that is itself waiting), whole tiles, and the
// part of a tile it starts in (whose other part the previous pair parked;
// processed last).
struct Sched {
    int first, step, ndp, nseg, S;
    Seg seg[3];
    LLMINT8_HD int count() const { return ndp + nseg; }
    LLMINT8_HD Seg item(int w) const
    {
        if (w < ndp)
            return Seg{first + w * step, 0, S};
        return seg[w - ndp];
    }
};

LLMINT8_HD Sched make_sched(int num_tiles, int sk_tiles, int first, int step, int S)
{
    Sched sc;
    sc.first = first;
    sc.step = step;
    sc.S = S;
    sc.nseg = 0;
    const int dp_end = num_tiles - sk_tiles;
    sc.ndp = first < dp_end ? (dp_end - first + step - 1) / step : 0;
    if (sk_tiles > 0) {
        const int64_t U = (int64_t)sk_tiles * S;
        const int64_t g0 = U * first / step;
        int64_t e = U * (first + 1) / step;
        while (e > g0 && sc.nseg < 3) {
            const int64_t t = (e - 1) / S;
            const int64_t lo = g0 > t * S ? g0 : t * S;
            sc.seg[sc.nseg++] = Seg{dp_end + (int)t, (int)(lo - t * S), (int)(e - t * S)};
            e = lo;
        }
    }
    return sc;
}

// Tiles that run stream-K when `tiles` tiles (more than `pairs`) are
// planned that way: the last one to two rounds' worth, at least one tile
// per pair.
LLMINT8_HD int sk_tile_count(int tiles, int pairs) { return tiles - (tiles / pairs - 1) * pairs; }

// Tile width for CTA-pair tiles (kPairRows x BN), and whether the last tiles
// run stream-K: the plan that minimises the tile rounds times the time of
// one tile. A tile's time is proportional to its width divided by the
// tensor pipe's efficiency at that width (measured on B200: N = 224 runs at
// about 95% of the per-column rate of N = 256). Stream-K (N = 256 tiles,
// when the workspace has the slots and a tile has at least two K stages)
// spreads the tiles' work evenly over the pairs; its fix-ups (a parked
// partial per pair, stored once and read once) are charged as 2% of the
// total.
struct PairPlan {
    int bn;
    bool stream_k;
};

inline PairPlan pick_pair_plan(int64_t M, int64_t N, int64_t K, int num_pairs, bool sk_slots, int sk_max_pairs)
{
    static const int cands[] = {256, 224, 192, 128};
    static const int eff_permille[] = {1000, 946, 920, 950};
    const int64_t m_blk = (M + kPairRows - 1) / kPairRows;
    PairPlan best{256, false};
    int64_t best_cost = INT64_MAX;
    for (int i = 0; i < 4; ++i) {
        const int bn = cands[i];
        const int64_t tiles = m_blk * ((N + bn - 1) / bn);
        const int64_t pairs = tiles < num_pairs ? tiles : num_pairs;
        const int64_t cost = ((tiles + pairs - 1) / pairs) * bn * 1000000 / eff_permille[i];
        if (cost < best_cost) {
            best_cost = cost;
            best = PairPlan{bn, false};
        }
    }
    const int64_t tiles = m_blk * ((N + 255) / 256);
    const int64_t slices = (K + kSliceBytes - 1) / kSliceBytes;
    const int64_t stages = (slices + kStageSlices - 1) / kStageSlices;
    if (sk_slots && num_pairs <= sk_max_pairs && tiles > num_pairs && tiles % num_pairs != 0 && stages >= 2) {
        const int64_t cost = tiles * 256 * 1020 / num_pairs;
        if (cost < best_cost)
            best = PairPlan{256, true};
    }
    return best;
}

} // namespace llmint8
