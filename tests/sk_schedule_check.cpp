// CPU check of the CTA-pair GEMM's work lists (csrc/sched.h, the code the
// kernel runs), built and run by tests/test_stream_k_schedule.py.
//
// For every shape given on stdin ("M N K pairs" per line) it takes the
// library's tile plan and, when the plan is stream-K, checks over all pairs:
//   - every (tile, K stage) is processed exactly once;
//   - a pair parks at most one part of a tile (stages [0, st1) with st1 < S),
//     and it is the first item after its whole tiles;
//   - a part that holds a tile's last stage but not its first (the fix-up)
//     is its pair's last item, and the previous pair parked exactly the
//     tile's stages before it;
//   - every stream-K range spans at least one tile's stages and at most three
//     segments.
// It prints one line per shape: "M N K pairs bn stream_k sk_tiles ok".
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "sched.h"

using namespace llmint8;

static int fail(const char *what, long M, long N, long K, int pairs)
{
    std::printf("FAIL %s at M=%ld N=%ld K=%ld pairs=%d\n", what, M, N, K, pairs);
    return 1;
}

int main()
{
    long M, N, K;
    int P;
    int bad = 0;
    while (std::scanf("%ld %ld %ld %d", &M, &N, &K, &P) == 4) {
        const PairPlan plan = pick_pair_plan(M, N, K, P, true, 80);
        const int m_blk = (int)((M + kPairRows - 1) / kPairRows);
        const int tiles = m_blk * (int)((N + plan.bn - 1) / plan.bn);
        const int pairs = tiles < P ? tiles : P;
        const int S = (int)(((K + kSliceBytes - 1) / kSliceBytes + kStageSlices - 1) / kStageSlices);
        const int sk = plan.stream_k ? sk_tile_count(tiles, pairs) : 0;
        if (plan.stream_k && (sk < pairs || sk >= 2 * pairs))
            bad |= fail("stream-K tile count", M, N, K, P);
        std::vector<int> seen((size_t)tiles * S, 0);
        std::vector<Seg> parked(pairs, Seg{-1, 0, 0});
        std::vector<Sched> all;
        for (int p = 0; p < pairs; ++p) {
            const Sched sc = make_sched(tiles, sk, p, pairs, S);
            all.push_back(sc);
            int parks = 0;
            for (int w = 0; w < sc.count(); ++w) {
                const Seg it = sc.item(w);
                if (it.tile < 0 || it.tile >= tiles || it.st0 < 0 || it.st0 >= it.st1 || it.st1 > S) {
                    bad |= fail("segment out of range", M, N, K, P);
                    continue;
                }
                for (int st = it.st0; st < it.st1; ++st)
                    ++seen[(size_t)it.tile * S + st];
                if (it.st1 < S) {
                    ++parks;
                    parked[p] = it;
                    if (w != sc.ndp || it.st0 != 0)
                        bad |= fail("parked part not first or not from stage 0", M, N, K, P);
                }
            }
            if (parks > 1)
                bad |= fail("more than one parked part", M, N, K, P);
            if (sk > 0) {
                const long long U = (long long)sk * S;
                const long long len = U * (p + 1) / pairs - U * p / pairs;
                if (len < S || sc.nseg > 3)
                    bad |= fail("stream-K range", M, N, K, P);
            }
        }
        for (size_t i = 0; i < seen.size(); ++i)
            if (seen[i] != 1)
                bad |= fail("stage not processed exactly once", M, N, K, P);
        for (int p = 0; p < pairs; ++p) {
            const Sched &sc = all[p];
            for (int w = 0; w < sc.count(); ++w) {
                const Seg it = sc.item(w);
                if (it.st1 == S && it.st0 > 0) {
                    if (w != sc.count() - 1)
                        bad |= fail("fix-up not last", M, N, K, P);
                    if (p == 0 || parked[p - 1].tile != it.tile || parked[p - 1].st1 != it.st0)
                        bad |= fail("fix-up without the matching park", M, N, K, P);
                }
            }
        }
        std::printf("%ld %ld %ld %d %d %d %d ok\n", M, N, K, P, plan.bn, plan.stream_k ? 1 : 0, sk);
    }
    return bad;
}
