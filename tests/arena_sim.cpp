// Host simulation of the megakernel's stage arena: the producer reserves
// stages of mixed sizes (StageAlloc + stage_blocked, the same code the
// kernel's producer runs), an in-order consumer frees them at random
// times, and every reservation is checked by brute force against the
// stages still in flight.  Exit status 0 = no reservation overlapped.
//
// argv[1] = seed, argv[2] = reservations, argv[3] = 1 to use the rule that
// only checks the oldest in-flight stage (expected to fail: the regression
// this simulation guards against).  With the library's rule every decision
// is also compared with a brute-force check over the stages in flight.
#include <cstdio>
#include <cstdlib>
#include <deque>
#include <random>

#include "et_shared.h"

using namespace et;

static bool tail_only_blocked(uint32_t off, uint32_t size, uint32_t tail, uint32_t nst, const uint32_t* r_off,
                              const uint32_t* r_end) {
    if (nst - tail >= (uint32_t)kSlots) return true;
    if (tail == nst) return false;
    const uint32_t ts = tail % kSlots;
    return off < r_end[ts] && r_off[ts] < off + size;
}

int main(int argc, char** argv) {
    const unsigned seed = argc > 1 ? (unsigned)atoi(argv[1]) : 1u;
    const long n_res = argc > 2 ? atol(argv[2]) : 100000;
    const bool tail_only = argc > 3 && atoi(argv[3]) == 1;
    std::mt19937 rng(seed);
    uint32_t r_off[kSlots], r_end[kSlots];
    uint32_t tail = 0, nst = 0;
    StageAlloc alloc;
    struct Range { uint32_t id, lo, hi; };
    std::deque<Range> inflight;
    long max_inflight = 0;
    for (long i = 0; i < n_res; ++i) {
        // a stage of a tensor-core task (weight tile + N rows, N = 16..128)
        // or of a stream task (1 KB multiples)
        uint32_t size;
        if (rng() % 4 == 0) {
            size = 1024u * (1u + rng() % 64u);
        } else {
            const uint32_t n = 16u * (1u + rng() % 8u);
            size = (uint32_t)kAStageBytes + 2u * n * 128u;
        }
        // the consumer finishes zero or more of the oldest stages
        const uint32_t done = rng() % 3u;
        for (uint32_t k = 0; k < done && tail < nst; ++k) {
            ++tail;
            inflight.pop_front();
        }
        const uint32_t off = alloc.next(size);
        for (;;) {
            const bool blocked = tail < nst && (tail_only ? tail_only_blocked(off, size, tail, nst, r_off, r_end)
                                                          : stage_blocked(off, size, tail, nst, r_off, r_end));
            if (!tail_only) {
                // the O(1) rule must agree with the brute-force one both ways:
                // no overwrite, and no wait that is not needed
                bool brute = inflight.size() >= (size_t)kSlots;
                for (const Range& r : inflight) brute = brute || (off < r.hi && r.lo < off + size);
                if (brute != blocked) {
                    printf("stage %ld [%u, %u): rule says %d, brute force %d\n", i, off, off + size, (int)blocked,
                           (int)brute);
                    return 4;
                }
            }
            if (!blocked) break;
            ++tail;  // wait for the oldest stage
            inflight.pop_front();
        }
        if (off + size > (uint32_t)kArenaBytes) {
            printf("stage %ld [%u, %u) beyond the arena\n", i, off, off + size);
            return 1;
        }
        for (const Range& r : inflight)
            if (off < r.hi && r.lo < off + size) {
                printf("stage %ld [%u, %u) overwrites in-flight stage %u [%u, %u)\n", i, off, off + size, r.id,
                       r.lo, r.hi);
                return 2;
            }
        if (inflight.size() >= (size_t)kSlots) {
            printf("stage %ld: %zu stages in flight for %d slots\n", i, inflight.size(), kSlots);
            return 3;
        }
        const uint32_t slot = nst % kSlots;
        r_off[slot] = off;
        r_end[slot] = off + size;
        inflight.push_back({nst, off, off + size});
        ++nst;
        if ((long)inflight.size() > max_inflight) max_inflight = (long)inflight.size();
    }
    printf("ok %ld reservations, up to %ld stages in flight\n", n_res, max_inflight);
    return 0;
}
