// units.cuh -- dynamic hand-out of work units to the persistent attention kernels.
//
// A work unit is one (tile, sequence, head) triple: a query tile of a sequence in the
// forward, a key tile in the backward.  Units are numbered tile rank first, then sequence,
// then head, with the tile ranks ordered so that the most expensive tiles come first.  One
// producer thread per CTA takes the next number from a global counter and publishes it in a
// ring of kUnitRing slots in shared memory; the CTA's other roles read the ring in order.
// A CTA that drew cheap units draws more, so all CTAs finish at about the same time
// whatever the mix of sequence lengths.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace hstu {

using sm100::mbar_arrive;
using sm100::mbar_wait;

constexpr int kUnitRing = 4;

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, long long limit)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit));
}

// One arrival per warp on `bar` (counted per warp), after the whole warp got here.
__device__ __forceinline__ void warp_arrive(uint64_t *bar)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

enum FeedRole { FEED_PRODUCER, FEED_THREAD, FEED_WARP };

// One published unit: its number (-1: no more units) and its sequence, read once by the
// producer so that consumers start the unit without global loads.
struct UnitSlot {
    int64_t u;
    SeqInfo s;
};

// The shared-memory ring and the global counter of one CTA.
struct FeedRing {
    uint64_t *full, *empty;      // kUnitRing barriers each
    UnitSlot *slots;             // kUnitRing slots
    unsigned long long *ctr;
};

// ROLE: FEED_PRODUCER (the one thread that draws units), FEED_THREAD (a single consumer
// thread) or FEED_WARP (a whole warp that consumes as one, arriving once).  Each full
// barrier of the ring counts 1 arrival, each empty barrier one per consumer (thread or
// warp).  TILE is the tile height in tokens; ASCENDING numbers tile rank r as tile r, else
// as tile ntiles - 1 - r.
template <int ROLE, bool ASCENDING, int TILE>
struct UnitFeed {
    const DevParams &p;
    uint64_t *full, *empty;
    UnitSlot *slots;
    unsigned long long *ctr;
    int ntiles;
    int64_t total;
    int k = 0;                   // units taken so far
    bool ok = true;              // false once a bounded wait gave up
    SeqInfo s;
    int tile = 0, b = 0, h = 0;

    __device__ UnitFeed(const DevParams &p_, const FeedRing &r, int ntiles_)
        : p(p_), full(r.full), empty(r.empty), slots(r.slots), ctr(r.ctr), ntiles(ntiles_),
          total((int64_t)ntiles_ * p_.B * p_.H) {}

    __device__ __forceinline__ void decode(int64_t u)
    {
        const int64_t bh = (int64_t)p.B * p.H;
        const int r = (int)(u / bh);
        tile = ASCENDING ? r : ntiles - 1 - r;
        const int rem = (int)(u % bh);
        b = rem / p.H;
        h = rem % p.H;
    }

    // Decodes x and tells whether its tile lies inside its sequence (leaves s loaded).
    __device__ __forceinline__ bool admissible(int64_t x)
    {
        decode(x);
        if (!seq_may_have_tile(p, b, tile)) return false;
        s = load_seq(p, b, false);
        // the forward in candidates-only mode skips query tiles without a candidate row
        if (!ASCENDING && (p.flags & HSTU_FLAG_CANDIDATES_ONLY) && (tile + 1) * TILE <= s.E)
            return false;
        return tile * TILE < s.L;
    }

    // The next unit from the global counter, or -1 once they are exhausted.  The draw is
    // made only when the producer is ready for the unit: drawing earlier (a unit ahead)
    // measured slower, as a CTA then holds a unit that an idle CTA could have taken.
    __device__ __forceinline__ int64_t claim()
    {
        while (true) {
            const int64_t x = (int64_t)atomicAdd(ctr, 1ull);
            if (x >= total) return -1;
            if (admissible(x)) return x;
        }
    }

    // Takes the next unit: true with tile, b, h and s set; false when there are no more
    // units or a bounded wait gave up (ok false).
    __device__ __forceinline__ bool next()
    {
        const int sl = k % kUnitRing;
        const uint32_t round = (uint32_t)(k / kUnitRing);
        ++k;
        if constexpr (ROLE == FEED_PRODUCER) {
            const int64_t u = claim();
            if (round > 0 && !mbar_wait(&empty[sl], (round - 1) & 1, p.wait_limit)) {
                ok = false;
                return false;
            }
            slots[sl].u = u;
            if (u >= 0) slots[sl].s = s;
            mbar_arrive(&full[sl]);      // releases the slot's contents
            return u >= 0;
        } else {
            const bool got = ROLE == FEED_WARP ? warp_wait(&full[sl], round & 1, p.wait_limit)
                                               : mbar_wait(&full[sl], round & 1, p.wait_limit);
            if (!got) {
                ok = false;
                return false;
            }
            const int64_t u = slots[sl].u;
            if (u >= 0) s = slots[sl].s;
            if constexpr (ROLE == FEED_WARP) warp_arrive(&empty[sl]);
            else mbar_arrive(&empty[sl]);
            if (u < 0) return false;
            decode(u);
            return true;
        }
    }
};

}  // namespace hstu
