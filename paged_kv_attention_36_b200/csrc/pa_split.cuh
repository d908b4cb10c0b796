// pa_split.cuh -- the decode CTAs' shares of the work line (host and device).
//
// The decode lays every (sequence, head group) out on one line of units (a
// unit is one page of a head group's K and V, plus a fixed weight per
// segment) and gives CTA k the units [start(k), start(k+1)).  The shares are
// equal shares of the line minus E * extra units (the first rem of them one
// unit longer), and the first E CTAs take extra units more each:
//     start(k) = k * per + min(k, rem) + min(k, E) * extra.
// owner(u) is the CTA whose share holds unit u.  E = 0 is the plain equal
// split; E > 0 serves a decode whose first E CTAs start while the other SMs
// still run the shared-prefix pass.  Compiled by the host tests too.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define PA_SPLIT_FN __host__ __device__ __forceinline__
#else
#define PA_SPLIT_FN inline
#endif

namespace pa {

struct Split {
    int64_t per, rem;
    int64_t E = 0, extra = 0;
    PA_SPLIT_FN int64_t start(int64_t k) const {
        return k * per + (k < rem ? k : rem) + (k < E ? k : E) * extra;
    }
    PA_SPLIT_FN int32_t owner(int64_t u) const {
        if (u < start(E)) {  // the first E shares: per + extra units (+1 for the first rem)
            const int64_t pe = per + extra, r = rem < E ? rem : E;
            const int64_t big = r * (pe + 1);
            return int32_t(u < big ? u / (pe + 1) : r + (u - big) / pe);
        }
        const int64_t v = u - E * extra;
        const int64_t big = rem * (per + 1);
        return int32_t(v < big ? v / (per + 1) : rem + (v - big) / per);
    }
};

// The split of W units over `grid` CTAs whose first `early` CTAs would take
// `want_extra` units more each, trimmed so that every share keeps at least
// min_pages units (else the equal split).  Needs W >= grid >= 1 (the decode's
// grid is at most ceil(W / min_pages)).
PA_SPLIT_FN Split make_split(int64_t W, int64_t grid, int64_t early, int64_t want_extra, int64_t min_pages) {
    Split s{W / grid, W % grid, 0, 0};
    if (early > 0 && want_extra > 0) {
        const int64_t E = early < grid ? early : grid;
        const int64_t room = (W - grid * min_pages) / E;
        const int64_t x = want_extra < room ? want_extra : room;
        if (x > 0) s = Split{(W - E * x) / grid, (W - E * x) % grid, E, x};
    }
    return s;
}

}  // namespace pa
