// Brute-force check of the decode's share split (csrc/pa_split.cuh) on the
// host: for random line lengths, grids, early-CTA counts and extras, the
// shares tile the line in order, the early CTAs get exactly their extra, no
// share falls below the minimum the split promises, and owner() is the
// inverse of start() for every unit of small lines.  Prints "ok <checks>".
#include <cstdio>
#include <cstdint>
#include <random>

#include "pa_split.cuh"

static int fail(const char* what, int64_t W, int64_t g, int64_t e, int64_t x, int64_t mp, int64_t k) {
    std::printf("FAIL %s: W=%lld grid=%lld early=%lld want=%lld min=%lld k=%lld\n", what, (long long)W,
                (long long)g, (long long)e, (long long)x, (long long)mp, (long long)k);
    return 1;
}

int main() {
    std::mt19937_64 rng(36036);
    long long checks = 0;
    for (int it = 0; it < 200000; ++it) {
        const int64_t min_pages = 1 + int64_t(rng() % 6);
        const int64_t W = 1 + int64_t(rng() % (it % 10 == 0 ? 200000 : 3000));
        const int64_t gmax = 1 + int64_t(rng() % 1100);
        const int64_t want_g = (W + min_pages - 1) / min_pages;  // the decode's grid: at most ceil(W / min)
        const int64_t grid = gmax < want_g ? gmax : want_g;
        const int64_t early = int64_t(rng() % (grid + 8));
        const int64_t want = (rng() % 4 == 0) ? 0 : int64_t(rng() % 200);
        const pa::Split s = pa::make_split(W, grid, early, want, min_pages);
        if (s.start(0) != 0 || s.start(grid) != W) return fail("ends", W, grid, early, want, min_pages, -1);
        if (s.extra < 0 || s.extra > want || s.E < 0 || s.E > grid) return fail("extra", W, grid, early, want, min_pages, -1);
        if (s.extra > 0 && s.E != (early < grid ? early : grid)) return fail("E", W, grid, early, want, min_pages, -1);
        const int64_t floor_len = W / grid;  // the equal split's shortest share
        for (int64_t k = 0; k < grid; ++k) {
            const int64_t a = s.start(k), b = s.start(k + 1);
            const int64_t len = b - a;
            if (len < 1) return fail("empty share", W, grid, early, want, min_pages, k);
            if (s.extra > 0 && len < min_pages) return fail("short share", W, grid, early, want, min_pages, k);
            if (s.extra == 0 && len < floor_len) return fail("equal share", W, grid, early, want, min_pages, k);
            if (k + 1 < grid && k + 1 != s.E) {  // neighbours inside one region differ by at most one unit
                const int64_t len2 = s.start(k + 2) - b;
                if (len2 > len || len - len2 > 1) return fail("order", W, grid, early, want, min_pages, k);
            }
            if (k < s.E && k + 1 < grid && s.E < grid && len < s.start(s.E + 1) - s.start(s.E) + s.extra - 1)
                return fail("early share", W, grid, early, want, min_pages, k);
            if (s.owner(a) != k || s.owner(b - 1) != k) return fail("owner ends", W, grid, early, want, min_pages, k);
            if (W <= 3000)
                for (int64_t u = a; u < b; ++u)
                    if (s.owner(u) != k) return fail("owner", W, grid, early, want, min_pages, k);
            ++checks;
        }
    }
    std::printf("ok %lld\n", checks);
    return 0;
}
