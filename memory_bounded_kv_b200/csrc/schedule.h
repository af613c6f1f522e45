// Host-side scheduling of the round-robin decode attention (plain C++, no CUDA): included by
// kvb.cu and compiled on its own by the CPU tests.
#pragma once

#include <numeric>

namespace kvb {

// Grid of the round-robin attention (CTA c takes units c, c + grid, ...): as many CTAs as keep every
// CTA's unit count equal to the busiest one's (the makespan in units is unchanged and no CTA idles
// while the others finish). With fixed-length splits a row's first splits hold its slots and its
// last ones are empty, and CTA c meets only the split indices congruent to c modulo gcd(grid, S):
// then the grid is lowered to the nearest count coprime with S, if that adds at most one unit to
// the busiest CTA's count and it had at least four (measured on the memento workload: splits of
// 1280 slots, 14 per row, on 287 CTAs, 7 modulo 14, took 125 us per step against 86 us at 768).
inline int rr_grid(int units, int slots, int S, bool fixed_splits) {
    const int per_cta = (units + slots - 1) / slots;
    const int grid = (units + per_cta - 1) / per_cta;
    if (!fixed_splits || S < 2 || per_cta < 4 || std::gcd(grid, S) == 1) return grid;
    for (int g = grid - 1; g > 0; --g) {
        if ((units + g - 1) / g > per_cta + 1) break;
        if (std::gcd(g, S) == 1) return g;
    }
    return grid;
}

}  // namespace kvb
