// plan.h -- host-only arithmetic of the persistent kernels' work plans (no
// CUDA types; compiled into the library and, on its own, into a CPU test).
#pragma once

#include <cstdint>

namespace duo {

// Makespan of g persistent CTAs that take the items of a list round robin
// (item x goes to CTA x mod g): n_a items of cost cost_a first, then n_b items
// of cost cost_b.  CTA b runs the a-items x < n_a with x = b (mod g), which is
// n_a / g of them plus one more for b < n_a mod g, and the b-items likewise,
// one more for the CTAs of the cyclic range [n_a mod g, n_a mod g + n_b mod g).
// So every CTA falls into one of four classes (one more a-item or not, one more
// b-item or not), and the makespan is the largest cost of a class that has a
// CTA in it.  Each cost is the same expression, count_a * cost_a + count_b *
// cost_b, as a per-CTA loop would evaluate, so the result is bit-identical.
inline double round_robin_makespan(int64_t n_a, double cost_a, int64_t n_b, double cost_b, int64_t g) {
    const int64_t qa = n_a / g, ra = n_a % g;
    const int64_t qb = n_b / g, rb = n_b % g;
    // CTAs with one more b-item: [ra, ra + rb) taken cyclically; the part past
    // g wraps onto [0, ra + rb - g), which lies inside [0, ra) because rb < g
    const int64_t wrap = ra + rb > g ? ra + rb - g : 0;
    const int64_t both = wrap;                          // extra a and extra b
    const int64_t only_a = ra - wrap;                   // extra a only
    const int64_t only_b = rb - wrap;                   // extra b only
    const int64_t neither = g - both - only_a - only_b;
    double span = 0.0;
    auto take = [&](int64_t members, int64_t ea, int64_t eb) {
        if (members <= 0) return;
        const double c = (double)(qa + ea) * cost_a + (double)(qb + eb) * cost_b;
        if (c > span) span = c;
    };
    take(both, 1, 1);
    take(only_a, 1, 0);
    take(only_b, 0, 1);
    take(neither, 0, 0);
    return span;
}

}  // namespace duo
