"""The verify-block planner's makespan in closed form (csrc/plan.h) against a
per-CTA count of the same round-robin assignment, compiled with g++ on the
CPU: every (n_a, n_b, g) of a grid, for several costs, bit for bit."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kv_cache_reduction_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <cstdint>
#include <algorithm>
#include "plan.h"

// the makespan counted CTA by CTA: item x (0 <= x < n_a + n_b) goes to CTA x mod g;
// items below n_a cost cost_a, the others cost_b
static double per_cta(int64_t n_a, double cost_a, int64_t n_b, double cost_b, int64_t g) {
    double span = 0.0;
    for (int64_t b = 0; b < g; ++b) {
        int64_t ca = 0, cb = 0;
        for (int64_t x = b; x < n_a + n_b; x += g) (x < n_a ? ca : cb) += 1;
        span = std::max(span, ca * cost_a + cb * cost_b);
    }
    return span;
}

int main() {
    const double costs[][2] = {{1.8, 3.8}, {6.0, 1.5}, {33.4, 5.4}, {2.6, 2.6}};
    long checked = 0, bad = 0;
    for (auto &c : costs)
        for (int64_t n_a = 1; n_a <= 120; ++n_a)
            for (int64_t n_b = 0; n_b <= 120; n_b += (n_b < 20 ? 1 : 7))
                for (int64_t g = 1; g <= 150; ++g) {
                    const double want = per_cta(n_a, c[0], n_b, c[1], g);
                    const double got = duo::round_robin_makespan(n_a, c[0], n_b, c[1], g);
                    ++checked;
                    if (got != want) {
                        if (bad < 5) std::printf("n_a %ld n_b %ld g %ld: %.17g vs %.17g\n",
                                                 (long)n_a, (long)n_b, (long)g, got, want);
                        ++bad;
                    }
                }
    std::printf("checked %ld mismatches %ld\n", checked, bad);
    return bad != 0;
}
"""


def test_round_robin_makespan_matches_a_per_cta_count(tmp_path):
    src = os.path.join(tmp_path, "plan_check.cpp")
    exe = os.path.join(tmp_path, "plan_check")
    with open(src, "w") as f:
        f.write(HARNESS)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", CSRC, "-o", exe, src])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout
    assert "mismatches 0" in r.stdout
