"""The order in which a persistent kernel's CTAs take their items (``alt_item`` in csrc/pp_meta.cuh), checked on the
host by compiling the header with g++: over every grid size and item count tried, the CTAs together take every item
exactly once, each CTA's loop ends, and each round deals the next block of grid-size items."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "shared_prefix_packed_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "pp_meta.cuh"
// The kernels' loop: for (int rnd = 0, item = b; item < n; item = alt_item(++rnd, b, g)) { ... }
int main() {
    int bad = 0;
    for (int g : {1, 2, 3, 7, 148, 296}) {
        for (int n = 0; n <= 5 * g + 3; ++n) {
            std::vector<int> seen(n, 0);
            for (int b = 0; b < g; ++b) {
                int steps = 0;
                for (int rnd = 0, item = b; item < n; item = pp::alt_item(++rnd, b, g)) {
                    if (item < rnd * g || item >= (rnd + 1) * g) ++bad;     // round rnd deals [rnd g, rnd g + g)
                    ++seen[item];
                    if (++steps > n) { ++bad; break; }                       // the loop must end
                }
            }
            for (int i = 0; i < n; ++i) bad += seen[i] != 1;                  // every item exactly once
        }
    }
    // items of decreasing cost: the alternating deal keeps the busiest CTA closer to the mean than round-robin
    const int g = 148, n = 12 * g + 37;
    std::vector<long> alt(g, 0), rr(g, 0);
    for (int b = 0; b < g; ++b) {
        for (int rnd = 0, item = b; item < n; item = pp::alt_item(++rnd, b, g)) alt[b] += n - item;
        for (int item = b; item < n; item += g) rr[b] += n - item;
    }
    long amax = 0, rmax = 0;
    for (int b = 0; b < g; ++b) { amax = alt[b] > amax ? alt[b] : amax; rmax = rr[b] > rmax ? rr[b] : rmax; }
    if (!(amax < rmax)) ++bad;
    std::printf("%d\n", bad);
    return bad != 0;
}
"""


def test_alternating_item_order_covers_every_item_once(tmp_path):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ unavailable")
    src = tmp_path / "order.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "order"
    subprocess.run([gxx, "-std=c++17", "-O1", "-D__host__=", "-D__device__=", "-D__forceinline__=inline",
                    f"-I{CSRC}", str(src), "-o", str(exe)], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "0", out.stdout + out.stderr
