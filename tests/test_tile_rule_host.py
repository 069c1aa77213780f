"""The kernels' tile rule (``tile_class`` in csrc/pp_meta.cuh, shared by every kernel and by pp_meta_tiles), compiled
for the host with g++ and compared with the oracle's brute-force tile classes over many small tile shapes, so that
tile boundaries fall on every kind of position (inside the prefix, on a response start, past the group's end).

The GPU tests check the same rule at the kernels' 128 x 128 tiles through pp_meta_tiles; here the shapes are small
and varied, and no GPU is needed. The program receives the group lengths and writes the non-empty tiles as packed
(q_row0, kv_row0, class) triples, with s0first and s0last formed as the schedule builder forms them."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from tests.conftest import random_groups

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "shared_prefix_packed_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "pp_meta.cuh"
// stdin: bm bn G, then per group: P k S_1 .. S_k. stdout: non-empty tiles "q_row0 kv_row0 class".
int main() {
    int bm, bn, G;
    if (std::scanf("%d %d %d", &bm, &bn, &G) != 3) return 2;
    int o = 0;
    for (int g = 0; g < G; ++g) {
        int P, k;
        if (std::scanf("%d %d", &P, &k) != 2) return 2;
        std::vector<int> start(k), len(k);
        int L = P;
        for (int i = 0; i < k; ++i) {
            if (std::scanf("%d", &len[i]) != 1) return 2;
            start[i] = L;
            L += len[i];
        }
        auto seg_start = [&](int x) {              // in-group start of the segment holding offset x (x < L)
            if (x < P) return 0;
            for (int i = 0; i < k; ++i)
                if (x >= start[i] && x < start[i] + len[i]) return start[i];
            return -1;
        };
        for (int x0 = 0; x0 < L; x0 += bm) {
            const int xm = (x0 + bm < L ? x0 + bm : L) - 1;
            const int s0first = x0 >= P ? seg_start(x0) : P;
            const int s0last = xm >= P ? seg_start(xm) : 0;
            for (int y0 = 0; y0 < L; y0 += bn) {
                const int c = pp::tile_class(x0, bm, y0, bn, L, P, s0first, s0last);
                if (c != pp::TILE_EMPTY) std::printf("%d %d %d\n", o + x0, o + y0, c);
            }
        }
        o += L;
    }
    return 0;
}
"""


@pytest.fixture(scope="module")
def tile_rule_exe(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ unavailable")
    d = tmp_path_factory.mktemp("tile_rule")
    src = d / "tile_rule.cpp"
    src.write_text(PROGRAM)
    exe = d / "tile_rule"
    subprocess.run([gxx, "-std=c++17", "-O1", "-D__host__=", "-D__device__=", "-D__forceinline__=inline",
                    f"-I{CSRC}", str(src), "-o", str(exe)], check=True, capture_output=True, text=True)
    return str(exe)


def _rule_tiles(exe, P, S, bm, bn):
    lines = [f"{bm} {bn} {len(P)}"] + [" ".join(str(x) for x in [p, len(ss)] + list(ss)) for p, ss in zip(P, S)]
    out = subprocess.run([exe], input="\n".join(lines) + "\n", capture_output=True, text=True, check=True).stdout
    return sorted(tuple(int(v) for v in ln.split()) for ln in out.splitlines())


SHAPES = [(1, 1), (2, 3), (4, 4), (5, 2), (3, 8), (8, 8), (7, 16), (16, 5)]
CASES = [
    ([3], [[2, 0, 3]]),
    ([0], [[5, 7]]),
    ([9], [[]]),
    ([6], [[0, 0, 7]]),
    ([1], [[1] * 9]),
    ([8], [[8, 8]]),
    ([7, 9, 1], [[1, 15], [3], [0]]),
    ([0, 0], [[0], [4]]),
]


@pytest.mark.parametrize("bm,bn", SHAPES)
def test_tile_rule_matches_bruteforce_on_edge_cases(tile_rule_exe, bm, bn):
    for P, S in CASES:
        assert _rule_tiles(tile_rule_exe, P, S, bm, bn) == oracle.tile_classes_bruteforce(P, S, bm, bn), (P, S)


@pytest.mark.parametrize("seed", range(6))
def test_tile_rule_matches_bruteforce_on_random_groups(tile_rule_exe, seed):
    rng = np.random.default_rng(900 + seed)
    P, S = random_groups(rng, 1 + seed % 4, 40, 30, 5)
    for bm, bn in SHAPES:
        assert _rule_tiles(tile_rule_exe, P, S, bm, bn) == oracle.tile_classes_bruteforce(P, S, bm, bn), (P, S, bm, bn)
