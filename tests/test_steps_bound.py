"""``bwd_steps_bound`` (csrc/pp_meta.cuh), compiled for the host with g++: it must bound the backward steps of one kv
head of any batch of T tokens, because the backward keeps dS tiles only where that bound fits the int32 counters
of the schedule builder. The steps of a batch are its non-empty (key tile, query tile) pairs times r, taken here
from the oracle's tile classes, which the schedule's own key ranges are checked against on the GPU."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import workloads as W
from tests.conftest import random_groups

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "shared_prefix_packed_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include "pp_meta.cuh"
int main() {   // stdin: lines "T r"; stdout: the bound for each
    long long T;
    int r;
    while (std::scanf("%lld %d", &T, &r) == 2) std::printf("%lld\n", (long long)pp::bwd_steps_bound(T, r));
    return 0;
}
"""


@pytest.fixture(scope="module")
def bound():
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ unavailable")
    import tempfile
    d = tempfile.mkdtemp()
    src = os.path.join(d, "bound.cpp")
    with open(src, "w") as f:
        f.write(PROGRAM)
    exe = os.path.join(d, "bound")
    subprocess.run([gxx, "-std=c++17", "-D__host__=", "-D__device__=", "-D__forceinline__=inline", f"-I{CSRC}",
                    src, "-o", exe], check=True, capture_output=True, text=True)

    def f(pairs):
        inp = "".join(f"{T} {r}\n" for T, r in pairs)
        out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout.split()
        return [int(x) for x in out]
    return f


def _steps(P, S, r):
    return r * len(oracle.tile_classes(P, S, 128, 128))


def test_bound_holds_on_random_and_extreme_layouts(bound):
    rng = np.random.default_rng(31)
    layouts = [random_groups(rng, int(rng.integers(1, 7)), 3000, 2000, 6) for _ in range(40)]
    layouts += [([5000], [[]]), ([128 * 40], [[]]), ([0], [[1] * 300]), ([1] * 200, [[]] * 200),
                ([129] * 30, [[]] * 30), ([2000], [[1] * 50]), ([0], [[0]])]
    for r in (1, 4, 7):
        T = [W.packed_total(P, S) for P, S in layouts]
        got = bound([(t, r) for t in T])
        for (P, S), t, b in zip(layouts, T, got):
            assert b >= _steps(P, S, r), (P, S, r)


def test_bound_is_tight_for_one_long_group(bound):
    """One prefix-only group of n whole tiles has exactly n (n + 1) / 2 pairs; the bound adds only T."""
    for n in (1, 7, 40):
        T = 128 * n
        assert _steps([T], [[]], 1) == n * (n + 1) // 2
        assert bound([(T, 1)]) == [T + n * (n + 1) // 2]


def test_kept_ds_stays_on_for_every_workload(bound):
    """The guard only matters for batches of millions of tokens: every workload here keeps its dS tiles."""
    for name, w in W.WORKLOADS.items():
        P, S = W.group_lengths(name)
        T = W.packed_total(P, S)
        r = w.num_heads_q // w.num_heads_kv
        assert bound([(T, r)])[0] <= 2 ** 31 - 1, name
    assert bound([(4_200_000, 4)])[0] > 2 ** 31 - 1         # about where it turns the kept-dS path off at r = 4
