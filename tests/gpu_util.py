"""Helpers shared by the GPU tests (device buffers via torch; every computation goes through libpp)."""
import numpy as np
import torch

import workloads as W


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def to_np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def random_case(seed, n_groups, pmax, smax, kmax, allow_zero=True):
    rng = np.random.default_rng(seed)
    P, S = [], []
    lo = 0 if allow_zero else 1
    for _ in range(n_groups):
        P.append(int(rng.integers(lo, pmax + 1)))
        k = int(rng.integers(lo, kmax + 1))
        S.append([int(rng.integers(lo, smax + 1)) for _ in range(k)])
    if W.packed_total(P, S) == 0:
        P[0] = 1
    return P, S


def sample_rows(prefix_lens, suffix_lens, n, seed=0):
    """Rows spread over groups, always including each group's first/last row and segment boundaries."""
    rng = np.random.default_rng(seed)
    rows = set()
    off = 0
    for p, ss in zip(prefix_lens, suffix_lens):
        L = p + sum(ss)
        if L:
            rows.update([off, off + L - 1])
            b = off
            for seg in [p] + list(ss):
                if seg:
                    rows.update([b, b + seg - 1])
                b += seg
        off += L
    T = off
    extra = rng.integers(0, T, size=max(0, n - len(rows)))
    rows.update(int(x) for x in extra)
    return sorted(rows)
