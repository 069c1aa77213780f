"""Pins for the oracle's layout, grouped position ids, mask and tile classes (CPU only)."""
import os

import numpy as np
import pytest

import oracle
from oracle.packed_attention import FULL, PARTIAL
from tests.conftest import random_groups

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def test_position_ids_golden():
    """Hand-worked examples of the page's rule ("prefix_grouper_utils.py" §1)."""
    for ln in _read("position_ids.txt"):
        lhs, rhs = ln.split("|")
        p, ss = lhs.split(";")
        p = int(p)
        ss = [int(x) for x in ss.split(",") if x.strip()]
        want = [int(x) for x in rhs.split()]
        got = oracle.position_ids([p], [ss]).tolist()
        assert got == want, (ln, got)


def test_position_ids_multi_group_concatenates():
    P, S = [3, 0, 2], [[2, 0, 3], [2], [1]]
    pos = oracle.position_ids(P, S).tolist()
    assert pos == [0, 1, 2, 3, 4, 3, 4, 5] + [0, 1] + [0, 1, 2]


def test_position_id_equals_allowed_count_minus_one():
    """Independent pin: under the mask, row i sees exactly pos(i)+1 keys (each suffix continues the prefix)."""
    rng = np.random.default_rng(7)
    for _ in range(30):
        P, S = random_groups(rng, int(rng.integers(1, 4)), 9, 7, 4)
        m = oracle.allowed_mask(P, S)
        pos = oracle.position_ids(P, S)
        assert np.array_equal(m.sum(axis=1) - 1, pos)


def test_mask_properties_and_pair_count():
    rng = np.random.default_rng(11)
    for _ in range(40):
        P, S = random_groups(rng, int(rng.integers(1, 4)), 10, 8, 4)
        m = oracle.allowed_mask(P, S)
        lay = oracle.layout_of(P, S)
        assert m.sum() == oracle.allowed_pair_count(P, S)
        assert np.all(np.diag(m))                       # every row sees itself: no empty row, finite LSE
        assert not np.any(np.triu(m, 1))                # causal in packed order
        same_group = lay.group_of[:, None] == lay.group_of[None, :]
        assert not np.any(m & ~same_group)              # never across groups
        sib = (lay.seg_of[:, None] != lay.seg_of[None, :]) & (lay.seg_of[None, :] != 0) & same_group
        assert not np.any(m & sib)                      # never a sibling response
        _, _, cnt = oracle.allowed_pairs_per_row(lay)
        assert np.array_equal(cnt, m.sum(axis=1))


def test_tile_classes_golden():
    want = sorted(tuple(int(x) for x in ln.split()) for ln in _read("tile_classes.txt"))
    assert oracle.tile_classes_bruteforce([2], [[2, 2]], 2, 2) == want
    assert oracle.tile_classes([2], [[2, 2]], 2, 2) == want


@pytest.mark.parametrize("BM,BN", [(2, 2), (4, 2), (3, 5), (8, 8), (16, 8)])
def test_tile_classes_interval_equals_bruteforce(BM, BN):
    rng = np.random.default_rng(100 + BM * 7 + BN)
    for _ in range(12):
        P, S = random_groups(rng, int(rng.integers(1, 4)), 20, 14, 4)
        assert oracle.tile_classes(P, S, BM, BN) == oracle.tile_classes_bruteforce(P, S, BM, BN)


def test_tiles_cover_allowed_set():
    """FULL and PARTIAL tiles together cover every allowed pair; FULL tiles hold only allowed pairs."""
    rng = np.random.default_rng(5)
    for _ in range(10):
        P, S = random_groups(rng, 3, 20, 12, 3)
        m = oracle.allowed_mask(P, S)
        T = m.shape[0]
        cov = np.zeros_like(m)
        for q0, k0, c in oracle.tile_classes(P, S, 4, 4):
            blk = m[q0:q0 + 4, k0:k0 + 4]
            if c == FULL:
                assert blk.shape == (4, 4) and blk.all()
            else:
                assert c == PARTIAL and blk.any() and not (blk.shape == (4, 4) and blk.all())
            cov[q0:q0 + 4, k0:k0 + 4] = True
        assert not np.any(m & ~cov)
        assert T == oracle.layout_of(P, S).T
