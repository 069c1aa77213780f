"""GPU parity of pp_build_meta: position ids and the canonical tile sets bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import random_case
from tests.schedule_checks import check_backward_schedule, check_forward_schedule

pytestmark = pytest.mark.gpu


def _batch(P, S, hq=4, hkv=2, d=128):
    from shared_prefix_packed_b200 import PackedBatch
    return PackedBatch(P, S, hq, hkv, d)


CASES = [
    ([3], [[2, 0, 3]]),                       # hand-worked example
    ([0], [[5, 7]]),                          # no prefix: block-diagonal causal
    ([300], [[]]),                              # prefix only (k = 0)
    ([200], [[0, 0, 129]]),                   # zero-length responses
    ([1], [[1] * 40]),                        # many tiny responses
    ([128], [[128, 128]]),                    # every boundary on a tile boundary
    ([127, 129, 1], [[1, 255], [3], [0]]),    # ragged tails, tiles straddling groups
]


@pytest.mark.parametrize("P,S", CASES)
def test_meta_small_cases(P, S):
    b = _batch(P, S)
    torch.cuda.synchronize()
    assert np.array_equal(b.pos_ids[: b.T].cpu().numpy(), oracle.position_ids(P, S))
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD, pp_get_status
    assert b.tiles(PP_PASS_FWD) == oracle.tile_classes(P, S, 128, 128)
    assert b.tiles(PP_PASS_BWD) == oracle.tile_classes(P, S, 128, 128)
    pp_get_status()


@pytest.mark.parametrize("seed", range(12))
def test_meta_random_groups(seed):
    P, S = random_case(seed, 1 + seed % 5, 700, 500, 6)
    b = _batch(P, S)
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD
    assert np.array_equal(b.pos_ids[: b.T].cpu().numpy(), oracle.position_ids(P, S))
    assert b.tiles(PP_PASS_FWD) == oracle.tile_classes(P, S, 128, 128)
    assert b.tiles(PP_PASS_BWD) == oracle.tile_classes(P, S, 128, 128)


@pytest.mark.parametrize("name", ["tiny", "dpo", "grpo", "longprefix", "hetero"])
def test_meta_full_workloads(name):
    P, S = W.group_lengths(name)
    w = W.WORKLOADS[name]
    b = _batch(P, S, w.num_heads_q, w.num_heads_kv, w.head_dim)
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD
    assert np.array_equal(b.pos_ids[: b.T].cpu().numpy(), oracle.position_ids(P, S))
    assert b.tiles(PP_PASS_FWD) == oracle.tile_classes(P, S, 128, 128)
    assert b.tiles(PP_PASS_BWD) == oracle.tile_classes(P, S, 128, 128)


SCHED_CASES = CASES + [([2100], [[700, 900]]), ([4000, 10], [[3000, 3000, 3000], [5]])]


@pytest.mark.parametrize("P,S", SCHED_CASES)
def test_schedule_small_cases(P, S):
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD
    b = _batch(P, S)
    check_forward_schedule(P, S, b.schedule(PP_PASS_FWD))
    check_backward_schedule(P, S, b.schedule(PP_PASS_BWD))


@pytest.mark.parametrize("seed", range(8))
def test_schedule_random_groups(seed):
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD
    P, S = random_case(500 + seed, 1 + seed % 5, 3000, 1500, 6)
    b = _batch(P, S)
    check_forward_schedule(P, S, b.schedule(PP_PASS_FWD))
    check_backward_schedule(P, S, b.schedule(PP_PASS_BWD))


@pytest.mark.parametrize("name", ["tiny", "dpo", "grpo", "longprefix", "hetero"])
def test_schedule_full_workloads(name):
    """The executed schedule of every workload, in the launch configuration the bench times."""
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD
    P, S = W.group_lengths(name)
    w = W.WORKLOADS[name]
    b = _batch(P, S, w.num_heads_q, w.num_heads_kv, w.head_dim)
    check_forward_schedule(P, S, b.schedule(PP_PASS_FWD))
    check_backward_schedule(P, S, b.schedule(PP_PASS_BWD))


def test_device_detects_inconsistent_descriptors():
    from shared_prefix_packed_b200 import _lib
    groups = torch.tensor([[4, 2]], dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, 3, 5, 9], dtype=torch.int32, device="cuda")    # prefix segment 3 != prefix_len 4
    meta = torch.empty(_lib.pp_meta_bounds(1, 3, 9, 4, 2), dtype=torch.uint8, device="cuda")
    pos = torch.empty(9, dtype=torch.int32, device="cuda")
    _lib.pp_build_meta(groups, cu, 9, 4, 2, pos, meta)
    with pytest.raises(_lib.PPError, match="DEVICE_INPUT"):
        _lib.pp_get_status()
    cu_bad = torch.tensor([0, 4, 3, 9], dtype=torch.int32, device="cuda")  # not monotone
    _lib.pp_build_meta(groups, cu_bad, 9, 4, 2, pos, meta)
    with pytest.raises(_lib.PPError, match="DEVICE_INPUT"):
        _lib.pp_get_status()
    _lib.pp_get_status()   # the word was cleared


def test_host_validation_rejects_bad_arguments():
    from shared_prefix_packed_b200 import _lib
    groups = torch.tensor([[4, 1]], dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, 4, 9], dtype=torch.int32, device="cuda")
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    pos = torch.empty(9, dtype=torch.int32, device="cuda")
    with pytest.raises(_lib.PPError, match="WORKSPACE"):
        _lib.pp_build_meta(groups, cu, 9, 4, 2, pos, small)
    with pytest.raises(_lib.PPError, match="INVALID_ARG"):
        _lib.pp_build_meta(groups, cu, 9, 4, 3, pos, small)
