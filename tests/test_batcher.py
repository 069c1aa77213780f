"""Parity of the native batch planner (pp_plan_batches, host-only, so this runs without a GPU) with the oracle:
bit-exact on random inputs, including ties, zero-token groups and groups over the capacity."""
import numpy as np
import pytest

import oracle


def test_plan_batches_matches_oracle():
    from shared_prefix_packed_b200 import pp_plan_batches
    rng = np.random.default_rng(11)
    for it in range(500):
        G = int(rng.integers(0, 300))
        toks = rng.integers(0, 4000, size=G)
        if it % 3 == 0:
            toks = (toks // 500) * 500                       # many ties
        cap = int(rng.integers(1, 20000))
        srt = bool(it % 2)
        assert pp_plan_batches(toks, cap, srt) == oracle.plan_batches(toks.tolist(), cap, srt)


def test_plan_batches_dpo_sized():
    import workloads as W
    from shared_prefix_packed_b200 import pp_plan_batches
    P, S = W.group_lengths("grpo")
    toks = [p + sum(ss) for p, ss in zip(P, S)]
    for cap in (8192, 16384, 65536):
        assert pp_plan_batches(toks, cap, True) == oracle.plan_batches(toks, cap, True)


def test_plan_batches_rejects_bad_input():
    from shared_prefix_packed_b200 import pp_plan_batches
    with pytest.raises(ValueError):
        pp_plan_batches([3, -1], 10)
    with pytest.raises(ValueError):
        pp_plan_batches([3, 1], 0)
    assert pp_plan_batches([], 5) == ([], [], 0)
