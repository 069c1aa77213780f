"""GPU parity of pp_rope against the fp64 oracle RoPE: within 2 bf16 ulps of max(|y_ref|, 2^-6) per element."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import bf16_ulp, random_case, to_np64

pytestmark = pytest.mark.gpu


def _check(P, S, hq, hkv, d, dtype, seed, inverse=False):
    from shared_prefix_packed_b200 import PackedBatch
    b = PackedBatch(P, S, hq, hkv, d)
    inp = W.make_inputs("dpo", P, S, seed=seed, with_dout=False, heads=(hq, hkv, d), dtype=dtype)
    q, k = inp["q"].cuda(), inp["k"].cuda()
    b.rope(q, k, inverse=inverse)
    pos = oracle.position_ids(P, S)
    for got, x in ((q, inp["q"]), (k, inp["k"])):
        ref = oracle.rope(to_np64(x), pos, inverse=inverse)
        err = np.abs(to_np64(got) - ref)
        if dtype == "bf16":
            bound = 2 * bf16_ulp(np.maximum(np.abs(ref), 2.0 ** -6))
        else:
            bound = 1e-5 * np.maximum(np.abs(ref), 2.0 ** -6)
        assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("d", [64, 128])
def test_rope_random(seed, d):
    P, S = random_case(seed, 3, 400, 300, 4)
    _check(P, S, 8, 2, d, "bf16", seed)


def test_rope_fp32_and_inverse():
    P, S = random_case(9, 2, 300, 200, 3)
    _check(P, S, 4, 4, 64, "fp32", 9)
    _check(P, S, 4, 2, 128, "bf16", 10, inverse=True)


def test_rope_full_dpo():
    P, S = W.group_lengths("dpo")
    _check(P, S, 32, 8, 128, "bf16", 1002)
