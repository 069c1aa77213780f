"""Empty inputs on the GPU: a batch with no tokens at all, and empty groups among non-empty ones.

A batch whose groups all have zero length (P = 0 and only zero-length responses, or no responses) has T = 0: the
metadata build must succeed with empty tile sets and schedules, and every other call must accept the empty tensors
and return without error. Empty groups between non-empty ones contribute no tiles and must not disturb the others:
forward and backward are compared with the fp64 oracle as in the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import bf16_ulp, to_np64

pytestmark = pytest.mark.gpu

EMPTY = [
    ([0], [[0, 0]]),          # one group: no prefix, two zero-length responses
    ([0, 0], [[], [0]]),      # two groups, neither with a token
]


@pytest.mark.parametrize("P,S", EMPTY)
def test_empty_batch_every_call(P, S):
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD, PackedBatch, pp_get_status
    hq, hkv, d = 4, 2, 128
    b = PackedBatch(P, S, hq, hkv, d)
    assert b.T == 0 == W.packed_total(P, S)
    assert b.tiles(PP_PASS_FWD) == [] == oracle.tile_classes(P, S, 128, 128)
    assert b.tiles(PP_PASS_BWD) == []
    assert b.schedule(PP_PASS_FWD) == [] and b.schedule(PP_PASS_BWD) == []
    q = torch.empty(0, hq, d, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(0, hkv, d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    b.rope(q, k)
    o, lse = b.forward(q, k, v)
    assert o.shape == (0, hq, d) and lse.shape == (hq, 0)
    dq, dk, dv = b.backward(q, k, v, o, lse, torch.empty_like(o))
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape
    lp = b.response_logprobs(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"),
                             torch.empty(0, dtype=torch.int32, device="cuda"))
    assert lp.shape == (0,)
    pp_get_status()


def test_empty_groups_among_non_empty():
    """Groups with no token before, between and after non-empty ones (one of them a long prefix whose key tiles
    are split over chunks): O, LSE and the gradients match the oracle."""
    from shared_prefix_packed_b200 import PP_PASS_BWD, PP_PASS_FWD, PackedBatch, pp_get_status
    P = [0, 3, 0, 1100, 0]
    S = [[0], [2, 0], [], [1, 129, 0], [0, 0]]
    hq, hkv, d = 4, 2, 128
    inp = W.make_inputs("dpo", P, S, seed=911, with_dout=True, heads=(hq, hkv, d))
    b = PackedBatch(P, S, hq, hkv, d)
    assert np.array_equal(b.pos_ids[: b.T].cpu().numpy(), oracle.position_ids(P, S))
    assert b.tiles(PP_PASS_FWD) == oracle.tile_classes(P, S, 128, 128)
    assert b.tiles(PP_PASS_BWD) == oracle.tile_classes(P, S, 128, 128)
    q, k, v, do = (inp[x].cuda() for x in ("q", "k", "v", "dout"))
    o, lse = b.forward(q, k, v)
    dq, dk, dv = b.backward(q, k, v, o, lse, do)
    pp_get_status()
    O_ref, L_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], P, S)
    assert float(np.max(np.abs(to_np64(o) - O_ref) - 0.5 * bf16_ulp(O_ref))) <= 1e-2
    assert float(np.max(np.abs(to_np64(lse) - L_ref))) <= 1e-3
    for got, want in zip((dq, dk, dv), oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S)):
        assert np.linalg.norm(to_np64(got) - want) / np.linalg.norm(want) <= 1e-2
