"""The kernels' bounded waits end in an error status, not a hang: pp_selftest_bounded_wait runs the attention
kernels' own wait code on an mbarrier that nothing arrives on, with a short limit. The test checks that the wait
gives up after about that limit, that pp_get_status reports PP_ERR_DEVICE_TIMEOUT once, and that the context stays
usable: a forward pass right after returns PP_OK and matches the oracle. No fault, trap or endless loop is used."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ms", [5, 50])
def test_bounded_wait_times_out_and_the_context_survives(limit_ms):
    from shared_prefix_packed_b200 import PackedBatch, _lib
    _lib.pp_get_status()                                            # start from a clear error word
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    _lib.pp_selftest_bounded_wait(limit_ms * 1_000_000, waited)
    with pytest.raises(_lib.PPError, match="DEVICE_TIMEOUT"):
        _lib.pp_get_status()
    ns = int(waited.item())
    assert limit_ms * 1e6 <= ns < limit_ms * 1e6 + 200e6, ns         # gave up after the limit, not much later
    _lib.pp_get_status()                                            # the word was cleared
    P, S = [300, 40], [[200, 90], [17]]
    inp = W.make_inputs("dpo", P, S, seed=9, with_dout=False, heads=(4, 2, 128))
    b = PackedBatch(P, S, 4, 2, 128)
    o, lse = b.forward(*(inp[x].cuda() for x in "qkv"))
    assert _lib.pp_get_status() == _lib.PP_OK
    _, L_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], P, S)
    assert np.max(np.abs(lse.cpu().double().numpy() - L_ref)) <= 1e-3


def test_bounded_wait_rejects_bad_limits():
    from shared_prefix_packed_b200 import _lib
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    for bad in (0, 999, 3_000_000_000):
        with pytest.raises(_lib.PPError, match="INVALID_ARG"):
            _lib.pp_selftest_bounded_wait(bad, waited)
