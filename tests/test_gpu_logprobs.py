"""GPU parity of pp_response_logprobs against the fp64 oracle (oracle/response_logprobs.py).

Tolerance: 1e-4 absolute on each log-probability. The kernel sums exp2 terms in fp32 (each from ex2.approx, relative
error about 2^-22) and adds one fp32 logit; at |log-sum-exp| of about 20 (V = 151,936 and logits of std 4) that is
about 1e-6, so 1e-4 leaves a wide margin while still catching a wrong row, a wrong token or a missing temperature.
Rows that no row predicts (prefix rows, a response's first token when P = 0) must be exactly 0.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _run(P, S, V, dtype, temperature, seed):
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    logits, ids = W.make_logits(P, S, vocab=V, seed=seed, dtype=dtype)
    b = PackedBatch(P, S, 4, 2, 128)
    lp = b.response_logprobs(logits.cuda(), ids.cuda(), temperature=temperature)
    pp_get_status()
    return logits, ids, lp.cpu().double().numpy()


CASES = [
    ([3], [[2, 0, 3]]),
    ([0], [[5, 1]]),              # no prefix: the first tokens have no predicting row
    ([4], [[]]),                  # prefix only: nothing to score
    ([1], [[1] * 9]),
    ([7, 0, 2], [[3, 1], [4], [0, 2]]),
    ([130], [[129, 1, 300]]),
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("V,dtype,temperature", [(1, "bf16", 1.0), (7, "fp32", 0.6), (1000, "bf16", 1.0),
                                                 (32771, "bf16", 0.7), (4099, "fp32", 1.3)])
def test_logprobs_small(case, V, dtype, temperature):
    P, S = CASES[case]
    logits, ids, got = _run(P, S, V, dtype, temperature, 3000 + case)
    want, valid = oracle.response_logprobs(logits, ids, P, S, temperature=temperature)
    assert np.all(got[~valid] == 0.0)
    if valid.any():
        err = np.max(np.abs(got[valid] - want[valid]))
        assert err <= TOL, err


def test_logprobs_full_layout_sampled_rows():
    """The dpo layout (T = 17,801) at the read-out's bench vocabulary (151,936): sampled rows against the oracle,
    every response first token among them, and properties of all rows."""
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    P, S = W.group_lengths("dpo")
    V = W.LOGPROB_VOCAB
    logits, ids = W.make_logits(P, S, vocab=V, seed=2001)
    b = PackedBatch(P, S, 32, 8, 128)
    lp = b.response_logprobs(logits.cuda(), ids.cuda(), temperature=0.9).cpu().double().numpy()
    pp_get_status()
    src = oracle.response_source_rows(P, S)
    firsts = [int(x) for x in np.nonzero((src >= 0) & (src != np.arange(len(src)) - 1))[0]]
    rng = np.random.default_rng(7)
    rows = sorted(set(firsts) | set(int(r) for r in rng.choice(np.nonzero(src >= 0)[0], 200, replace=False)))
    want, valid = oracle.response_logprobs_rows(logits, ids, P, S, rows, temperature=0.9)
    assert valid.all()
    assert np.max(np.abs(lp[rows] - want)) <= TOL
    assert np.all(lp[src < 0] == 0.0)
    assert np.all(np.isfinite(lp)) and np.all(lp[src >= 0] < 0)


@pytest.mark.parametrize("V,dtype", [(1000, "bf16"), (4099, "fp32"), (32771, "bf16")])
def test_logprobs_negative_infinity_entries(V, dtype):
    """Masked vocabulary entries (-inf logits): a padded tail of every row, scattered entries, whole 16-byte vectors
    and the scalar head and tail. They add nothing to the sum; a token whose own logit is -inf gets -inf."""
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    P, S = [130], [[129, 1, 300]]
    logits, ids = W.make_logits(P, S, vocab=V, seed=77, dtype=dtype)
    rng = np.random.default_rng(78)
    ninf = float("-inf")
    logits[:, V - 37:] = ninf                                   # padded tail of every row
    logits[torch.from_numpy(rng.random(logits.shape) < 0.3)] = ninf   # 30 % scattered
    logits[:, 8:64] = ninf                                      # whole vectors in a row
    logits[:, :3] = ninf                                        # part of the head
    src = oracle.response_source_rows(P, S)
    resp = np.nonzero(src >= 0)[0]
    ids[int(resp[5])] = V - 1                                   # a token whose logit is -inf
    ids[int(resp[9])] = 10
    b = PackedBatch(P, S, 4, 2, 128)
    got = b.response_logprobs(logits.cuda(), ids.cuda(), temperature=0.8).cpu().double().numpy()
    pp_get_status()
    want, valid = oracle.response_logprobs(logits, ids, P, S, temperature=0.8)
    assert not np.isnan(got).any()
    assert np.all(got[~valid] == 0.0)
    inf_rows = valid & np.isneginf(want)
    assert inf_rows.sum() >= 2 and np.all(np.isneginf(got[inf_rows]))
    fin = valid & np.isfinite(want)
    assert np.max(np.abs(got[fin] - want[fin])) <= TOL


def test_logprobs_bad_token_is_reported():
    from shared_prefix_packed_b200 import PackedBatch, PPError, pp_get_status
    P, S = [3], [[4]]
    logits, ids = W.make_logits(P, S, vocab=50, seed=1)
    ids[5] = 50                                       # out of range, at a response row
    b = PackedBatch(P, S, 4, 2, 128)
    lp = b.response_logprobs(logits.cuda(), ids.cuda())
    with pytest.raises(PPError, match="DEVICE_INPUT"):
        pp_get_status()
    got = lp.cpu().numpy()
    assert np.isnan(got[5]) and np.isfinite(np.delete(got, 5)).all()
