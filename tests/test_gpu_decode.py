"""GPU parity of pp_decode_attn (one decoding step over a group-contiguous KV cache) against the fp64 oracle.

The query of a response is its newest token, the last row of its segment in the packed cache, so the oracle is the
packed forward evaluated at those rows (oracle.attention_forward_rows with the decode queries placed there).
Bounds as for the forward: O max-abs error beyond its bf16 rounding <= 1e-2, LSE max-abs error <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import bf16_ulp, random_case, to_np64

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
LSE_TOL = 1e-3


def _decode_case(P, S, hq, hkv, seed):
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    inp = W.make_inputs("grpo", P, S, seed=seed, with_dout=False, heads=(hq, hkv, 128))
    T = W.packed_total(P, S)
    cu = W.segment_bounds(P, S)
    n_resp = sum(len(ss) for ss in S)
    # response ordinal -> its segment's last packed row (None for an empty response)
    last_rows = []
    s = 0
    for ss in S:
        s += 1                                             # the group's prefix segment
        for _ in ss:
            last_rows.append(int(cu[s + 1]) - 1 if cu[s + 1] > cu[s] else None)
            s += 1
    rng = np.random.default_rng(seed + 7)
    qd = torch.from_numpy(rng.standard_normal((n_resp, hq, 128), dtype=np.float32)).to(torch.bfloat16)
    b = PackedBatch(P, S, hq, hkv, 128)
    o, lse = b.decode(qd.cuda(), inp["k"].cuda(), inp["v"].cuda())
    pp_get_status()
    return inp, qd, last_rows, T, o.cpu(), lse.cpu()


def _check(P, S, hq, hkv, seed):
    inp, qd, last_rows, T, o, lse = _decode_case(P, S, hq, hkv, seed)
    valid = [i for i, r in enumerate(last_rows) if r is not None]
    if valid:
        rows = [last_rows[i] for i in valid]
        qp = torch.zeros((T, hq, 128), dtype=torch.bfloat16)
        qp[rows] = qd[valid]
        O_ref, L_ref = oracle.attention_forward_rows(qp, inp["k"], inp["v"], P, S, rows)
        err_o = np.max(np.abs(to_np64(o[valid]) - O_ref) - 0.5 * bf16_ulp(O_ref))
        err_l = np.max(np.abs(lse[:, valid].double().numpy() - L_ref))
        assert err_o <= O_TOL and err_l <= LSE_TOL, (err_o, err_l)
    assert torch.isfinite(o.float()).all()


SMALL = [
    ([3], [[2, 5, 3]]),
    ([0], [[130, 77]]),             # no prefix
    ([513], [[200, 300, 64]]),
    ([1], [[1] * 40]),              # 40 responses share one prefix chunk: several query passes per chunk
    ([127, 129, 1], [[1, 255], [3], [64, 65]]),
    ([700], [[1]]),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("heads", [(8, 2), (7, 1), (4, 4)])
def test_decode_small(case, heads):
    P, S = SMALL[case]
    _check(P, S, heads[0], heads[1], 500 + case)


@pytest.mark.parametrize("seed", range(4))
def test_decode_random(seed):
    P, S = random_case(600 + seed, 1 + seed % 4, 900, 400, 9)
    S = [[max(1, s) for s in ss] for ss in S]            # every decoding response holds at least its new token
    _check(P, S, 8, 2, seed)


def test_decode_full_grpo_cache():
    """The grpo layout as the cache (T = 81,860, 16 groups x 8 responses), all 128 queries, 32/8 heads."""
    P, S = W.group_lengths("grpo")
    _check(P, S, 32, 8, 2024)


def test_decode_rejects_inconsistent_bounds():
    from shared_prefix_packed_b200 import PackedBatch, PPError, _lib, pp_get_status
    P, S = [5], [[3, 2]]
    b = PackedBatch(P, S, 4, 2, 128)
    T = b.T
    k = torch.zeros((T, 2, 128), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(4, 2, dtype=torch.float32, device="cuda")
    ws = torch.empty(_lib.pp_decode_workspace_bytes(b.groups.cpu(), b.cu_seqlens.cpu(), 4), dtype=torch.uint8,
                     device="cuda")
    bad = b.cu_seqlens.clone()
    bad[-1] = T + 5                                        # bounds past the cache
    _lib.pp_decode_attn(q, k, k, b.groups, bad, o, lse, ws)
    with pytest.raises(PPError, match="DEVICE_INPUT"):
        pp_get_status()
    assert torch.isnan(lse).all()


EMPTY_RESP = [
    ([5], [[0, 3, 0]]),             # zero-length responses: their query sees the prefix alone
    ([0, 130], [[0, 2], [0]]),      # no prefix and no rows: no key at all; a prefix of two chunks alone
]


@pytest.mark.parametrize("case", range(len(EMPTY_RESP)))
@pytest.mark.parametrize("heads", [(8, 2), (4, 4)])
def test_decode_zero_length_responses(case, heads):
    """A response with no cached row decodes against its group's prefix alone, which is what the prefix's last row
    attends in the packed forward; with no prefix either it sees no key and gets O = 0 and LSE = -inf."""
    P, S = EMPTY_RESP[case]
    hq, hkv = heads
    inp, qd, last_rows, T, o, lse = _decode_case(P, S, hq, hkv, 700 + case)
    rows, i, start = [], 0, 0
    for p, ss in zip(P, S):
        for _ in ss:
            rows.append(last_rows[i] if last_rows[i] is not None else (start + p - 1 if p > 0 else None))
            i += 1
        start += p + sum(ss)
    assert any(r is None for r in last_rows)
    for i, row in enumerate(rows):
        if row is None:
            assert torch.all(o[i].float() == 0) and torch.all(torch.isneginf(lse[:, i]))
            continue
        qp = torch.zeros((T, hq, 128), dtype=torch.bfloat16)
        qp[row] = qd[i]
        O_ref, L_ref = oracle.attention_forward_rows(qp, inp["k"], inp["v"], P, S, [row])
        assert np.max(np.abs(to_np64(o[i : i + 1]) - O_ref) - 0.5 * bf16_ulp(O_ref)) <= O_TOL
        assert np.max(np.abs(lse[:, i : i + 1].double().numpy() - L_ref)) <= LSE_TOL
