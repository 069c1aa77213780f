"""Pins for the micro-batch packing oracle (oracle/pack_batch.py): hand-worked fixtures, run-length grouping by an
independent route (itertools.groupby), the segment boundaries by workloads.segment_bounds, and a round trip."""
import itertools
import json
import os

import numpy as np

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _random_batch(seed, bs=9, Lp=6, Lr=5):
    rng = np.random.default_rng(seed)
    uids = np.repeat(rng.integers(0, 4, size=bs), 1)
    uids = np.sort(rng.integers(0, 3, size=bs)) if seed % 2 else uids        # sorted and unsorted uid orders
    prompts = rng.integers(1, 1000, size=(bs, Lp))
    responses = rng.integers(1, 1000, size=(bs, Lr))
    # left-padded prompts, right-padded responses, some empty
    pl = rng.integers(0, Lp + 1, size=bs)
    rl = rng.integers(0, Lr + 1, size=bs)
    pm = (np.arange(Lp)[None, :] >= (Lp - pl)[:, None]).astype(np.uint8)
    rm = (np.arange(Lr)[None, :] < rl[:, None]).astype(np.uint8)
    return prompts, pm, responses, rm, uids


def test_pack_batch_golden():
    n = 0
    for ln in open(os.path.join(GOLDEN, "pack_batch.txt")):
        if not ln.strip() or ln.startswith("#"):
            continue
        c = json.loads(ln)
        ids, P, S, cu, off = oracle.pack_batch(c["prompts"], c["prompt_mask"], c["responses"], c["response_mask"],
                                               c["uids"])
        assert ids.tolist() == c["packed"] and P == c["P"] and S == c["S"]
        assert cu.tolist() == c["cu"] and off.tolist() == c["offsets"]
        n += 1
    assert n == 3


def test_pack_batch_properties():
    for seed in range(8):
        prompts, pm, responses, rm, uids = _random_batch(seed)
        ids, P, S, cu, off = oracle.pack_batch(prompts, pm, responses, rm, uids)
        sizes = [len(list(g)) for _, g in itertools.groupby(uids.tolist())]
        assert [len(s) for s in S] == sizes
        assert cu.tolist() == W.segment_bounds(P, S).tolist()
        assert len(ids) == sum(P) + sum(map(sum, S))
        heads = np.cumsum([0] + sizes[:-1])
        for g, h in enumerate(heads):
            want = prompts[h][pm[h] != 0]
            assert ids[off[h, 0]:off[h, 0] + P[g]].tolist() == want.tolist()
        for i in range(len(uids)):
            want = responses[i][rm[i] != 0]
            assert ids[off[i, 1]:off[i, 1] + len(want)].tolist() == want.tolist()
            assert (off[i, 0] >= 0) == (i in set(heads.tolist()))
