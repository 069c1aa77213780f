"""GPU parity of pp_pack_batch against the plain-Python oracle (oracle/pack_batch.py): bit-exact."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _check(prompts, pm, responses, rm, uids):
    from shared_prefix_packed_b200 import pack_batch, pp_get_status
    t = lambda x, dt: torch.as_tensor(np.asarray(x), dtype=dt).cuda()
    ids, P, S, cu, off = pack_batch(t(prompts, torch.int32), t(pm, torch.uint8), t(responses, torch.int32),
                                    t(rm, torch.uint8), t(uids, torch.int64))
    pp_get_status()
    w_ids, w_P, w_S, w_cu, w_off = oracle.pack_batch(prompts, pm, responses, rm, uids)
    assert P == w_P and S == w_S
    assert ids.cpu().numpy().tolist() == w_ids.tolist()
    assert cu.cpu().numpy().tolist() == w_cu.tolist() == W.segment_bounds(P, S).tolist()
    assert off.cpu().numpy().tolist() == w_off.tolist()
    return P, S


def test_pack_golden():
    for ln in open(os.path.join(GOLDEN, "pack_batch.txt")):
        if ln.strip() and not ln.startswith("#"):
            c = json.loads(ln)
            _check(c["prompts"], c["prompt_mask"], c["responses"], c["response_mask"], c["uids"])


def _random(seed, bs, Lp, Lr, n_uids):
    rng = np.random.default_rng(seed)
    uids = rng.integers(0, n_uids, size=bs)
    if seed % 2:
        uids = np.sort(uids)
    prompts = rng.integers(0, 151936, size=(bs, Lp))
    responses = rng.integers(0, 151936, size=(bs, Lr))
    pl = rng.integers(0, Lp + 1, size=bs)
    rl = rng.integers(0, Lr + 1, size=bs)
    left = bool(seed % 3)
    pm = (np.arange(Lp)[None, :] >= (Lp - pl)[:, None]) if left else (np.arange(Lp)[None, :] < pl[:, None])
    rm = np.arange(Lr)[None, :] < rl[:, None]
    if seed % 5 == 0:                                   # scattered masks, not only padding at one side
        rm = rng.random((bs, Lr)) < 0.6
    return prompts, pm.astype(np.uint8), responses, rm.astype(np.uint8), uids


@pytest.mark.parametrize("seed", range(10))
def test_pack_random(seed):
    _check(*_random(seed, bs=1 + 7 * seed, Lp=40 + 33 * seed, Lr=300 - 17 * seed, n_uids=1 + seed % 4))


def test_pack_large_batches():
    _check(*_random(11, bs=4096, Lp=20, Lr=30, n_uids=600))                  # many samples, run lengths of ~1
    _check(*_random(12, bs=128, Lp=1024, Lr=2048, n_uids=16))               # grpo-like rows


def test_pack_empty_and_limits():
    from shared_prefix_packed_b200 import PPError, pack_batch
    z = torch.zeros(0, 4, dtype=torch.int32, device="cuda")
    ids, P, S, cu, off = pack_batch(z, z.to(torch.uint8), z, z.to(torch.uint8), torch.zeros(0, dtype=torch.int64,
                                                                                              device="cuda"))
    assert ids.numel() == 0 and P == [] and S == [] and cu.cpu().tolist() == [0]
    big = torch.zeros(8193, 1, dtype=torch.int32, device="cuda")
    with pytest.raises(PPError, match="UNSUPPORTED"):
        pack_batch(big, big.to(torch.uint8), big, big.to(torch.uint8), torch.zeros(8193, dtype=torch.int64,
                                                                                     device="cuda"))
