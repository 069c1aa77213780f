"""Pins for the batch-planning oracle (oracle/batcher.py): hand-worked fixtures and the plan's defining
properties (capacity, greedy maximality, permutation, sort order) on random inputs."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ints(x):
    return [int(v) for v in x.split()]


def test_plan_batches_golden():
    n = 0
    for ln in open(os.path.join(GOLDEN, "plan_batches.txt")):
        if not ln.strip() or ln.startswith("#"):
            continue
        head, order, batch, nb = ln.split("|")
        cap, srt, toks = head.split(";")
        got = oracle.plan_batches(_ints(toks), int(cap), bool(int(srt)))
        assert got == (_ints(order), _ints(batch), int(nb)), ln
        n += 1
    assert n == 6


def test_plan_batches_properties():
    rng = np.random.default_rng(3)
    for it in range(200):
        G = int(rng.integers(0, 40))
        toks = rng.integers(0, 50, size=G).tolist()
        cap = int(rng.integers(1, 120))
        srt = bool(it % 2)
        order, batch, nb = oracle.plan_batches(toks, cap, srt)
        assert sorted(order) == list(range(G))
        if srt:
            assert all(toks[a] >= toks[b] for a, b in zip(order, order[1:]))
        seq = [batch[g] for g in order]
        assert seq == sorted(seq) and (not seq or (seq[0] == 0 and seq[-1] == nb - 1))
        totals = [0] * nb
        for g in order:
            totals[batch[g]] += toks[g]
        for b in range(nb):
            members = [g for g in order if batch[g] == b]
            assert totals[b] <= cap or len(members) == 1           # over capacity only for a lone group
            if b + 1 < nb:                                          # greedy: the next batch's first group did not fit
                first_next = next(g for g in order if batch[g] == b + 1)
                assert totals[b] + toks[first_next] > cap
