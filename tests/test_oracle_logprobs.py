"""Pins for the response log-probability oracle (oracle/response_logprobs.py).

The row mapping is pinned by hand-worked fixtures and by an independent route (ordinary next-token log-probs on the
unpacked sequence prefix || response, with scipy's log_softmax); the arithmetic by closed forms.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import log_softmax

import oracle
from tests.conftest import random_groups

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_groups(spec):
    P, S = [], []
    for part in spec.split("/"):
        p, s = part.split(";")
        P.append(int(p))
        S.append([int(x) for x in s.split(",") if x.strip()])
    return P, S


def test_source_rows_golden():
    n = 0
    for ln in open(os.path.join(GOLDEN, "logprob_source_rows.txt")):
        if not ln.strip() or ln.startswith("#"):
            continue
        spec, want = ln.split("|")
        P, S = _parse_groups(spec)
        got = oracle.response_source_rows(P, S)
        assert got.tolist() == [int(x) for x in want.split()], (spec, got)
        n += 1
    assert n == 5


def test_logprobs_tiny_golden():
    rows = [ln for ln in open(os.path.join(GOLDEN, "logprob_tiny.txt")) if ln.strip() and not ln.startswith("#")]
    temperature = 2.0
    logits = np.array([[2 * math.log(float(w)) for w in r.split("|")[1].split()] for r in rows])
    ids = np.array([int(r.split("|")[2]) for r in rows])
    got, valid = oracle.response_logprobs(logits, ids, [2], [[2, 1]], temperature=temperature)
    for i, r in enumerate(rows):
        want = r.split("|")[3].strip()
        if want == "-":
            assert not valid[i] and got[i] == 0.0
        else:
            num, den = want.split()[1].split("/")
            assert valid[i] and abs(got[i] - math.log(float(num) / float(den))) < 1e-12


def test_uniform_logits_closed_form():
    P, S = [5, 0, 3], [[4, 2], [3], [1, 1]]
    T = sum(P) + sum(map(sum, S))
    V = 37
    logits = np.full((T, V), 1.25)
    ids = np.arange(T) % V
    got, valid = oracle.response_logprobs(logits, ids, P, S, temperature=0.7)
    assert np.allclose(got[valid], -math.log(V), atol=1e-13)
    # responses with a predicting row: all response tokens except the first one of the P = 0 group
    assert valid.sum() == sum(map(sum, S)) - 1


@pytest.mark.parametrize("seed", range(4))
def test_matches_unpacked_next_token_logprobs(seed):
    """Packed oracle == ordinary next-token log-probs on each unpacked sequence prefix || response (scipy)."""
    P, S = random_groups(np.random.default_rng(100 + seed), 3, 7, 6, 3)
    lay = oracle.layout_of(P, S)
    T, V, temp = lay.T, 11, 1.3
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, V)) * 3.0
    ids = rng.integers(0, V, size=T)
    got, valid = oracle.response_logprobs(logits, ids, P, S, temperature=temp)
    want = np.zeros(T)
    want_valid = np.zeros(T, dtype=bool)
    for g in range(len(P)):
        o = int(lay.group_start[g])
        prefix_rows = list(range(o, o + P[g]))
        start = o + P[g]
        for s in S[g]:
            rows = prefix_rows + list(range(start, start + s))       # the unpacked sequence, as packed row indices
            lp = log_softmax(logits[rows] / temp, axis=1)
            for t in range(len(prefix_rows), len(rows)):             # response positions
                if t == 0:
                    continue                                          # nothing precedes it
                want[rows[t]] = lp[t - 1, ids[rows[t]]]
                want_valid[rows[t]] = True
            start += s
    assert (valid == want_valid).all()
    assert np.allclose(got, want, atol=1e-12)


def test_shift_and_temperature_invariances():
    P, S = [4], [[3, 3]]
    T, V = 10, 9
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((T, V))
    ids = rng.integers(0, V, size=T)
    a, va = oracle.response_logprobs(logits, ids, P, S, temperature=1.0)
    b, _ = oracle.response_logprobs(logits + rng.standard_normal((T, 1)) * 10, ids, P, S, temperature=1.0)
    c, _ = oracle.response_logprobs(logits * 3.0, ids, P, S, temperature=3.0)
    assert np.allclose(a, b, atol=1e-12) and np.allclose(a, c, atol=1e-12)
    assert (a[va] < 0).all()
