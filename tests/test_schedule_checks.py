"""CPU checks that the schedule checkers used by the GPU tests accept a valid schedule and reject plausible
mistakes (a dropped, duplicated or misplaced tile, a wrong order, a wrong split flag, a chunk with a gap)."""
import pytest

import oracle
from tests.schedule_checks import check_backward_schedule, check_forward_schedule

P, S = [2100, 300], [[700, 900], [130, 0, 260]]


def _fwd_schedule():
    tiles = oracle.tile_classes(P, S, 128, 128)
    by_q = {}
    for q, k, c in tiles:
        by_q.setdefault(q, []).append((k, c))
    order = sorted(by_q, key=lambda q: -len(by_q[q]))
    return [(i, q, k, c, 0) for i, q in enumerate(order) for k, c in by_q[q]]


def _bwd_schedule(chunk=3):
    tiles = oracle.tile_classes(P, S, 128, 128)
    by_k = {}
    for q, k, c in tiles:
        by_k.setdefault(k, []).append((q, c))
    chunks = []
    for k, qs in by_k.items():
        qs.sort()
        parts = [qs[i:i + chunk] for i in range(0, len(qs), chunk)]
        for part in parts:
            chunks.append((k, part, 1 if len(parts) > 1 else 0))
    chunks.sort(key=lambda x: -len(x[1]))
    return [(i, q, k, c, sp) for i, (k, part, sp) in enumerate(chunks) for q, c in part]


def test_valid_schedules_pass():
    check_forward_schedule(P, S, _fwd_schedule())
    check_backward_schedule(P, S, _bwd_schedule())


@pytest.mark.parametrize("mistake", ["drop", "dup", "order", "two_rows"])
def test_forward_checker_rejects(mistake):
    recs = _fwd_schedule()
    if mistake == "drop":
        recs = recs[1:]
    elif mistake == "dup":
        recs = recs + [recs[-1]]
    elif mistake == "order":                       # the cheapest item placed first
        last = max(r[0] for r in recs)
        recs = [((0 if r[0] == last else r[0] + 1),) + r[1:] for r in recs]
    elif mistake == "two_rows":                    # an item that mixes two query tiles
        it0 = [r for r in recs if r[0] == 0]
        it1 = [r for r in recs if r[0] == 1]
        recs = [r for r in recs if r[0] not in (0, 1)] + it0 + [(0,) + r[1:] for r in it1]
    with pytest.raises(AssertionError):
        check_forward_schedule(P, S, recs)


@pytest.mark.parametrize("mistake", ["drop", "dup", "split_flag", "gap", "order", "too_many"])
def test_backward_checker_rejects(mistake):
    recs = _bwd_schedule()
    if mistake == "drop":
        recs = recs[:-1]
    elif mistake == "dup":
        recs = recs + [recs[0]]
    elif mistake == "split_flag":
        recs = [r[:4] + (1 - r[4],) if r[0] == 0 else r for r in recs]
    elif mistake == "gap":                         # a chunk whose query tiles are not contiguous
        it = [r for r in recs if r[0] == 0]
        rest = [r for r in recs if r[0] != 0]
        victim = next(r for r in rest if r[2] == it[0][2] and r[1] > it[-1][1] + 128)
        recs = [r for r in rest if r != victim] + it + [(0,) + victim[1:]]
    elif mistake == "order":
        last = max(r[0] for r in recs)
        recs = [((0 if r[0] == last else r[0] + 1),) + r[1:] for r in recs]
    elif mistake == "too_many":
        recs = _bwd_schedule(chunk=1)
    with pytest.raises(AssertionError):
        check_backward_schedule(P, S, recs, max_chunks=16 if mistake != "too_many" else 4)
