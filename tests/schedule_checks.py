"""Checks of an executed tile schedule against the oracle's canonical tile set (host logic, used by the GPU tests
and pinned on the CPU by tests/test_schedule_checks.py)."""
import oracle


def check_forward_schedule(P, S, recs):
    """The cost-ordered query tiles the forward (and the dQ kernel) execute: every query tile of the layout appears
    as exactly one item, items are in non-increasing cost (key tiles visited), and the union of their key tiles is
    the oracle's canonical tile set with each tile exactly once."""
    want = oracle.tile_classes(P, S, 128, 128)
    assert sorted((q, k, c) for _, q, k, c, _ in recs) == want          # also: no tile twice
    rows_of_item, cost = {}, {}
    for it, q, _, _, split in recs:
        assert split == 0
        rows_of_item.setdefault(it, set()).add(q)
        cost[it] = cost.get(it, 0) + 1
    assert all(len(v) == 1 for v in rows_of_item.values())              # one query tile per item
    qrows = [next(iter(rows_of_item[i])) for i in sorted(rows_of_item)]
    assert sorted(qrows) == sorted({q for q, _, _ in want})              # a permutation of the query tiles
    assert sorted(rows_of_item) == list(range(len(qrows)))               # items 0..n-1, none missing
    costs = [cost[i] for i in sorted(cost)]
    assert all(a >= b for a, b in zip(costs, costs[1:]))                  # longest first


def check_backward_schedule(P, S, recs, max_chunks=16):
    """The backward work chunks: the chunks of each key tile partition its query tiles disjointly and completely (so
    the expanded chunks are the canonical tile set, each tile once), every chunk is one contiguous run of query
    tiles of one key tile, `split` is set exactly when a key tile has more than one chunk, and chunks are stored
    in non-increasing cost."""
    want = oracle.tile_classes(P, S, 128, 128)
    assert sorted((q, k, c) for _, q, k, c, _ in recs) == want          # disjoint and complete
    key_of, qrows, split_of = {}, {}, {}
    for it, q, k, c, split in recs:
        assert key_of.setdefault(it, k) == k                              # one key tile per chunk
        qrows.setdefault(it, []).append(q)
        assert split_of.setdefault(it, split) == split
    assert sorted(key_of) == list(range(len(key_of)))
    chunks_of_key = {}
    for it, rows in qrows.items():
        rows.sort()
        assert all(b - a == 128 for a, b in zip(rows, rows[1:]))          # contiguous query tiles
        chunks_of_key.setdefault(key_of[it], []).append(it)
    for k, items in chunks_of_key.items():
        assert len(items) <= max_chunks
        assert all(split_of[i] == (1 if len(items) > 1 else 0) for i in items)
    costs = [len(qrows[i]) for i in sorted(qrows)]
    assert all(a >= b for a, b in zip(costs, costs[1:]))
