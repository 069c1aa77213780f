"""Plain-Python oracle for planning batches of packed preference groups on the host.

TEST INFRASTRUCTURE (see the package docstring): never imported by the product path.

"Preference Packing" (abstract and method digest): preference packing combines with batch sorting (sorting the
data by length before batching), and the batch size is adjusted to the data's lengths to balance compute and
memory. Restated as a plan over groups (each group = one prompt with its responses, packed once): a group costs its
packed length L_g = P_g + sum_i S_gi tokens; with sorting, groups are taken longest first (ties keep their input
order); batches are filled greedily in that order up to a token capacity, so the number of groups per batch
follows their lengths; a group longer than the capacity forms a batch of its own.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def plan_batches(group_tokens: Sequence[int], capacity: int, sort_by_length: bool) -> Tuple[List[int], List[int], int]:
    """Returns (order, batch_of_group, n_batches): the groups in batch order, each group's batch, the batch count."""
    G = len(group_tokens)
    order = list(range(G))
    if sort_by_length:
        order.sort(key=lambda g: -int(group_tokens[g]))        # Python's sort is stable: ties keep input order
    batch_of_group = [0] * G
    batch, filled, members = 0, 0, 0
    for g in order:
        t = int(group_tokens[g])
        if members > 0 and filled + t > capacity:              # the group does not fit: close the batch
            batch, filled, members = batch + 1, 0, 0
        batch_of_group[g] = batch
        filled += t
        members += 1
    return order, batch_of_group, (batch + 1 if G else 0)
