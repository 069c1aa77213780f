"""Plain-Python oracle for building a packed batch from an ungrouped micro-batch.

TEST INFRASTRUCTURE (see the package docstring): never imported by the product path.

"prefix_grouper_utils.py" §2 (building the grouper from a micro-batch): the samples of a micro-batch carry a uid;
consecutive samples with the same uid form a group (the group sizes are the run lengths of equal consecutive uids),
a group's prefix is the prompt of its first sample, and the packed input is, group by group, the prefix's valid
tokens followed by each sample's valid response tokens (concat_input with the prefix and response masks).
Here the result is pad-free: one flat sequence of T tokens, with the descriptors (P_g, k_g) and the segment
boundaries (for each group its prefix, then each response; zero-length segments kept) that describe it.
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np


def pack_batch(prompts, prompt_mask, responses, response_mask, uids):
    """Returns (packed_ids int32[T], prefix_lens [G], suffix_lens [G][k_g], cu_seqlens int32[nseg+1],
    sample_offsets int32[bs, 2]).

    sample_offsets[i] = (packed offset of sample i's prompt tokens if it heads its group, else -1;
                         packed offset of sample i's response tokens).
    Masks: nonzero marks a valid token; valid tokens keep their order. Padding may be on either side.
    """
    prompts = np.asarray(prompts)
    responses = np.asarray(responses)
    pm = np.asarray(prompt_mask) != 0
    rm = np.asarray(response_mask) != 0
    uids = np.asarray(uids)
    bs = len(uids)
    # group sizes: run lengths of equal consecutive uids
    sizes: List[int] = []
    for i in range(bs):
        if i == 0 or uids[i] != uids[i - 1]:
            sizes.append(1)
        else:
            sizes[-1] += 1
    packed: List[int] = []
    P: List[int] = []
    S: List[List[int]] = []
    cu = [0]
    offsets = np.full((bs, 2), -1, dtype=np.int32)
    i = 0
    for gs in sizes:
        head = i
        prefix = [int(t) for t, m in zip(prompts[head], pm[head]) if m]
        offsets[head, 0] = len(packed)
        packed.extend(prefix)
        P.append(len(prefix))
        cu.append(len(packed))
        S.append([])
        for j in range(head, head + gs):
            resp = [int(t) for t, m in zip(responses[j], rm[j]) if m]
            offsets[j, 1] = len(packed)
            packed.extend(resp)
            S[-1].append(len(resp))
            cu.append(len(packed))
        i += gs
    return (np.array(packed, dtype=np.int32), P, S, np.array(cu, dtype=np.int32), offsets)
