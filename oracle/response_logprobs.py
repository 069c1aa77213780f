"""fp64 CPU oracle for the log-probabilities of response tokens, read off the logits of a packed sequence.

TEST INFRASTRUCTURE (see the package docstring): never imported by the product path.

"prefix_grouper_utils.py" §3 (the forward with the grouper): after the model runs on the packed sequence, the
grouper splits the logits into a prefix part and a suffix part, the suffix part of each response starting with the
prefix's last row (split_output with include_prefix_last=1). The last row of each such block is dropped, the rest
is divided by the sampling temperature, and the log-probability of each completion token is read from the
log-softmax of its row.

Restated on the pad-free packed layout (groups in order, each its prefix then its responses): the token at packed
row y of response i of group g is predicted by row y - 1, except the response's first token, which is predicted by
the group's last prefix row o_g + P_g - 1 (not by the last row of the previous response). That is ordinary
next-token prediction on the unpacked sequence prefix || response. A group with P_g = 0 has no row that predicts its
responses' first tokens; those rows, and all prefix rows, have no log-probability here (value 0, valid False).
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from .packed_attention import layout_of


def response_source_rows(prefix_lens, suffix_lens) -> np.ndarray:
    """int64[T]: the packed row whose logits predict the token at each row, or -1 where there is none.

    Prefix rows get -1 (only response tokens are scored). A response's first row gets the group's last prefix row,
    or -1 when the group has no prefix; every other response row gets the row before it.
    """
    lay = layout_of(prefix_lens, suffix_lens)
    src = np.full(lay.T, -1, dtype=np.int64)
    for t in range(lay.T):
        if lay.seg_of[t] == 0:
            continue
        g = int(lay.group_of[t])
        if t == lay.seg_start[t]:
            P = lay.prefix_lens[g]
            src[t] = int(lay.group_start[g]) + P - 1 if P > 0 else -1
        else:
            src[t] = t - 1
    return src


def _log_softmax_at(row: np.ndarray, index: int, temperature: float) -> float:
    """log softmax(row / temperature)[index] in fp64: x_i - (m + ln sum_j exp(x_j - m)) with m = max_j x_j."""
    x = np.asarray(row, dtype=np.float64) / float(temperature)
    m = float(np.max(x))
    return float(x[index] - (m + np.log(np.sum(np.exp(x - m)))))


def response_logprobs_rows(logits, token_ids, prefix_lens, suffix_lens, rows: Sequence[int],
                           temperature: float = 1.0) -> Tuple[np.ndarray, np.ndarray]:
    """(log-probabilities, valid) at the given packed rows; see the module docstring for the row mapping.

    logits: [T, V] (any float dtype or torch tensor; read as fp64). token_ids: [T] integers in [0, V).
    """
    L = logits.detach().cpu().double().numpy() if hasattr(logits, "detach") else np.asarray(logits, np.float64)
    ids = token_ids.detach().cpu().numpy() if hasattr(token_ids, "detach") else np.asarray(token_ids)
    src = response_source_rows(prefix_lens, suffix_lens)
    out = np.zeros(len(rows), dtype=np.float64)
    valid = np.zeros(len(rows), dtype=bool)
    for n, y in enumerate(rows):
        s = int(src[y])
        if s < 0:
            continue
        out[n] = _log_softmax_at(L[s], int(ids[y]), temperature)
        valid[n] = True
    return out, valid


def response_logprobs(logits, token_ids, prefix_lens, suffix_lens,
                      temperature: float = 1.0) -> Tuple[np.ndarray, np.ndarray]:
    """(log-probabilities [T], valid [T]) for every packed row."""
    T = layout_of(prefix_lens, suffix_lens).T
    return response_logprobs_rows(logits, token_ids, prefix_lens, suffix_lens, range(T), temperature)
