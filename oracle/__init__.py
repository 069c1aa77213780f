"""Plain, slow fp64 CPU oracle for exact attention over a preference-packed sequence.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg (and its
``--impl reference`` arm) may import this package. The product path (the C-ABI library and its Python binding)
never imports, calls or links it, and this package imports nothing from the product path. Both sides draw inputs
from ``workloads`` only.

Every function restates the definition it follows; the pages it cites are
  * "Preference Packing: Efficient Preference Optimization for LLMs" (abstract and method digest),
  * "prefix_grouper_utils.py" (verl fork documentation: §1 building position ids, §2 building the grouper from a
    micro-batch,
    §3 forward including the split of the logits and the log-probabilities of the responses, and its
    prefix-sharing diagram),
  * "PackInfer: Compute- and I/O-Efficient Attention for Batched LLM Inference" (abstract).

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` (brute force, closed forms, library
cross-checks, finite differences, hand-worked fixtures under ``tests/golden/``). No function is "parity unpinned".
"""
from .packed_attention import (  # noqa: F401
    PackedLayout,
    allowed_mask,
    allowed_pair_count,
    allowed_pairs_per_row,
    attention_backward,
    attention_forward,
    attention_forward_rows,
    causal_attention,
    causal_attention_backward,
    layout_of,
    position_ids,
    rope,
    tile_classes,
    tile_classes_bruteforce,
    unpacked_backward,
    unpacked_forward,
)
from .batcher import plan_batches  # noqa: F401
from .pack_batch import pack_batch  # noqa: F401
from .response_logprobs import (  # noqa: F401
    response_logprobs,
    response_logprobs_rows,
    response_source_rows,
)
