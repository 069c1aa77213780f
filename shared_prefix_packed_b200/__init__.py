"""Exact softmax attention over preference-packed sequences on B200 (sm_100a).

A group packs one prompt prefix once, followed by its responses; a prefix token attends causally within the prefix,
a response token attends to the whole prefix and causally within its own response, and position ids restart at
the prefix length for every response ("Preference Packing" abstract; "prefix_grouper_utils.py" sections 1-2;
"PackInfer" abstract). The work runs in libpp.so, a C-ABI CUDA library (include/pp.h); this package is its thin
binding (``_lib``) plus :class:`PackedBatch`, which allocates the buffers with torch and calls the library.
"""
from ._lib import (  # noqa: F401
    PP_BF16, PP_FP32, PP_PASS_BWD, PP_PASS_FWD, PPError,
    pp_attn_bwd, pp_attn_fwd, pp_build_meta, pp_bwd_ds_bytes, pp_decode_attn, pp_decode_workspace_bytes, pp_get_status,
    pp_meta_bounds, pp_meta_schedule, pp_meta_tiles, pp_pack_batch, pp_plan_batches,
    pp_response_logprobs,
    pp_rope,
    pp_version, pp_workspace_bytes,
)
from .packed import PackedBatch, pack_batch  # noqa: F401
