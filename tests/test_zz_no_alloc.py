"""pp_attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a plugin or custom op that a host framework hands only its input and output pointers, with the
framework's own caching allocator owning the device memory; code that must not allocate at that point) cannot
provide the workspace pp_attn_bwd asks for. pp_attn_bwd_noalloc uses a 64 MiB scratch array compiled into the
library instead. This file is collected last so that, if it fails, a run stopping at the first failure has already
run every other test; it must pass both on its own in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2   # the backward tests' relative Frobenius bound


def _rel(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def test_noalloc_backward_matches_workspace_backward_twice():
    from shared_prefix_packed_b200 import PackedBatch, _lib
    P, S = [700, 300], [[400, 250], [600, 0, 90]]      # T = 2340: fits the 64 MiB scratch at 32/8 heads
    hq, hkv, d = 32, 8, 128
    T = W.packed_total(P, S)
    assert _lib.pp_workspace_bytes(_lib.PP_PASS_BWD, T, hq, hkv, d) <= _lib.NOALLOC_SCRATCH_BYTES
    inp = W.make_inputs("dpo", P, S, seed=11, with_dout=True, heads=(hq, hkv, d))
    b = PackedBatch(P, S, hq, hkv, d)
    q, k, v, do = (inp[x].cuda() for x in ("q", "k", "v", "dout"))
    o, lse = b.forward(q, k, v)
    ref = b.backward(q, k, v, o, lse, do)                # the existing entry point, caller workspace
    _lib.pp_get_status()
    for _ in range(2):                                   # two calls in a row share (and reuse) the scratch
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        _lib.pp_attn_bwd_noalloc(q, k, v, o, lse, do, b.meta, dq, dk, dv)
        _lib.pp_get_status()
        for got, want in zip((dq, dk, dv), ref):
            assert _rel(got, want) <= REL_TOL


def test_noalloc_rejects_sizes_beyond_the_scratch():
    """A call whose scratch would not fit is refused on the host with a clear error; nothing is enqueued."""
    from shared_prefix_packed_b200 import _lib
    T, hq, hkv, d = 20000, 32, 8, 128
    assert _lib.pp_workspace_bytes(_lib.PP_PASS_BWD, T, hq, hkv, d) > _lib.NOALLOC_SCRATCH_BYTES
    q = torch.empty(T, hq, d, dtype=torch.bfloat16, device="cuda")
    kv = torch.empty(T, hkv, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(hq, T, dtype=torch.float32, device="cuda")
    meta = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.PPError, match="WORKSPACE") as e:
        _lib.pp_attn_bwd_noalloc(q, kv, kv, q, lse, q, meta, q, kv, kv)
    assert "built-in array holds" in str(e.value)
