"""GPU parity of pp_attn_bwd against the fp64 oracle: dQ, dK, dV each within relative Frobenius error 1e-2.

The GPU backward consumes the GPU forward's O (bf16) and LSE, as a training step would; the oracle recomputes
everything in fp64 from the same bf16 inputs. At full workload sizes the oracle runs on whole groups (groups are
independent, so a group's gradients are exact on their own) for a subset of kv heads.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import random_case, to_np64

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2


def rel_fro(got, ref):
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


def _fwd_bwd(P, S, hq, hkv, d, seed, name="dpo"):
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    inp = W.make_inputs(name, P, S, seed=seed, with_dout=True, heads=(hq, hkv, d))
    b = PackedBatch(P, S, hq, hkv, d)
    q, k, v, do = (inp[x].cuda() for x in ("q", "k", "v", "dout"))
    o, lse = b.forward(q, k, v)
    dq, dk, dv = b.backward(q, k, v, o, lse, do)
    pp_get_status()
    return inp, dq, dk, dv


SMALL = [
    ([3], [[2, 0, 3]]),
    ([0], [[130, 77]]),
    ([300], [[]]),
    ([200], [[0, 0, 129]]),
    ([1], [[1] * 40]),
    ([128], [[128, 128]]),
    ([127, 129, 1], [[1, 255], [3], [0]]),
    ([513], [[200, 300, 64]]),
    ([2100], [[700, 900]]),       # long prefix: its key tiles are split over several chunks
]


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("heads", [(4, 2), (7, 1), (2, 2)])
def test_bwd_small(case, heads):
    P, S = SMALL[case]
    hq, hkv = heads
    inp, dq, dk, dv = _fwd_bwd(P, S, hq, hkv, 128, 300 + case)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S)
    for got, want in zip((dq, dk, dv), ref):
        assert rel_fro(to_np64(got), want) <= REL_TOL


@pytest.mark.parametrize("seed", range(4))
def test_bwd_random(seed):
    P, S = random_case(400 + seed, 1 + seed % 4, 1500, 800, 6)
    inp, dq, dk, dv = _fwd_bwd(P, S, 8, 2, 128, seed)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S)
    for got, want in zip((dq, dk, dv), ref):
        assert rel_fro(to_np64(got), want) <= REL_TOL


@pytest.mark.parametrize("name", ["dpo", "grpo", "longprefix"])
def test_bwd_full_workload_sampled_groups(name):
    """Full-size workload in the launch configuration the bench times; the oracle checks whole groups."""
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    w = W.WORKLOADS[name]
    P, S = W.group_lengths(name)
    inp = W.make_inputs(name, P, S)
    b = PackedBatch(P, S, w.num_heads_q, w.num_heads_kv, w.head_dim)
    q, k, v, do = (inp[x].cuda() for x in ("q", "k", "v", "dout"))
    o, lse = b.forward(q, k, v)
    dq, dk, dv = b.backward(q, k, v, o, lse, do)
    pp_get_status()
    assert all(torch.isfinite(t.float()).all() for t in (dq, dk, dv))
    lay = oracle.layout_of(P, S)
    groups = [0, len(P) - 1]
    kv_heads = [0, w.num_heads_kv - 1]
    r = w.num_heads_q // w.num_heads_kv
    qh = [h for kh in kv_heads for h in range(kh * r, (kh + 1) * r)]
    dQ, dK, dV = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S, groups=groups,
                                           kv_heads=kv_heads)
    rows = np.concatenate([np.arange(lay.group_start[g], lay.group_start[g] + lay.group_len[g]) for g in groups])
    assert rel_fro(to_np64(dq[rows][:, qh]), dQ[rows][:, qh]) <= REL_TOL
    assert rel_fro(to_np64(dk[rows][:, kv_heads]), dK[rows][:, kv_heads]) <= REL_TOL
    assert rel_fro(to_np64(dv[rows][:, kv_heads]), dV[rows][:, kv_heads]) <= REL_TOL


def test_bwd_rejects_unsupported():
    from shared_prefix_packed_b200 import PackedBatch, PPError
    P, S = [10], [[5]]
    b = PackedBatch(P, S, 4, 2, 64)
    x = torch.zeros(15, 4, 64, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(15, 2, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(4, 15, device="cuda")
    with pytest.raises(PPError, match="UNSUPPORTED"):
        b.backward(x, kv, kv, x, lse, x)


@pytest.mark.parametrize("case", [0, 4, 6, 8])
def test_bwd_both_dq_paths(case):
    """The same backward with the base workspace (dQ kernel recomputes S and dP) and with room for every step's dS
    tile (dQ formed from the kept tiles): both within the bound of the oracle, and only the second writes dS."""
    from shared_prefix_packed_b200 import PackedBatch, _lib, pp_get_status
    P, S = SMALL[case]
    hq, hkv, d = 4, 2, 128
    inp = W.make_inputs("dpo", P, S, seed=700 + case, with_dout=True, heads=(hq, hkv, d))
    b = PackedBatch(P, S, hq, hkv, d)
    q, k, v, do = (inp[x].cuda() for x in ("q", "k", "v", "dout"))
    o, lse = b.forward(q, k, v)
    base = _lib.pp_workspace_bytes(_lib.PP_PASS_BWD, b.T, hq, hkv, d)
    extra = _lib.pp_bwd_ds_bytes(b.groups_host, b.cu_host, hq, hkv)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S)
    for ws_bytes in (base, base + extra):
        ws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device="cuda")
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        _lib.pp_attn_bwd(q, k, v, o, lse, do, b.meta, dq, dk, dv, ws)
        pp_get_status()
        for got, want in zip((dq, dk, dv), ref):
            assert rel_fro(to_np64(got), want) <= REL_TOL
        if ws_bytes > base:
            kept = ws[(base + 1023) // 1024 * 1024:]
            assert bool((kept[: extra - 1024] != 0xFF).any()), "the kept-dS path did not run"


def test_fwd_bwd_tensors_16_byte_aligned_only():
    """Every tensor 16-byte aligned but not 32-byte aligned (views 16 bytes into their buffers): the 32-byte vector
    loads and stores fall back to 16-byte ones, and the results still match the oracle."""
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    P, S = SMALL[8]
    hq, hkv, d = 4, 2, 128
    inp = W.make_inputs("dpo", P, S, seed=901, with_dout=True, heads=(hq, hkv, d))
    b = PackedBatch(P, S, hq, hkv, d)

    def offset_like(t):
        buf = torch.empty(t.numel() + 8, dtype=torch.bfloat16, device="cuda")
        v = buf[8:].view(t.shape)
        assert v.data_ptr() % 32 == 16
        return v

    q, k, v, do = (offset_like(inp[x]) for x in ("q", "k", "v", "dout"))
    for dst, x in zip((q, k, v, do), ("q", "k", "v", "dout")):
        dst.copy_(inp[x].cuda())
    o = offset_like(q)
    o, lse = b.forward(q, k, v, out=o)
    dq, dk, dv = offset_like(q), offset_like(k), offset_like(v)
    b.backward(q, k, v, o, lse, do, dq=dq, dk=dk, dv=dv)
    pp_get_status()
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S)
    for got, want in zip((dq, dk, dv), ref):
        assert rel_fro(to_np64(got), want) <= REL_TOL


def test_bwd_ds_budget_zero_uses_the_recompute_path():
    """PackedBatch with ds_budget_bytes=0 allocates only the base workspace (the dQ kernel recomputes S and dP); the
    gradients agree with the oracle either way."""
    from shared_prefix_packed_b200 import PackedBatch, _lib, pp_get_status
    P, S = SMALL[6]
    hq, hkv, d = 4, 2, 128
    inp = W.make_inputs("dpo", P, S, seed=950, with_dout=True, heads=(hq, hkv, d))
    b = PackedBatch(P, S, hq, hkv, d, ds_budget_bytes=0)
    assert b.ws_bwd.numel() == _lib.pp_workspace_bytes(_lib.PP_PASS_BWD, b.T, hq, hkv, d)
    q, k, v, do = (inp[x].cuda() for x in ("q", "k", "v", "dout"))
    o, lse = b.forward(q, k, v)
    dq, dk, dv = b.backward(q, k, v, o, lse, do)
    pp_get_status()
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["dout"], P, S)
    for got, want in zip((dq, dk, dv), ref):
        assert rel_fro(to_np64(got), want) <= REL_TOL
