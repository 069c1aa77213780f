"""Pins for the oracle's forward and backward (CPU only, fp64)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import random_groups

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_qkv(rng, T, hq, hkv, d):
    return (rng.standard_normal((T, hq, d)), rng.standard_normal((T, hkv, d)), rng.standard_normal((T, hkv, d)),
            rng.standard_normal((T, hq, d)))


def _sdpa_fp64(q, k, v, mask, scale=None):
    """torch CPU fp64 scaled_dot_product_attention with an explicit boolean mask and GQA (library cross-check)."""
    qt = torch.from_numpy(q).permute(1, 0, 2).unsqueeze(0)
    kt = torch.from_numpy(k).permute(1, 0, 2).unsqueeze(0)
    vt = torch.from_numpy(v).permute(1, 0, 2).unsqueeze(0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask),
                                                         scale=scale, enable_gqa=True)
    return o[0].permute(1, 0, 2).numpy()


def test_forward_golden():
    q = np.zeros((3, 1, 4)); k = np.zeros((3, 1, 4)); v = np.zeros((3, 1, 4))
    q[0, 0, 0] = 1.0; k[0, 0, 0] = 2.0
    v[0, 0, 0] = 1.0; v[1, 0, 1] = 1.0; v[2, 0, 2] = 1.0
    O, L = oracle.attention_forward(q, k, v, [2], [[1]])
    with open(os.path.join(GOLDEN, "forward_tiny.txt")) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    for ln in rows:
        r, lse, o = ln.split("|")
        r = int(r)
        assert abs(L[0, r] - float(lse)) < 1e-15
        assert np.allclose(O[r, 0], [float(x) for x in o.split()], atol=1e-15)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (6, 2)])
def test_forward_matches_sdpa_with_bruteforce_mask(hq, hkv):
    rng = np.random.default_rng(20 + hq + hkv)
    for _ in range(6):
        P, S = random_groups(rng, int(rng.integers(1, 4)), 12, 9, 4)
        T = oracle.layout_of(P, S).T
        if T == 0:
            continue
        q, k, v, _ = _rand_qkv(rng, T, hq, hkv, 8)
        O, L = oracle.attention_forward(q, k, v, P, S, chunk=5)
        want = _sdpa_fp64(q, k, v, oracle.allowed_mask(P, S))
        assert np.allclose(O, want, atol=1e-12)
        # the LSE: ln of the masked row sums of exp(scaled scores), recomputed with scipy's logsumexp
        from scipy.special import logsumexp
        m = oracle.allowed_mask(P, S)
        for h in range(hq):
            s = (q[:, h, :] @ k[:, h // (hq // hkv), :].T) / math.sqrt(8)
            want_l = logsumexp(np.where(m, s, -np.inf), axis=1)
            assert np.allclose(L[h], want_l, atol=1e-12)
            assert np.all(L[h] >= np.where(m, s, -np.inf).max(axis=1) - 1e-12)


def test_forward_equals_unpacked_runs_with_rope():
    """Defining invariant: packed rows of S_i equal causal attention on P||S_i; prefix rows equal causal on P.
    RoPE is applied at the grouped positions on the packed side and at 0..len-1 on each unpacked run."""
    rng = np.random.default_rng(31)
    for _ in range(8):
        P, S = random_groups(rng, int(rng.integers(1, 4)), 14, 10, 4)
        T = oracle.layout_of(P, S).T
        if T == 0:
            continue
        q, k, v, _ = _rand_qkv(rng, T, 4, 2, 16)
        pos = oracle.position_ids(P, S)
        O, L = oracle.attention_forward(oracle.rope(q, pos), oracle.rope(k, pos), v, P, S, chunk=7)
        Ou, Lu = oracle.unpacked_forward(q, k, v, P, S, theta=10000.0)
        assert np.max(np.abs(O - Ou)) <= 1e-12
        assert np.max(np.abs(L - Lu)) <= 1e-12


def test_forward_special_cases_and_softmax_rows():
    rng = np.random.default_rng(41)
    # k = 1: exactly causal attention on P||S
    q, k, v, _ = _rand_qkv(rng, 23, 2, 1, 8)
    O, L = oracle.attention_forward(q, k, v, [10], [[13]])
    Oc, Lc = oracle.causal_attention(q, k, v)
    assert np.allclose(O, Oc, atol=1e-13) and np.allclose(L, Lc, atol=1e-13)
    # P = 0: each suffix is its own causal sequence (block-diagonal varlen causal)
    O, L = oracle.attention_forward(q, k, v, [0], [[9, 14]])
    O1, _ = oracle.causal_attention(q[:9], k[:9], v[:9])
    O2, _ = oracle.causal_attention(q[9:], k[9:], v[9:])
    assert np.allclose(O, np.concatenate([O1, O2]), atol=1e-13)
    # softmax rows sum to one: with v = all-ones, o = 1 exactly (up to rounding)
    ones = np.ones_like(v)
    O, _ = oracle.attention_forward(q, k, ones, [5], [[7, 0, 11]])
    assert np.max(np.abs(O - 1.0)) <= 1e-12


def test_forward_rows_sampler_matches_full():
    rng = np.random.default_rng(43)
    P, S = [9, 4], [[5, 7], [0, 6, 3]]
    T = oracle.layout_of(P, S).T
    q, k, v, _ = _rand_qkv(rng, T, 4, 2, 8)
    O, L = oracle.attention_forward(q, k, v, P, S)
    rows = [0, 3, 9, 14, 20, 21, 25, T - 1]
    Or, Lr = oracle.attention_forward_rows(q, k, v, P, S, rows)
    assert np.allclose(Or, O[rows], atol=1e-13) and np.allclose(Lr, L[:, rows], atol=1e-13)


def _loss(q, k, v, dout, P, S):
    O, _ = oracle.attention_forward(q, k, v, P, S)
    return float((O * dout).sum())


def test_backward_finite_differences():
    rng = np.random.default_rng(51)
    P, S = [3, 2], [[2, 0, 3], [1, 2]]
    T = oracle.layout_of(P, S).T
    q, k, v, do = _rand_qkv(rng, T, 4, 2, 4)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, P, S)
    eps = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, P, S)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, P, S)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])


def test_backward_matches_torch_autograd():
    rng = np.random.default_rng(52)
    for _ in range(4):
        P, S = random_groups(rng, int(rng.integers(1, 4)), 10, 8, 4)
        T = oracle.layout_of(P, S).T
        if T == 0:
            continue
        q, k, v, do = _rand_qkv(rng, T, 6, 2, 8)
        dq, dk, dv = oracle.attention_backward(q, k, v, do, P, S, chunk=4)
        qt, kt, vt = (torch.from_numpy(a).permute(1, 0, 2).unsqueeze(0).requires_grad_(True) for a in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=torch.from_numpy(oracle.allowed_mask(P, S)), enable_gqa=True)
        (o * torch.from_numpy(do).permute(1, 0, 2).unsqueeze(0)).sum().backward()
        for mine, t in ((dq, qt), (dk, kt), (dv, vt)):
            assert np.allclose(mine, t.grad[0].permute(1, 0, 2).numpy(), atol=1e-12)


def test_backward_equals_unpacked_identity():
    rng = np.random.default_rng(53)
    for _ in range(6):
        P, S = random_groups(rng, int(rng.integers(1, 4)), 12, 9, 4)
        T = oracle.layout_of(P, S).T
        if T == 0:
            continue
        q, k, v, do = _rand_qkv(rng, T, 4, 2, 8)
        got = oracle.attention_backward(q, k, v, do, P, S, chunk=6)
        want = oracle.unpacked_backward(q, k, v, do, P, S)
        for a, b in zip(got, want):
            assert np.max(np.abs(a - b)) <= 1e-11
