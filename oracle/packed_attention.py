"""fp64 CPU oracle: layout, grouped position ids, mask, tile classes, RoPE, forward and backward.

TEST INFRASTRUCTURE (see the package docstring): never imported by the product path.

Notation. Group g packs its prompt prefix (P_g tokens) once, then its k_g responses S_g1..S_gk back to back
("Preference Packing", abstract: the attention of a prompt shared by several responses is computed once;
"prefix_grouper_utils.py", prefix-sharing diagram: the prefix is computed once and each response suffix continues
it). T is the packed length. Q and dO are [T, Hq, d]; K and V are [T, Hkv, d]; q head h reads kv head h // (Hq/Hkv).

The attention mask is never written out on the pages; this oracle takes the reading the pages' prose supports:
query i may attend key j iff both are in the same group, j <= i, and j is in the prefix or in i's own segment.
A prefix token therefore attends causally within the prefix, and a token of S_i attends to all of P and causally
within S_i, never to a sibling response.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Sequence, Tuple

import numpy as np

FULL = 1
PARTIAL = 2


# ----------------------------------------------------------------------------------------------------------------
# Layout
# ----------------------------------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class PackedLayout:
    """Per-group offsets and per-token segment labels of the packed order.

    group_start[g], group_len[g]: packed offset and length L_g = P_g + sum_i S_gi of group g.
    seg_of[t]: 0 for a prefix token, i+1 for a token of response i (within its group).
    seg_start[t]: packed offset of the first token of t's segment.
    group_of[t]: group index of token t.
    """
    prefix_lens: Tuple[int, ...]
    suffix_lens: Tuple[Tuple[int, ...], ...]
    group_start: np.ndarray
    group_len: np.ndarray
    group_of: np.ndarray
    seg_of: np.ndarray
    seg_start: np.ndarray

    @property
    def T(self) -> int:
        return int(self.group_of.shape[0])


def layout_of(prefix_lens: Sequence[int], suffix_lens: Sequence[Sequence[int]]) -> PackedLayout:
    """Build the packed layout: groups in order, each its prefix then its suffixes in order.

    "prefix_grouper_utils.py" §2: the grouper concatenates each group's prefix ids with its valid response ids.
    Here the packing is pad-free (one flat row of T tokens) instead of the page's [num_groups, max_len] padded rows;
    the non-pad tokens and their order are the same.
    """
    P = tuple(int(p) for p in prefix_lens)
    S = tuple(tuple(int(s) for s in ss) for ss in suffix_lens)
    if len(P) != len(S):
        raise ValueError("one suffix list per group")
    if any(p < 0 for p in P) or any(s < 0 for ss in S for s in ss):
        raise ValueError("lengths must be non-negative")
    gl = np.array([p + sum(ss) for p, ss in zip(P, S)], dtype=np.int64)
    gs = np.zeros(len(P), dtype=np.int64)
    if len(P) > 1:
        gs[1:] = np.cumsum(gl)[:-1]
    T = int(gl.sum())
    group_of = np.empty(T, dtype=np.int64)
    seg_of = np.empty(T, dtype=np.int64)
    seg_start = np.empty(T, dtype=np.int64)
    for g, (p, ss) in enumerate(zip(P, S)):
        o = int(gs[g])
        group_of[o:o + gl[g]] = g
        seg_of[o:o + p] = 0
        seg_start[o:o + p] = o
        b = o + p
        for i, s in enumerate(ss):
            seg_of[b:b + s] = i + 1
            seg_start[b:b + s] = b
            b += s
    return PackedLayout(P, S, gs, gl, group_of, seg_of, seg_start)


def position_ids(prefix_lens, suffix_lens) -> np.ndarray:
    """Grouped position ids, int32[T].

    "prefix_grouper_utils.py" §1 (building position ids): the prefix takes positions 0..P-1, and every response
    suffix restarts at P (P, P+1, ...), so each suffix continues the prefix independently of its siblings;
    zero-length suffixes contribute nothing. Written here without the page's zero padding.
    """
    lay = layout_of(prefix_lens, suffix_lens)
    pos = np.empty(lay.T, dtype=np.int64)
    for g, (p, ss) in enumerate(zip(lay.prefix_lens, lay.suffix_lens)):
        o = int(lay.group_start[g])
        for t in range(p):
            pos[o + t] = t
        cur = o + p
        for s in ss:
            for t in range(s):
                pos[cur + t] = p + t
            cur += s
    return pos.astype(np.int32)


# ----------------------------------------------------------------------------------------------------------------
# Mask
# ----------------------------------------------------------------------------------------------------------------
def allowed_mask(prefix_lens, suffix_lens) -> np.ndarray:
    """Dense boolean mask [T, T] (query i, key j) by the definition, element by element. Small T only."""
    lay = layout_of(prefix_lens, suffix_lens)
    T = lay.T
    m = np.zeros((T, T), dtype=bool)
    for i in range(T):
        for j in range(i + 1):
            if lay.group_of[i] != lay.group_of[j]:
                continue
            if lay.seg_of[j] == 0 or lay.seg_of[j] == lay.seg_of[i]:
                m[i, j] = True
    return m


def allowed_pairs_per_row(lay: PackedLayout) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Each row's allowed key set as two packed intervals [a1, b1) U [a2, b2).

    Prefix row i of group g: [o_g, i+1) and an empty second interval.
    Row i of response r: the whole prefix [o_g, o_g+P_g) and its own segment's keys up to i, [seg_start(i), i+1).
    Returns (a1b1 [T,2], a2b2 [T,2], count [T]).
    """
    T = lay.T
    o = lay.group_start[lay.group_of]
    P = np.asarray(lay.prefix_lens, dtype=np.int64)[lay.group_of]
    idx = np.arange(T, dtype=np.int64)
    in_prefix = lay.seg_of == 0
    i1 = np.stack([o, np.where(in_prefix, idx + 1, o + P)], axis=1)
    i2 = np.stack([np.where(in_prefix, idx + 1, lay.seg_start), idx + 1], axis=1)
    cnt = (i1[:, 1] - i1[:, 0]) + (i2[:, 1] - i2[:, 0])
    return i1, i2, cnt


def allowed_pair_count(prefix_lens, suffix_lens) -> int:
    """Allowed (query, key) pairs of one head: sum_g [P(P+1)/2 + sum_i (S_i P + S_i(S_i+1)/2)] (closed form)."""
    tot = 0
    for p, ss in zip(prefix_lens, suffix_lens):
        tot += p * (p + 1) // 2
        for s in ss:
            tot += s * p + s * (s + 1) // 2
    return int(tot)


# ----------------------------------------------------------------------------------------------------------------
# Tile classes
# ----------------------------------------------------------------------------------------------------------------
def _tile_grid(lay: PackedLayout, BM: int, BN: int):
    for g in range(len(lay.prefix_lens)):
        o = int(lay.group_start[g])
        L = int(lay.group_len[g])
        for a in range(-(-L // BM)):
            for b in range(-(-L // BN)):
                yield g, o, L, o + a * BM, o + b * BN


def tile_classes_bruteforce(prefix_lens, suffix_lens, BM: int, BN: int) -> List[Tuple[int, int, int]]:
    """Non-empty tiles as sorted (q_row0, kv_row0, class) by enumerating every pair of every tile.

    Tiles are aligned to each group's start: q tile a of group g covers packed rows o_g + a*BM + [0, BM) and kv tile
    b covers o_g + b*BN + [0, BN), for a, b over ceil(L_g/BM) and ceil(L_g/BN). Positions outside the group (past
    its end) count as not allowed, so a tile that sticks out of its group is never FULL. A tile is FULL iff all its
    BM*BN pairs are allowed and EMPTY iff none is; EMPTY tiles are left out of the list.
    """
    lay = layout_of(prefix_lens, suffix_lens)
    m = allowed_mask(prefix_lens, suffix_lens)
    T = lay.T
    out = []
    for g, o, L, q0, k0 in _tile_grid(lay, BM, BN):
        n = 0
        for i in range(q0, q0 + BM):
            for j in range(k0, k0 + BN):
                if i < T and j < T and i < o + L and j < o + L and m[i, j]:
                    n += 1
        if n == BM * BN:
            out.append((q0, k0, FULL))
        elif n > 0:
            out.append((q0, k0, PARTIAL))
    return sorted(out)


def tile_classes(prefix_lens, suffix_lens, BM: int, BN: int) -> List[Tuple[int, int, int]]:
    """Same result as :func:`tile_classes_bruteforce`, by interval arithmetic (fast enough for full workloads).

    For each row the allowed keys are two intervals (:func:`allowed_pairs_per_row`); the allowed count of a
    (row, kv tile) pair is the sum of the two intersection lengths, and a tile's count is the sum over its rows.
    """
    lay = layout_of(prefix_lens, suffix_lens)
    i1, i2, _ = allowed_pairs_per_row(lay)
    out = []
    for g in range(len(lay.prefix_lens)):
        o = int(lay.group_start[g])
        L = int(lay.group_len[g])
        if L == 0:
            continue
        na, nb = -(-L // BM), -(-L // BN)
        rows = np.arange(o, o + L)
        k0 = o + np.arange(nb, dtype=np.int64) * BN
        k1 = k0 + BN
        def inter(iv):
            lo = np.maximum(iv[rows, 0][:, None], k0[None, :])
            hi = np.minimum(iv[rows, 1][:, None], k1[None, :])
            return np.maximum(hi - lo, 0)
        cnt = inter(i1) + inter(i2)                       # [L, nb]
        pad = na * BM - L
        cnt = np.concatenate([cnt, np.zeros((pad, nb), dtype=cnt.dtype)], axis=0)
        tile = cnt.reshape(na, BM, nb).sum(axis=1)        # [na, nb]
        for a in range(na):
            for b in range(nb):
                n = int(tile[a, b])
                if n == BM * BN:
                    out.append((o + a * BM, int(k0[b]), FULL))
                elif n > 0:
                    out.append((o + a * BM, int(k0[b]), PARTIAL))
    return sorted(out)


# ----------------------------------------------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------------------------------------------
def rope(x, pos, theta: float = 10000.0, inverse: bool = False) -> np.ndarray:
    """Rotate-half rotary embedding in fp64, applied per head at the grouped position ids.

    "prefix_grouper_utils.py" §1: the grouped position ids exist so that every suffix is embedded as if it
    directly followed the prefix. The pages do not name the RoPE variant; this takes the rotate-half form with
    theta=10000: for m < d/2, w_m = theta^(-2m/d), a = pos * w_m,
      y_m       = x_m cos a - x_{m+d/2} sin a
      y_{m+d/2} = x_{m+d/2} cos a + x_m sin a.
    ``inverse`` rotates by -a (the transpose), which maps gradients w.r.t. the rotated tensor back.
    x: [T, H, d]; pos: [T]. Returns fp64 [T, H, d].
    """
    x = np.asarray(x, dtype=np.float64)
    T, H, d = x.shape
    half = d // 2
    m = np.arange(half, dtype=np.float64)
    w = theta ** (-2.0 * m / d)
    a = np.asarray(pos, dtype=np.float64)[:, None] * w[None, :]          # [T, d/2]
    if inverse:
        a = -a
    c = np.cos(a)[:, None, :]
    s = np.sin(a)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ----------------------------------------------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------------------------------------------
def _f64(t):
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def _segment_blocks(lay: PackedLayout, g: int):
    """(query rows [r0, r1), prefix keys [o, o+P), own keys start, segment is prefix) for each segment of group g."""
    o = int(lay.group_start[g])
    p = lay.prefix_lens[g]
    yield o, o + p, o, o + p, True
    b = o + p
    for s in lay.suffix_lens[g]:
        yield b, b + s, o, o + p, False
        b += s


def attention_forward(q, k, v, prefix_lens, suffix_lens, scale: float | None = None, chunk: int = 512,
                      heads: Sequence[int] | None = None, groups: Sequence[int] | None = None):
    """Exact packed attention forward in fp64.

    Per q head h (kv head h // r): s_ij = scale * q_i . k_j over the allowed keys j of row i, with scale = 1/sqrt(d)
    unless given; lse_i = m_i + ln sum_j exp(s_ij - m_i) (natural log of the scaled scores); p_ij = exp(s_ij - lse_i);
    o_i = sum_j p_ij v_j. Rows are processed per segment in chunks of at most ``chunk`` rows. ``heads`` and ``groups``
    restrict the work to a subset (other entries stay zero / -inf): groups are independent, so a group's rows are
    exact on their own.

    Returns (O fp64 [T, Hq, d], LSE fp64 [Hq, T]).
    """
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    T, Hq, d = qf.shape
    Hkv = kf.shape[1]
    r = Hq // Hkv
    sc = 1.0 / math.sqrt(d) if not scale else float(scale)
    lay = layout_of(prefix_lens, suffix_lens)
    O = np.zeros((T, Hq, d))
    LSE = np.full((Hq, T), -np.inf)
    hs = range(Hq) if heads is None else heads
    gs = range(len(lay.prefix_lens)) if groups is None else groups
    for g in gs:
        for r0, r1, pk0, pk1, is_prefix in _segment_blocks(lay, g):
            for c0 in range(r0, r1, chunk):
                c1 = min(c0 + chunk, r1)
                rows = np.arange(c0, c1)
                if is_prefix:
                    keys = np.arange(pk0, c1)
                    mask = keys[None, :] <= rows[:, None]
                else:
                    keys = np.concatenate([np.arange(pk0, pk1), np.arange(r0, c1)])
                    mask = (keys[None, :] < pk1) | (keys[None, :] <= rows[:, None])
                for h in hs:
                    kh = h // r
                    s = sc * (qf[c0:c1, h, :] @ kf[keys, kh, :].T)
                    s = np.where(mask, s, -np.inf)
                    mx = s.max(axis=1, keepdims=True)
                    e = np.exp(s - mx)
                    l = e.sum(axis=1, keepdims=True)
                    lse = mx + np.log(l)
                    p = np.exp(s - lse)
                    O[c0:c1, h, :] = p @ vf[keys, kh, :]
                    LSE[h, c0:c1] = lse[:, 0]
    return O, LSE


def attention_forward_rows(q, k, v, prefix_lens, suffix_lens, rows: Sequence[int], scale: float | None = None,
                           heads: Sequence[int] | None = None):
    """Forward for a sample of single rows (for checks at full workload sizes). Returns (O [n, Hq, d], LSE [Hq, n])."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    T, Hq, d = qf.shape
    Hkv = kf.shape[1]
    r = Hq // Hkv
    sc = 1.0 / math.sqrt(d) if not scale else float(scale)
    lay = layout_of(prefix_lens, suffix_lens)
    hs = list(range(Hq)) if heads is None else list(heads)
    O = np.zeros((len(rows), Hq, d))
    LSE = np.full((Hq, len(rows)), -np.inf)
    for n, i in enumerate(rows):
        g = int(lay.group_of[i])
        o = int(lay.group_start[g])
        p = lay.prefix_lens[g]
        if lay.seg_of[i] == 0:
            keys = np.arange(o, i + 1)
        else:
            keys = np.concatenate([np.arange(o, o + p), np.arange(int(lay.seg_start[i]), i + 1)])
        for h in hs:
            s = sc * (kf[keys, h // r, :] @ qf[i, h, :])
            mx = s.max()
            lse = mx + math.log(np.exp(s - mx).sum())
            O[n, h, :] = np.exp(s - lse) @ vf[keys, h // r, :]
            LSE[h, n] = lse
    return O, LSE


def attention_backward(q, k, v, dout, prefix_lens, suffix_lens, scale: float | None = None, chunk: int = 512,
                       groups: Sequence[int] | None = None, kv_heads: Sequence[int] | None = None):
    """Exact gradient of L = sum(O * dO) w.r.t. q, k, v in fp64 (recomputes the forward).

    D_i = dO_i . o_i (with this function's own fp64 O); dP_ij = dO_i . v_j; dS_ij = p_ij (dP_ij - D_i);
    dQ_i = scale sum_j dS_ij k_j; dK_j = scale sum_{h in the kv head's group} sum_i dS_ij q_i;
    dV_j = sum_{h in group} sum_i p_ij dO_i. ``groups`` / ``kv_heads`` restrict the work (other entries stay zero).
    Returns (dQ, dK, dV) fp64 with the shapes of q, k, v.
    """
    qf, kf, vf, dof = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, Hq, d = qf.shape
    Hkv = kf.shape[1]
    r = Hq // Hkv
    sc = 1.0 / math.sqrt(d) if not scale else float(scale)
    lay = layout_of(prefix_lens, suffix_lens)
    dQ = np.zeros_like(qf)
    dK = np.zeros_like(kf)
    dV = np.zeros_like(vf)
    gs = range(len(lay.prefix_lens)) if groups is None else groups
    khs = range(Hkv) if kv_heads is None else kv_heads
    for g in gs:
        for r0, r1, pk0, pk1, is_prefix in _segment_blocks(lay, g):
            for c0 in range(r0, r1, chunk):
                c1 = min(c0 + chunk, r1)
                rows = np.arange(c0, c1)
                if is_prefix:
                    keys = np.arange(pk0, c1)
                    mask = keys[None, :] <= rows[:, None]
                else:
                    keys = np.concatenate([np.arange(pk0, pk1), np.arange(r0, c1)])
                    mask = (keys[None, :] < pk1) | (keys[None, :] <= rows[:, None])
                for kh in khs:
                    for h in range(kh * r, (kh + 1) * r):
                        qh = qf[c0:c1, h, :]
                        kk = kf[keys, kh, :]
                        vv = vf[keys, kh, :]
                        s = sc * (qh @ kk.T)
                        s = np.where(mask, s, -np.inf)
                        mx = s.max(axis=1, keepdims=True)
                        lse = mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True))
                        p = np.exp(s - lse)
                        o = p @ vv
                        do = dof[c0:c1, h, :]
                        D = (do * o).sum(axis=1, keepdims=True)
                        dp = do @ vv.T
                        ds = p * (dp - D)
                        dQ[c0:c1, h, :] += sc * (ds @ kk)
                        np.add.at(dK[:, kh, :], keys, sc * (ds.T @ qh))
                        np.add.at(dV[:, kh, :], keys, p.T @ do)
    return dQ, dK, dV


# ----------------------------------------------------------------------------------------------------------------
# Unpacked reference (a second, independent path)
# ----------------------------------------------------------------------------------------------------------------
def causal_attention(q, k, v, scale: float | None = None):
    """Standard causal attention on ONE sequence, fp64: rows attend keys 0..i. Returns (O [n,Hq,d], LSE [Hq,n])."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    n, Hq, d = qf.shape
    r = Hq // kf.shape[1]
    sc = 1.0 / math.sqrt(d) if not scale else float(scale)
    O = np.zeros((n, Hq, d))
    LSE = np.zeros((Hq, n))
    mask = np.tril(np.ones((n, n), dtype=bool))
    for h in range(Hq):
        s = np.where(mask, sc * (qf[:, h, :] @ kf[:, h // r, :].T), -np.inf)
        mx = s.max(axis=1, keepdims=True)
        lse = mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True))
        O[:, h, :] = np.exp(s - lse) @ vf[:, h // r, :]
        LSE[h] = lse[:, 0]
    return O, LSE


def causal_attention_backward(q, k, v, dout, scale: float | None = None):
    """Gradient of sum(O * dO) for :func:`causal_attention` (fp64). Returns (dQ, dK, dV)."""
    qf, kf, vf, dof = _f64(q), _f64(k), _f64(v), _f64(dout)
    n, Hq, d = qf.shape
    r = Hq // kf.shape[1]
    sc = 1.0 / math.sqrt(d) if not scale else float(scale)
    dQ, dK, dV = np.zeros_like(qf), np.zeros_like(kf), np.zeros_like(vf)
    mask = np.tril(np.ones((n, n), dtype=bool))
    for h in range(Hq):
        kh = h // r
        s = np.where(mask, sc * (qf[:, h, :] @ kf[:, kh, :].T), -np.inf)
        mx = s.max(axis=1, keepdims=True)
        p = np.exp(s - (mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True))))
        o = p @ vf[:, kh, :]
        D = (dof[:, h, :] * o).sum(axis=1, keepdims=True)
        ds = p * (dof[:, h, :] @ vf[:, kh, :].T - D)
        dQ[:, h, :] = sc * ds @ kf[:, kh, :]
        dK[:, kh, :] += sc * ds.T @ qf[:, h, :]
        dV[:, kh, :] += p.T @ dof[:, h, :]
    return dQ, dK, dV


def _unpacked_runs(lay: PackedLayout, g: int):
    """Packed row indices of each unpacked run of group g: the prefix alone, then P || S_i for every suffix."""
    o = int(lay.group_start[g])
    p = lay.prefix_lens[g]
    pref = np.arange(o, o + p)
    runs = []
    b = o + p
    for s in lay.suffix_lens[g]:
        runs.append(np.concatenate([pref, np.arange(b, b + s)]))
        b += s
    return pref, runs


def unpacked_forward(q, k, v, prefix_lens, suffix_lens, scale=None, theta=None, raw=True):
    """The defining invariant's right-hand side: run plain causal attention on each materialised P||S_i (and on P
    alone for the prefix rows), then scatter the rows back to packed order.

    With ``theta`` set, q/k are the raw (un-rotated) tensors and RoPE is applied per unpacked run at its own
    positions 0..len-1, which is what an unpacked model would do. Returns (O [T,Hq,d], LSE [Hq,T]).
    """
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    lay = layout_of(prefix_lens, suffix_lens)
    T, Hq, d = qf.shape
    O = np.zeros((T, Hq, d))
    LSE = np.zeros((Hq, T))
    for g in range(len(lay.prefix_lens)):
        pref, runs = _unpacked_runs(lay, g)
        p = len(pref)
        for idx, rows_out in [(pref, pref)] + [(run, run[p:]) for run in runs]:
            if len(idx) == 0:
                continue
            qq, kk = qf[idx], kf[idx]
            if theta is not None:
                pos = np.arange(len(idx))
                qq, kk = rope(qq, pos, theta), rope(kk, pos, theta)
            o_run, l_run = causal_attention(qq, kk, vf[idx], scale)
            n_out = len(rows_out)
            O[rows_out] = o_run[len(idx) - n_out:]
            LSE[:, rows_out] = l_run[:, len(idx) - n_out:]
    return O, LSE


def unpacked_backward(q, k, v, dout, prefix_lens, suffix_lens, scale=None):
    """Gradients assembled from unpacked runs (no RoPE; q/k given as the attention inputs).

    Prefix rows: dQ from the prefix-only causal run. Suffix rows: dQ, dK, dV from run P||S_i. Prefix dK/dV:
    sum_i (run i's prefix dK/dV) - (k-1) * (prefix-only run's dK/dV), because the packed loss counts the prefix rows'
    term once while the k runs count it k times. Returns (dQ, dK, dV) fp64.
    """
    qf, kf, vf, dof = _f64(q), _f64(k), _f64(v), _f64(dout)
    lay = layout_of(prefix_lens, suffix_lens)
    dQ, dK, dV = np.zeros_like(qf), np.zeros_like(kf), np.zeros_like(vf)
    for g in range(len(lay.prefix_lens)):
        pref, runs = _unpacked_runs(lay, g)
        p = len(pref)
        kk = len(runs)
        if p:
            dq0, dk0, dv0 = causal_attention_backward(qf[pref], kf[pref], vf[pref], dof[pref], scale)
            dQ[pref] = dq0
            dK[pref] -= (kk - 1) * dk0
            dV[pref] -= (kk - 1) * dv0
        for run in runs:
            if len(run) == 0:
                continue
            dq, dk, dv = causal_attention_backward(qf[run], kf[run], vf[run], dof[run], scale)
            dQ[run[p:]] = dq[p:]
            dK[run] += dk
            dV[run] += dv
    return dQ, dK, dV
