"""Seeded synthetic workloads for attention over preference-packed sequences.

This module holds only the recipes that draw group lengths and random tensors. It contains none of the attention
arithmetic (no masks, no position ids, no RoPE, no softmax), so the CPU oracle and the CUDA path can both draw their
inputs from it without sharing any of the method's code.

Packed layout (the one both sides consume): groups are concatenated; group g is its prompt prefix of P_g tokens
followed by its k_g responses S_g1..S_gk, in order ("Preference Packing", abstract; "prefix_grouper_utils.py",
§2 building the grouper from a micro-batch). The pages name no dataset sizes, so the five workloads below are
synthetic stand-ins with the shapes of the pages' use cases (DPO pairs, GRPO groups, long multimodal prefixes,
heterogeneous batched prefill as in the PackInfer abstract).

Distributions (readings where the pages are silent):
  * "uniform[a,b]" draws integers with both ends included;
  * "log-uniform in [a,b]" is exp(U(ln a, ln b)) rounded to the nearest integer;
  * "lognormal, median 1024" uses sigma = 1.0, rounds, and clamps to [1, 16384];
  * "geometric(p=0.3) capped at 16" has support {1, 2, ...}; group sizes are drawn until 64 requests are placed,
    the last group truncated so that the total is exactly 64;
  * "K/V ~ N(0, 0.5)" reads 0.5 as the standard deviation (image-block rows of the long-prefix workload);
  * tensors are drawn in float32 from numpy's PCG64 (``default_rng``) in the order q, k, v, dout and rounded to
    bfloat16 with round-to-nearest-even (the tiny workload stays float32).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Tuple

import numpy as np

__all__ = ["Workload", "WORKLOADS", "group_lengths", "make_inputs", "packed_total", "segment_bounds"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_heads_q: int
    num_heads_kv: int
    head_dim: int
    dtype: str            # "fp32" or "bf16": the dtype of Q/K/V/dO handed to the kernels
    rope: bool            # grouped-position RoPE applied to Q and K before attention
    backward: bool        # the workload runs the backward pass too
    shape_seed: int
    tensor_seed: int
    description: str


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 4, 4, 64, "fp32", False, False, 101, 1001,
                     "2 groups: (P=37; 8,19,32) and (P=64; 4 x U[8,32]); 4 heads, d=64, fp32, forward only"),
    "dpo": Workload("dpo", 32, 8, 128, "bf16", True, True, 102, 1002,
                    "8 groups x (P~U[512,2048]; 2 x U[128,1024]); 32/8 heads, d=128, bf16, RoPE, fwd+bwd"),
    "grpo": Workload("grpo", 32, 8, 128, "bf16", True, True, 103, 1003,
                     "16 groups x (P~U[256,1024]; 8 x logU[64,2048]); 32/8 heads, d=128, bf16, RoPE, fwd+bwd"),
    "longprefix": Workload("longprefix", 28, 4, 128, "bf16", True, True, 104, 1004,
                           "4 groups x (P~U[4096,8192] with K/V rows 0..2879 ~ N(0,0.5^2); k in {2,4} x U[256,512]); "
                           "28/4 heads, d=128, bf16, RoPE, fwd+bwd"),
    "hetero": Workload("hetero", 32, 8, 128, "bf16", True, False, 105, 1005,
                       "64 requests in geometric(0.3)<=16 groups; P~lognormal(median 1024, sigma 1)<=16384; "
                       "S~U[32,4096]; 32/8 heads, d=128, bf16, RoPE, forward only"),
}

IMAGE_BLOCK_ROWS = 2880   # long-prefix workload: first 2880 prefix positions are an "image" block
IMAGE_BLOCK_STD = 0.5


def group_lengths(name: str, seed: int | None = None) -> Tuple[List[int], List[List[int]]]:
    """Draw (prefix_lens, suffix_lens) for workload ``name``. ``seed`` overrides the workload's shape seed."""
    w = WORKLOADS[name]
    rng = np.random.default_rng(w.shape_seed if seed is None else seed)
    P: List[int] = []
    S: List[List[int]] = []
    if name == "tiny":
        P = [37, 64]
        S = [[8, 19, 32], [int(x) for x in rng.integers(8, 33, size=4)]]
    elif name == "dpo":
        for _ in range(8):
            P.append(int(rng.integers(512, 2049)))
            S.append([int(x) for x in rng.integers(128, 1025, size=2)])
    elif name == "grpo":
        for _ in range(16):
            P.append(int(rng.integers(256, 1025)))
            S.append([int(round(math.exp(u))) for u in rng.uniform(math.log(64), math.log(2048), size=8)])
    elif name == "longprefix":
        for _ in range(4):
            P.append(int(rng.integers(4096, 8193)))
            k = int(rng.choice([2, 4]))
            S.append([int(x) for x in rng.integers(256, 513, size=k)])
    elif name == "hetero":
        placed = 0
        while placed < 64:
            g = min(int(rng.geometric(0.3)), 16, 64 - placed)
            placed += g
            p = int(round(float(rng.lognormal(math.log(1024.0), 1.0))))
            P.append(min(max(p, 1), 16384))
            S.append([int(x) for x in rng.integers(32, 4097, size=g)])
    else:  # pragma: no cover - guarded by the dict lookup above
        raise KeyError(name)
    return P, S


def packed_total(prefix_lens, suffix_lens) -> int:
    """Number of packed tokens T = sum over groups of P_g + sum_i S_gi."""
    return int(sum(int(p) + sum(int(s) for s in ss) for p, ss in zip(prefix_lens, suffix_lens)))


def segment_bounds(prefix_lens, suffix_lens) -> np.ndarray:
    """Packed segment boundaries (cu_seqlens, int32[nseg+1]).

    Segments follow the packed order: for each group its prefix, then each suffix. Zero-length segments are kept so
    that the segment count is sum_g (1 + k_g). This is layout bookkeeping (a running sum of lengths), not part of the
    attention arithmetic.
    """
    lens: List[int] = []
    for p, ss in zip(prefix_lens, suffix_lens):
        lens.append(int(p))
        lens.extend(int(s) for s in ss)
    cu = np.zeros(len(lens) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    if cu[-1] >= 2 ** 31:
        raise ValueError("packed length does not fit int32")
    return cu.astype(np.int32)


def _round_bf16(x32: np.ndarray):
    import torch  # local: the oracle-only tests need numpy alone
    return torch.from_numpy(x32).to(torch.bfloat16)


def make_inputs(name: str, prefix_lens, suffix_lens, seed: int | None = None, with_dout: bool | None = None,
                heads: Tuple[int, int, int] | None = None, dtype: str | None = None):
    """Draw q [T,Hq,d], k and v [T,Hkv,d], and (for backward workloads) dout [T,Hq,d].

    Returns a dict of CPU torch tensors (bfloat16, or float32 for fp32 workloads) plus ``"scale_rows"``, the boolean
    mask of packed rows whose K/V were drawn with std 0.5 (long-prefix image block; all False elsewhere).
    ``heads`` = (Hq, Hkv, d) and ``dtype`` override the workload's shape for small test cases.
    """
    import torch
    w = WORKLOADS[name]
    hq, hkv, d = heads if heads is not None else (w.num_heads_q, w.num_heads_kv, w.head_dim)
    dt = dtype or w.dtype
    T = packed_total(prefix_lens, suffix_lens)
    rng = np.random.default_rng(w.tensor_seed if seed is None else seed)
    q = rng.standard_normal((T, hq, d), dtype=np.float32)
    k = rng.standard_normal((T, hkv, d), dtype=np.float32)
    v = rng.standard_normal((T, hkv, d), dtype=np.float32)
    want_dout = w.backward if with_dout is None else with_dout
    dout = rng.standard_normal((T, hq, d), dtype=np.float32) if want_dout else None
    scale_rows = np.zeros(T, dtype=bool)
    if name == "longprefix":
        off = 0
        for p, ss in zip(prefix_lens, suffix_lens):
            n = min(int(p), IMAGE_BLOCK_ROWS)
            scale_rows[off:off + n] = True
            off += int(p) + sum(int(s) for s in ss)
        k[scale_rows] *= IMAGE_BLOCK_STD
        v[scale_rows] *= IMAGE_BLOCK_STD
    out = {}
    for key, arr in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        if arr is None:
            continue
        out[key] = _round_bf16(arr) if dt == "bf16" else torch.from_numpy(arr)
    out["scale_rows"] = scale_rows
    return out


# Vocabulary of the response log-probability read-out: the pages name no model; 151,936 is the vocabulary size of
# the Qwen2-family models that verl-based pipelines like the one on "prefix_grouper_utils.py" commonly train.
LOGPROB_VOCAB = 151936
LOGPROB_LOGIT_STD = 4.0


def make_logits(prefix_lens, suffix_lens, vocab: int = LOGPROB_VOCAB, seed: int = 2001, dtype: str = "bf16",
                std: float = LOGPROB_LOGIT_STD):
    """Synthetic packed logits [T, vocab] ~ N(0, std^2) (rounded to bf16 unless dtype is "fp32") and token ids [T]
    uniform in [0, vocab), both seeded. Returns (logits, token_ids) as CPU torch tensors (token ids int32).

    Rows are drawn in blocks so that large T x vocab shapes do not need an fp32 copy of the whole array.
    """
    import torch
    T = packed_total(prefix_lens, suffix_lens)
    rng = np.random.default_rng(seed)
    ids = torch.from_numpy(rng.integers(0, vocab, size=T).astype(np.int32))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    logits = torch.empty((T, vocab), dtype=tdt)
    block = max(1, (1 << 24) // max(vocab, 1))
    for r0 in range(0, T, block):
        r1 = min(T, r0 + block)
        x = rng.standard_normal((r1 - r0, vocab), dtype=np.float32) * np.float32(std)
        logits[r0:r1] = torch.from_numpy(x).to(tdt)
    return logits, ids
