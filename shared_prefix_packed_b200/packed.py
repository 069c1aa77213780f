"""PackedBatch: one packed batch's device buffers and the four library calls in order.

Allocation (torch) and argument marshalling only; every step runs in libpp's kernels.
"""
from __future__ import annotations

from typing import Sequence

import torch

from . import _lib


class PackedBatch:
    """Group descriptors on the device, the schedule built by ``pp_build_meta``, and reusable workspaces.

    prefix_lens[g] = P_g, suffix_lens[g] = [S_g1, ..., S_gk]; the packed order is each group's prefix, then its
    responses ("prefix_grouper_utils.py" section 2).
    """

    def __init__(self, prefix_lens: Sequence[int], suffix_lens: Sequence[Sequence[int]], hq: int, hkv: int, d: int,
                 device="cuda", stream=None, ds_budget_bytes=None):
        """ds_budget_bytes: most device memory the backward may take to keep every step's dS tile (the faster dq
        path, ``pp_bwd_ds_bytes``); None means half of the memory free when the backward workspace is first made,
        0 disables it. Either way the results are the same."""
        self.hq, self.hkv, self.d = hq, hkv, d
        self.ds_budget_bytes = ds_budget_bytes
        self.device = torch.device(device)
        groups, lens = [], []
        for p, ss in zip(prefix_lens, suffix_lens):
            groups.append((int(p), len(ss)))
            lens.append(int(p))
            lens.extend(int(s) for s in ss)
        self.T = int(sum(lens))
        cu = [0]
        for n in lens:
            cu.append(cu[-1] + n)
        self.groups_host = torch.tensor(groups, dtype=torch.int32).reshape(-1, 2)
        self.cu_host = torch.tensor(cu, dtype=torch.int32)
        self.groups = self.groups_host.to(self.device)
        self.cu_seqlens = self.cu_host.to(self.device)
        nbytes = _lib.pp_meta_bounds(len(groups), len(lens), self.T, hq, hkv)
        self.meta = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.pos_ids = torch.empty(max(self.T, 1), dtype=torch.int32, device=self.device)
        self.ws_fwd = torch.empty(_lib.pp_workspace_bytes(_lib.PP_PASS_FWD, self.T, hq, hkv, d), dtype=torch.uint8,
                                  device=self.device)
        self._ws_bwd = None
        self.build(stream)

    def build(self, stream=None):
        _lib.pp_build_meta(self.groups, self.cu_seqlens, self.T, self.hq, self.hkv, self.pos_ids, self.meta, stream)

    @property
    def ws_bwd(self):
        """Backward workspace: the base scratch plus room to keep every step's dS tile (the faster dq path)."""
        if self._ws_bwd is None:
            n = _lib.pp_workspace_bytes(_lib.PP_PASS_BWD, self.T, self.hq, self.hkv, self.d)
            if self.d == 128:
                extra = _lib.pp_bwd_ds_bytes(self.groups_host, self.cu_host, self.hq, self.hkv)
                budget = self.ds_budget_bytes
                if budget is None:
                    budget = torch.cuda.mem_get_info(self.device)[0] // 2
                if extra <= budget:
                    n += extra
            self._ws_bwd = torch.empty(n, dtype=torch.uint8, device=self.device)
        return self._ws_bwd

    def rope(self, q, k, theta: float = 10000.0, inverse: bool = False, stream=None):
        _lib.pp_rope(q, k, self.pos_ids, self.hq, self.hkv, self.d, theta, inverse, stream)

    def forward(self, q, k, v, out=None, lse=None, softmax_scale: float = 0.0, stream=None):
        o = torch.empty_like(q) if out is None else out
        l = torch.empty(self.hq, self.T, dtype=torch.float32, device=q.device) if lse is None else lse
        _lib.pp_attn_fwd(q, k, v, self.meta, o, l, self.ws_fwd, softmax_scale, stream)
        return o, l

    def backward(self, q, k, v, o, lse, dout, dq=None, dk=None, dv=None, softmax_scale: float = 0.0, stream=None):
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        _lib.pp_attn_bwd(q, k, v, o, lse, dout, self.meta, dq, dk, dv, self.ws_bwd, softmax_scale, stream)
        return dq, dk, dv

    def response_logprobs(self, logits, token_ids, temperature: float = 1.0, out=None, stream=None):
        """Log-probability of every response token from the packed logits [T, V] (0 where no row predicts it)."""
        lp = torch.empty(self.T, dtype=torch.float32, device=logits.device) if out is None else out
        _lib.pp_response_logprobs(logits, token_ids, self.meta, lp, temperature, stream)
        return lp

    def decode(self, q, k_cache, v_cache, softmax_scale: float = 0.0, out=None, lse=None, stream=None):
        """One decoding step over this layout as a KV cache: q [n_resp, hq, d], one query per response (its newest
        token, the last row of its segment); returns (o [n_resp, hq, d], lse [hq, n_resp])."""
        n_resp = self.cu_host.numel() - 1 - self.groups_host.shape[0]
        o = torch.empty_like(q) if out is None else out
        l = torch.empty(self.hq, n_resp, dtype=torch.float32, device=q.device) if lse is None else lse
        if getattr(self, "_ws_dec", None) is None:
            n = _lib.pp_decode_workspace_bytes(self.groups_host, self.cu_host, self.hq)
            self._ws_dec = torch.empty(n, dtype=torch.uint8, device=self.device)
        _lib.pp_decode_attn(q, k_cache, v_cache, self.groups, self.cu_seqlens, o, l, self._ws_dec, softmax_scale,
                            stream)
        return o, l

    def tiles(self, which: int, stream=None):
        """Expanded schedule as a sorted list of (q_row0, kv_row0, class) (test and inspection helper)."""
        count = torch.zeros(1, dtype=torch.int32, device=self.device)
        _lib.pp_meta_tiles(self.meta, which, torch.empty(3, dtype=torch.int32, device=self.device), count, stream)
        n = int(count.item())
        buf = torch.empty(3 * max(n, 1), dtype=torch.int32, device=self.device)
        _lib.pp_meta_tiles(self.meta, which, buf, count, stream)
        rows = buf[: 3 * n].view(-1, 3).cpu().tolist()
        return sorted(tuple(r) for r in rows)

    def schedule(self, which: int, stream=None):
        """The executed work list as rows (item, q_row0, kv_row0, class, split), sorted by item (test helper)."""
        count = torch.zeros(1, dtype=torch.int32, device=self.device)
        _lib.pp_meta_schedule(self.meta, which, torch.empty(5, dtype=torch.int32, device=self.device), count,
                              stream)
        n = int(count.item())
        buf = torch.empty(5 * max(n, 1), dtype=torch.int32, device=self.device)
        _lib.pp_meta_schedule(self.meta, which, buf, count, stream)
        rows = buf[: 5 * n].view(-1, 5).cpu().tolist()
        return sorted(tuple(r) for r in rows)


def pack_batch(prompts, prompt_mask, responses, response_mask, uids, stream=None):
    """Pack an ungrouped micro-batch on the device (pp_pack_batch): returns (packed_ids [T], prefix_lens,
    suffix_lens, cu_seqlens [nseg + 1], sample_offsets [bs, 2]). The lengths come back to the host with one small
    synchronising copy, so they can be handed to PackedBatch."""
    dev = prompts.device
    bs, Lp = prompts.shape
    Lr = responses.shape[1]
    packed = torch.empty(max(1, bs * (Lp + Lr)), dtype=torch.int32, device=dev)
    groups = torch.empty(max(1, bs), 2, dtype=torch.int32, device=dev)
    cu = torch.empty(2 * bs + 1, dtype=torch.int32, device=dev)
    offsets = torch.empty(max(1, bs), 2, dtype=torch.int32, device=dev)
    counts = torch.zeros(3, dtype=torch.int32, device=dev)
    _lib.pp_pack_batch(prompts.to(torch.int32), prompt_mask.to(torch.uint8), responses.to(torch.int32),
                       response_mask.to(torch.uint8), uids.to(torch.int64), packed, groups, cu, offsets, counts,
                       stream)
    G, nseg, T = (int(x) for x in counts.cpu())
    g = groups[:G].cpu().tolist()
    P = [int(p) for p, _ in g]
    sizes = [int(k) for _, k in g]
    cu_h = cu[:nseg + 1]
    lens = (cu_h[1:] - cu_h[:-1]).cpu().tolist()
    S, seg = [], 0
    for k in sizes:
        S.append([int(x) for x in lens[seg + 1:seg + 1 + k]])
        seg += 1 + k
    return packed[:T], P, S, cu_h, offsets[:bs]
