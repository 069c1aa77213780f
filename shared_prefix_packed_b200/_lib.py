"""ctypes binding of libpp's C ABI (include/pp.h): same names, argument marshalling only.

Every step of the path runs in the library's CUDA kernels. torch is used for device memory (tensors are passed as
raw device pointers) and for the current stream. There is no fallback: if libpp.so is missing or fails to load,
every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpp.so")

PP_OK = 0
PP_ERR_INVALID_ARG = -1
PP_ERR_UNSUPPORTED = -2
PP_ERR_CUDA = -3
PP_ERR_DEVICE_TIMEOUT = -4
PP_ERR_WORKSPACE = -5
PP_ERR_DEVICE_INPUT = -6
PP_BF16 = 0
PP_FP32 = 1
PP_PASS_FWD = 0
PP_PASS_BWD = 1

STATUS_NAMES = {0: "PP_OK", -1: "PP_ERR_INVALID_ARG", -2: "PP_ERR_UNSUPPORTED", -3: "PP_ERR_CUDA",
                -4: "PP_ERR_DEVICE_TIMEOUT", -5: "PP_ERR_WORKSPACE", -6: "PP_ERR_DEVICE_INPUT"}

# exported symbol -> (restype, argtypes); the list mirrors include/pp.h
_VP, _I32, _I64, _F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
_I64P = ctypes.POINTER(ctypes.c_int64)
SIGNATURES = {
    "pp_meta_bounds": (_I32, [_I32, _I32, _I64, _I32, _I32, _I64P]),
    "pp_build_meta": (_I32, [_VP, _I32, _VP, _I32, _I64, _I32, _I32, _VP, _VP, _I64, _VP]),
    "pp_meta_tiles": (_I32, [_VP, _I32, _VP, _I64, _VP, _VP]),
    "pp_meta_schedule": (_I32, [_VP, _I32, _VP, _I64, _VP, _VP]),
    "pp_rope": (_I32, [_VP, _VP, _VP, _I64, _I32, _I32, _I32, _F32, _I32, _I32, _VP]),
    "pp_workspace_bytes": (_I32, [_I32, _I64, _I32, _I32, _I32, _I64P]),
    "pp_attn_fwd": (_I32, [_VP, _VP, _VP, _VP, _I64, _I32, _I32, _I32, _F32, _I32, _VP, _VP, _VP, _I64, _VP]),
    "pp_attn_bwd": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I64, _I32, _I32, _I32, _F32, _VP, _VP, _VP, _VP,
                           _I64, _VP]),
    "pp_attn_bwd_noalloc": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I64, _I32, _I32, _I32, _F32, _VP, _VP, _VP,
                                   _VP]),
    "pp_plan_batches": (_I32, [_VP, _I32, _I64, _I32, _VP, _VP, _VP]),
    "pp_decode_workspace_bytes": (_I32, [_VP, _I32, _VP, _I32, _I32, _I64P]),
    "pp_bwd_ds_bytes": (_I32, [_VP, _I32, _VP, _I32, _I32, _I32, _I64P]),
    "pp_decode_attn": (_I32, [_VP, _VP, _VP, _VP, _I32, _VP, _I32, _I64, _I32, _I32, _I32, _F32, _VP, _VP, _VP, _I64,
                              _VP]),
    "pp_pack_batch": (_I32, [_VP, _VP, _I32, _VP, _VP, _I32, _VP, _I32, _VP, _I64, _VP, _VP, _VP, _VP, _VP]),
    "pp_response_logprobs": (_I32, [_VP, _I32, _I64, _VP, _VP, _I64, _F32, _VP, _VP]),
    "pp_selftest_bounded_wait": (_I32, [_I64, _VP, _VP]),
    "pp_get_status": (_I32, [_VP]),
    "pp_last_error": (ctypes.c_char_p, []),
    "pp_version": (ctypes.c_char_p, []),
}

_lock = threading.Lock()
_lib = None


class PPError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib():
    """Load libpp.so once (no fallback: raises OSError if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise OSError(f"libpp.so not built at {LIB_PATH}: run python -m shared_prefix_packed_b200.build")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    if st != PP_OK:
        raise PPError(name, st, lib().pp_last_error().decode())
    return st


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return PP_BF16
    if t.dtype == torch.float32:
        return PP_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------------------------------------------------ calls
def pp_version() -> str:
    return lib().pp_version().decode()


def pp_meta_bounds(num_groups: int, num_segments: int, total_tokens: int, hq: int, hkv: int) -> int:
    out = ctypes.c_int64(0)
    _call("pp_meta_bounds", num_groups, num_segments, total_tokens, hq, hkv, ctypes.byref(out))
    return out.value


def pp_build_meta(groups_d, cu_seqlens_d, total_tokens: int, hq: int, hkv: int, pos_ids_d, meta_d, stream=None):
    """groups_d: int32 [G, 2] (prefix_len, num_suffixes); cu_seqlens_d: int32 [nseg+1]; all on the device."""
    G = groups_d.shape[0]
    nseg = cu_seqlens_d.shape[0] - 1
    _call("pp_build_meta", _ptr(groups_d), G, _ptr(cu_seqlens_d), nseg, total_tokens, hq, hkv, _ptr(pos_ids_d),
          _ptr(meta_d), meta_d.numel() * meta_d.element_size(), _stream(stream))


def pp_meta_tiles(meta_d, which: int, tiles_d, count_d, stream=None):
    cap = tiles_d.numel() // 3
    _call("pp_meta_tiles", _ptr(meta_d), which, _ptr(tiles_d), cap, _ptr(count_d), _stream(stream))


def pp_meta_schedule(meta_d, which: int, records_d, count_d, stream=None):
    cap = records_d.numel() // 5
    _call("pp_meta_schedule", _ptr(meta_d), which, _ptr(records_d), cap, _ptr(count_d), _stream(stream))


def pp_rope(q, k, pos_ids_d, hq: int, hkv: int, d: int, theta: float = 10000.0, inverse: bool = False,
            stream=None):
    ref = q if q is not None else k
    T = ref.shape[0]
    _call("pp_rope", _ptr(q), _ptr(k), _ptr(pos_ids_d), T, hq, hkv, d, float(theta), _dtype_code(ref),
          1 if inverse else 0, _stream(stream))


def pp_workspace_bytes(which: int, T: int, hq: int, hkv: int, d: int) -> int:
    out = ctypes.c_int64(0)
    _call("pp_workspace_bytes", which, T, hq, hkv, d, ctypes.byref(out))
    return out.value


def pp_attn_fwd(q, k, v, meta_d, o, lse, workspace, softmax_scale: float = 0.0, stream=None):
    T, hq, d = q.shape
    hkv = k.shape[1]
    _call("pp_attn_fwd", _ptr(q), _ptr(k), _ptr(v), _ptr(meta_d), T, hq, hkv, d, float(softmax_scale),
          _dtype_code(q), _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
          _stream(stream))


def pp_plan_batches(group_tokens, capacity: int, sort_by_length: bool = True):
    """Host-side batch plan (see pp.h): returns (order, batch_of_group, n_batches) as a list, a list and an int."""
    import numpy as np
    toks = np.ascontiguousarray(np.asarray(group_tokens, dtype=np.int64))
    if toks.ndim != 1 or (toks.size and toks.min() < 0) or int(capacity) < 1:
        raise ValueError("group_tokens must be a 1-D array of non-negative counts and capacity >= 1")
    G = toks.size
    order = np.zeros(max(G, 1), dtype=np.int32)
    batch = np.zeros(max(G, 1), dtype=np.int32)
    nb = ctypes.c_int32(0)
    st = lib().pp_plan_batches(toks.ctypes.data_as(ctypes.c_void_p), G, int(capacity), 1 if sort_by_length else 0,
                               order.ctypes.data_as(ctypes.c_void_p), batch.ctypes.data_as(ctypes.c_void_p),
                               ctypes.byref(nb))
    if st != 0:
        raise PPError("pp_plan_batches", st, "invalid arguments")
    return order[:G].tolist(), batch[:G].tolist(), int(nb.value)


def pp_decode_workspace_bytes(groups_host, cu_host, hq: int) -> int:
    """groups_host: int32 [G, 2] CPU tensor; cu_host: int32 [nseg + 1] CPU tensor."""
    out = ctypes.c_int64(0)
    g = groups_host.contiguous()
    c = cu_host.contiguous()
    _call("pp_decode_workspace_bytes", ctypes.c_void_p(g.data_ptr()), g.shape[0], ctypes.c_void_p(c.data_ptr()),
          c.numel() - 1, hq, ctypes.byref(out))
    return out.value


def pp_bwd_ds_bytes(groups_host, cu_host, hq: int, hkv: int) -> int:
    """Extra backward workspace for the kept-dS path. groups_host: int32 [G, 2] CPU tensor; cu_host: int32 [nseg + 1]
    CPU tensor."""
    out = ctypes.c_int64(0)
    g = groups_host.contiguous()
    c = cu_host.contiguous()
    _call("pp_bwd_ds_bytes", ctypes.c_void_p(g.data_ptr()), g.shape[0], ctypes.c_void_p(c.data_ptr()), c.numel() - 1,
          hq, hkv, ctypes.byref(out))
    return out.value


def pp_decode_attn(q, k_cache, v_cache, groups_d, cu_d, o, lse, workspace, softmax_scale: float = 0.0, stream=None):
    T, hkv, d = k_cache.shape
    hq = q.shape[1]
    _call("pp_decode_attn", _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(groups_d), groups_d.shape[0], _ptr(cu_d),
          cu_d.numel() - 1, T, hq, hkv, d, float(softmax_scale), _ptr(o), _ptr(lse), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))


def pp_pack_batch(prompts, prompt_mask, responses, response_mask, uids, packed_ids, groups, cu_seqlens,
                  sample_offsets, counts, stream=None):
    bs, Lp = prompts.shape
    Lr = responses.shape[1]
    _call("pp_pack_batch", _ptr(prompts), _ptr(prompt_mask), Lp, _ptr(responses), _ptr(response_mask), Lr, _ptr(uids),
          bs, _ptr(packed_ids), packed_ids.numel(), _ptr(groups), _ptr(cu_seqlens), _ptr(sample_offsets),
          _ptr(counts), _stream(stream))


def pp_response_logprobs(logits, token_ids, meta_d, out, temperature: float = 1.0, stream=None):
    T, V = logits.shape
    _call("pp_response_logprobs", _ptr(logits), _dtype_code(logits), V, _ptr(token_ids), _ptr(meta_d), T,
          float(temperature), _ptr(out), _stream(stream))


def pp_attn_bwd(q, k, v, o, lse, dout, meta_d, dq, dk, dv, workspace, softmax_scale: float = 0.0, stream=None):
    T, hq, d = q.shape
    hkv = k.shape[1]
    _call("pp_attn_bwd", _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(meta_d), T, hq, hkv, d,
          float(softmax_scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))


def pp_attn_bwd_noalloc(q, k, v, o, lse, dout, meta_d, dq, dk, dv, softmax_scale: float = 0.0, stream=None):
    """pp_attn_bwd without a workspace argument: the library's built-in 64 MiB scratch is used instead."""
    T, hq, d = q.shape
    hkv = k.shape[1]
    _call("pp_attn_bwd_noalloc", _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(meta_d), T, hq,
          hkv, d, float(softmax_scale), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream))


NOALLOC_SCRATCH_BYTES = 64 << 20


def pp_selftest_bounded_wait(limit_ns: int, waited_ns_d, stream=None):
    """Launch the bounded-wait self-test (a wait on an mbarrier nothing arrives on); waited_ns_d: int64 [1] device."""
    _call("pp_selftest_bounded_wait", int(limit_ns), _ptr(waited_ns_d), _stream(stream))


def pp_get_status(stream=None) -> int:
    """Synchronise the stream and read the device error word; raises PPError on a device-side error."""
    return _call("pp_get_status", _stream(stream))
