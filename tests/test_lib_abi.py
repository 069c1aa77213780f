"""CPU-only checks of the C-ABI boundary: libpp.so builds for sm_100a, loads, and exports every symbol that
include/pp.h declares, with the signatures the binding uses. No compute call is made (there may be no GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "pp.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"PP_API\s+[\w\s\*]+?\b(pp_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("pp_build_meta", "pp_rope", "pp_attn_fwd", "pp_attn_bwd", "pp_meta_bounds", "pp_get_status",
              "pp_last_error", "pp_workspace_bytes", "pp_meta_tiles"):
        assert n in names


def test_library_builds_loads_and_exports_every_declared_symbol():
    from shared_prefix_packed_b200 import build as B
    try:
        B.build()
    except RuntimeError as e:  # pragma: no cover - no toolchain
        pytest.skip(f"nvcc unavailable: {e}")
    L = ctypes.CDLL(B.LIB)
    for name in _declared():
        assert hasattr(L, name), name
    from shared_prefix_packed_b200 import _lib
    assert set(_declared()) == set(_lib.SIGNATURES), "binding and header disagree"
    assert _lib.pp_version().startswith("libpp")


def test_host_only_calls_and_validation():
    """pp_meta_bounds / pp_workspace_bytes run on the host only; invalid sizes are rejected with a message."""
    from shared_prefix_packed_b200 import _lib
    n = _lib.pp_meta_bounds(8, 24, 17801, 32, 8)
    assert n > 8 * 17801
    # backward workspace: (-lse/scale, -D) per q head and row, plus fp32 dK and dV for split key tiles, over the
    # padded rows (T + 256, rounded to 8), each section 256-byte aligned
    rows = (1000 + 256 + 7) & ~7
    a256 = lambda x: (x + 255) & ~255
    want = a256(8 * 32 * rows) + 2 * a256(4 * rows * 8 * 128)
    assert _lib.pp_workspace_bytes(_lib.PP_PASS_BWD, 1000, 32, 8, 128) == want
    with pytest.raises(_lib.PPError, match="INVALID_ARG"):
        _lib.pp_meta_bounds(0, 1, 10, 32, 8)
    with pytest.raises(_lib.PPError, match="INVALID_ARG"):
        _lib.pp_workspace_bytes(_lib.PP_PASS_FWD, 100, 32, 6, 128)      # hq % hkv != 0
    with pytest.raises(_lib.PPError, match="INVALID_ARG"):
        _lib.pp_workspace_bytes(_lib.PP_PASS_FWD, 100, 32, 8, 96)       # unsupported head dim
    with pytest.raises(_lib.PPError, match="INVALID_ARG"):
        _lib.pp_workspace_bytes(_lib.PP_PASS_FWD, -1, 32, 8, 128)


def test_noalloc_scratch_size_matches_the_header():
    """The binding's copy of PP_NOALLOC_SCRATCH_BYTES must equal the header's value (the no-allocation test sizes
    its case against it)."""
    with open(os.path.join(ROOT, "include", "pp.h")) as f:
        m = re.search(r"#define\s+PP_NOALLOC_SCRATCH_BYTES\s+\((\d+)ll\s*<<\s*(\d+)\)", f.read())
    assert m, "PP_NOALLOC_SCRATCH_BYTES not found in pp.h"
    from shared_prefix_packed_b200 import _lib
    assert _lib.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_bwd_ds_bytes_counts_the_nonempty_tile_pairs():
    """pp_bwd_ds_bytes (host only) = 1024 + 32 KiB per backward step, a step being a non-empty (query tile, key
    tile) pair of the mask times the q heads: checked against the oracle's tile set on edge cases and the
    workloads' group lengths."""
    import torch
    import oracle
    import workloads as W
    from shared_prefix_packed_b200 import _lib
    cases = [([3], [[2, 0, 3]]), ([0], [[130, 77]]), ([300], [[]]), ([127, 129, 1], [[1, 255], [3], [0]]),
             ([2100], [[700, 900]]), ([0], [[0]])]
    cases += [W.group_lengths(n) for n in ("dpo", "grpo")]
    for P, S in cases:
        groups = torch.tensor([(p, len(ss)) for p, ss in zip(P, S)], dtype=torch.int32).reshape(-1, 2)
        cu = [0]
        for p, ss in zip(P, S):
            cu.append(cu[-1] + p)
            for x in ss:
                cu.append(cu[-1] + x)
        pairs = len(oracle.tile_classes(P, S, 128, 128))
        for hq, hkv in ((4, 2), (32, 8), (7, 1)):
            got = _lib.pp_bwd_ds_bytes(groups, torch.tensor(cu, dtype=torch.int32), hq, hkv)
            assert got == 1024 + 32768 * pairs * hq, (P, S, hq, hkv)


def test_bwd_ds_bytes_rejects_inconsistent_descriptors():
    """Descriptors that disagree with the segment bounds are refused on the host (no size is returned)."""
    import pytest
    import torch
    from shared_prefix_packed_b200 import _lib
    groups = torch.tensor([[4, 2]], dtype=torch.int32)
    with pytest.raises(_lib.PPError):                      # prefix length 4, but the first segment holds 3 rows
        _lib.pp_bwd_ds_bytes(groups, torch.tensor([0, 3, 5, 9], dtype=torch.int32), 4, 2)
    with pytest.raises(_lib.PPError):                      # two responses declared, one segment present
        _lib.pp_bwd_ds_bytes(groups, torch.tensor([0, 4, 9], dtype=torch.int32), 4, 2)
    with pytest.raises(_lib.PPError):                      # a response with a negative row count
        _lib.pp_bwd_ds_bytes(groups, torch.tensor([0, 4, 3, 9], dtype=torch.int32), 4, 2)
    with pytest.raises(_lib.PPError):                      # hq not a multiple of hkv
        _lib.pp_bwd_ds_bytes(groups, torch.tensor([0, 4, 6, 9], dtype=torch.int32), 3, 2)
    assert _lib.pp_bwd_ds_bytes(groups, torch.tensor([0, 4, 6, 9], dtype=torch.int32), 4, 2) == 1024 + 32768 * 4
