import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Build libpp.so once if it is missing or older than its sources (a no-op otherwise).

    Only a missing toolchain is tolerated: the oracle-only tests still run, and tests that need the library fail
    loudly when they load it. A compile error is raised, so no test can pass against a library built from older
    sources."""
    from shared_prefix_packed_b200 import build as B
    try:
        B._nvcc()
    except RuntimeError:
        yield
        return
    B.build()
    yield


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def random_groups(rng, n_groups, pmax, smax, kmax, allow_zero=True):
    """Small random group descriptors, including the degenerate cases (P=0, k=0, zero-length suffixes)."""
    P, S = [], []
    lo = 0 if allow_zero else 1
    for _ in range(n_groups):
        P.append(int(rng.integers(lo, pmax + 1)))
        k = int(rng.integers(lo, kmax + 1))
        S.append([int(rng.integers(lo, smax + 1)) for _ in range(k)])
    return P, S
