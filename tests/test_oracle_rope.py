"""Pins for the oracle's rotate-half RoPE (CPU only)."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_rope_golden():
    with open(os.path.join(GOLDEN, "rope.txt")) as f:
        lines = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    for ln in lines:
        hdr, xs, ys = ln.split("|")
        d, pos = (int(t) for t in hdr.split())
        x = np.array([float(t) for t in xs.split()]).reshape(1, 1, d)
        y = np.array([float(t) for t in ys.split()])
        got = oracle.rope(x, np.array([pos]))[0, 0]
        assert np.allclose(got, y, atol=1e-15, rtol=0), (ln, got)


def test_rope_as_complex_multiplication():
    """Each (m, m+d/2) pair is the complex number x_m + i x_{m+d/2} multiplied by exp(i pos theta^(-2m/d))."""
    rng = np.random.default_rng(3)
    T, H, d = 17, 3, 16
    x = rng.standard_normal((T, H, d))
    pos = rng.integers(0, 20000, size=T)
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    freq = np.power(10000.0, -np.arange(0, d, 2) / d)
    w = np.exp(1j * np.outer(pos, freq))[:, None, :]
    zr = z * w
    want = np.concatenate([zr.real, zr.imag], axis=-1)
    assert np.allclose(oracle.rope(x, pos), want, atol=1e-12)


def test_rope_identity_norm_relative_and_inverse():
    rng = np.random.default_rng(4)
    T, H, d = 9, 2, 64
    x = rng.standard_normal((T, H, d))
    y = rng.standard_normal((T, H, d))
    assert np.array_equal(oracle.rope(x, np.zeros(T, dtype=int)), x)
    pos = rng.integers(0, 5000, size=T)
    rx = oracle.rope(x, pos)
    pair = lambda a: a[..., : d // 2] ** 2 + a[..., d // 2:] ** 2
    assert np.allclose(pair(rx), pair(x), atol=1e-12)
    assert np.allclose(oracle.rope(rx, pos, inverse=True), x, atol=1e-12)
    # relative position: rot(x, p) . rot(y, p') depends only on p - p'
    p, pp, shift = 1234, 77, 911
    a = (oracle.rope(x[:1], [p]) * oracle.rope(y[:1], [pp])).sum()
    b = (oracle.rope(x[:1], [p + shift]) * oracle.rope(y[:1], [pp + shift])).sum()
    assert abs(a - b) < 1e-10
