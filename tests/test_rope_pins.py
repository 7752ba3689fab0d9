"""Pins of the fp64 rotary-embedding oracle (oracle/rope.py), CPU only.

Each pin checks the oracle against something other than its own formula: a hand-worked
value, complex multiplication by a unit phasor (numpy's complex exponential), and the
properties the relocation relies on (identity at zero, composition, norm, and the score's
dependence on the position difference only).
"""
import json
import os

import numpy as np
import pytest

from oracle import rope

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "rope_small.json")))
    y = rope.rotate(np.array(g["x"]), g["pos"], g["base"])
    np.testing.assert_allclose(y, g["y_rotate_half"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("interleaved", [False, True])
def test_matches_complex_phasor(interleaved):
    rng = np.random.default_rng(7)
    d = 128
    x = rng.standard_normal((5, 3, d))
    pos = rng.integers(-300000, 300000, size=(5, 3)).astype(np.float64)
    y = rope.rotate(x, pos, 500000.0, interleaved)
    if interleaved:
        z, lo, hi = x[..., 0::2] + 1j * x[..., 1::2], slice(0, d, 2), slice(1, d, 2)
    else:
        z, lo, hi = x[..., : d // 2] + 1j * x[..., d // 2:], slice(0, d // 2), slice(d // 2, d)
    freq = 500000.0 ** (-np.arange(0, d, 2) / d)
    w = z * np.exp(1j * pos[..., None] * freq)
    np.testing.assert_allclose(y[..., lo], w.real, rtol=0, atol=1e-9)
    np.testing.assert_allclose(y[..., hi], w.imag, rtol=0, atol=1e-9)


def test_zero_offset_is_identity_and_norm_is_kept():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((7, 64))
    assert np.array_equal(rope.relocate(x, np.zeros(7)), x)
    y = rope.relocate(x, rng.integers(0, 10 ** 6, size=7))
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rotations_compose():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((4, 128))
    a, b = rng.integers(-5000, 5000, size=4), rng.integers(-5000, 5000, size=4)
    np.testing.assert_allclose(rope.rotate(rope.rotate(x, a), b), rope.rotate(x, a + b), rtol=0, atol=1e-10)


@pytest.mark.parametrize("interleaved", [False, True])
def test_relocated_query_scores_like_shifted_keys(interleaved):
    # a key cached at canonical position j, a query at true position p = delta + i: the
    # relocated query against the canonical key scores as the query against the key at j + delta
    rng = np.random.default_rng(10)
    d, delta = 128, 131000
    q, k = rng.standard_normal((6, d)), rng.standard_normal((6, d))
    p = delta + rng.integers(0, 4096, size=6)
    j = rng.integers(0, 4096, size=6)
    q_true = rope.rotate(q, p, 10000.0, interleaved)
    lhs = np.sum(rope.relocate(q_true, np.full(6, delta), 10000.0, interleaved) * rope.rotate(k, j, 10000.0, interleaved), -1)
    rhs = np.sum(q_true * rope.rotate(k, j + delta, 10000.0, interleaved), -1)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-9, atol=1e-9)
