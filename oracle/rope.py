"""fp64 rotary position embedding and query relocation -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this module.  It shares no code with the CUDA library.

What it computes.  The RedKnot-MLA review ("RedKnot-MLA: Multi-Head Offline-Online Reuse
for DeepSeek-V4 Long-Context Serving", Summary) describes documents prefilled offline at
canonical position zero whose local-head KV is reused at serving time by rotating the
queries by the negative position offset.  The pages name no rotary convention; the plainest
reading is the standard rotary embedding: dimension pairs rotate by the angle p * theta_i,
theta_i = base ** (-2 i / D), with pairs (i, i + D/2) ("rotate half", the default) or
(2 i, 2 i + 1) ("interleaved").  Relocating a query by an offset delta applies the rotation
for position -delta: a query already rotated to its true position p then scores against a
key rotated to canonical position j exactly as it would against that key at j + delta,
because a rotary score depends only on the difference of the two positions.
"""
from __future__ import annotations

import numpy as np


def _pairs(d: int, interleaved: bool):
    h = d // 2
    if interleaved:
        return np.arange(0, d, 2), np.arange(1, d, 2)
    return np.arange(h), np.arange(h, d)


def rotate(x: np.ndarray, pos, base: float = 10000.0, interleaved: bool = False) -> np.ndarray:
    """Rotary embedding of x [..., D] at positions ``pos`` (broadcast against x's leading
    axes), in fp64: for each pair (a_i, b_i), angle = pos * base ** (-2 i / D),
    a_i' = a_i cos - b_i sin, b_i' = b_i cos + a_i sin."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    lo, hi = _pairs(d, interleaved)
    theta = np.power(float(base), -2.0 * np.arange(d // 2, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    a, b = x[..., lo], x[..., hi]
    out[..., lo] = a * c - b * s
    out[..., hi] = b * c + a * s
    return out


def relocate(q: np.ndarray, delta, base: float = 10000.0, interleaved: bool = False) -> np.ndarray:
    """Query relocation by the offset ``delta``: the rotation for position -delta."""
    return rotate(q, -np.asarray(delta, dtype=np.float64), base, interleaved)
