"""Brute-force reference for tiny cases: numpy fp64, no paging at all.

It materialises the full per-head mask [Hq, Lq, L] from the visibility rule and runs a
dense masked softmax over contiguous K/V.  Used only to pin the oracle (which reads K/V
through its own page tables and ring).
"""
from __future__ import annotations

import numpy as np

from head_wise_sparse_b200.workloads import bf16_bits_to_f32


def dense_masked_attention(q_bits, k_bits, v_bits, q_pos, classes, window, scale):
    """q_bits [Lq, Hq, D], k/v_bits [L, Hkv, D] (positions 0..L-1), q_pos [Lq] absolute positions.
    Returns out [Lq, Hq, D], lse [Lq, Hq], counts [Hq] (fp64 / int)."""
    q = bf16_bits_to_f32(q_bits).astype(np.float64)
    k = bf16_bits_to_f32(k_bits).astype(np.float64)
    v = bf16_bits_to_f32(v_bits).astype(np.float64)
    Lq, Hq, D = q.shape
    L, Hkv, _ = k.shape
    G = Hq // Hkv
    key = np.arange(L)[None, :]
    qp = np.asarray(q_pos)[:, None]
    mask = np.zeros((Hq, Lq, L), dtype=bool)
    for h in range(Hq):
        if classes[h // G]:
            mask[h] = key <= qp
        else:
            mask[h] = (key <= qp) & (key > qp - window)
    out = np.zeros((Lq, Hq, D))
    lse = np.zeros((Lq, Hq))
    for h in range(Hq):
        kv = h // G
        s = scale * q[:, h, :] @ k[:, kv, :].T          # [Lq, L]
        s = np.where(mask[h], s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        out[:, h, :] = (e / z) @ v[:, kv, :]
        lse[:, h] = (m + np.log(z))[:, 0]
    counts = mask.sum(axis=(1, 2))
    return out, lse, counts


def dense_received_attention(q_bits, k_bits, q_pos, key_lo, key_hi, classes, window, scale):
    """Attention mass received by the keys at positions [key_lo, key_hi): for each, the sum
    over query heads and query rows of the dense masked softmax weight.  q_bits [Lq, Hq, D]
    at absolute positions q_pos; k_bits [L, Hkv, D] at positions 0..L-1.  fp64 [key_hi - key_lo]."""
    q = bf16_bits_to_f32(q_bits).astype(np.float64)
    k = bf16_bits_to_f32(k_bits).astype(np.float64)
    Lq, Hq, _ = q.shape
    L, Hkv, _ = k.shape
    G = Hq // Hkv
    key = np.arange(L)[None, :]
    qp = np.asarray(q_pos)[:, None]
    total = np.zeros(L)
    for h in range(Hq):
        kv = h // G
        mask = key <= qp if classes[kv] else (key <= qp) & (key > qp - window)
        s = np.where(mask, scale * q[:, h, :] @ k[:, kv, :].T, -np.inf)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        total += (e / e.sum(axis=1, keepdims=True)).sum(axis=0)
    return total[key_lo:key_hi]
