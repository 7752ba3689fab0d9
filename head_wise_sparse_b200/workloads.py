"""Seeded synthetic workloads for head-wise segmented paged attention.

This module only draws numbers and states shapes.  It holds none of the attention
arithmetic: no visibility rule, no page mapping, no softmax.  Both the CUDA path
(tests, bench) and the CPU oracle receive their inputs from here.

Recipe (every value is a pure function of its seed, so any slice can be regenerated):

* bf16 tensors: values are drawn by inverse-CDF sampling of N(0, 1) with 16-bit uniforms.
  ``TABLE[u] = bf16(ndtri((u + 0.5) / 65536) * scale)`` (float64 -> float32 RNE -> bf16 RNE),
  and the uniforms ``u`` are the raw bytes of ``np.random.default_rng(seed).bytes``.
  A tensor is generated in blocks of ``CHUNK`` = 64 token positions; the block holding
  positions [64c, 64c + 64) of sequence ``s`` in layer ``l`` uses
  ``seed = [cfg_id, stream, l, s, c]``, with stream 3 = Q, 4 = K, 5 = V.
* head classes: stream 0; page permutation (free list): stream 1; sequence lengths: stream 2.

The five workloads mirror the shapes of the pages' evaluation models (Mistral-7B,
Llama-3.3-70B and a 128K-context chunked prefill), with synthetic data standing in for
the QA suites the pages measure on.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

CHUNK = 64  # token positions per generation block

STREAM_CLASS, STREAM_PERM, STREAM_LEN, STREAM_Q, STREAM_K, STREAM_V = 0, 1, 2, 3, 4, 5


# ----------------------------------------------------------------------------- bf16 helpers
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


_TABLES: Dict[float, np.ndarray] = {}


def normal_table(scale: float = 1.0) -> np.ndarray:
    """65536-entry bf16 table of N(0, scale^2) quantiles (uint16 bits)."""
    t = _TABLES.get(scale)
    if t is None:
        from scipy.special import ndtri

        q = ndtri((np.arange(65536, dtype=np.float64) + 0.5) / 65536.0) * scale
        t = f32_to_bf16_bits(q.astype(np.float32))
        _TABLES[scale] = t
    return t


def _block(cfg_id: int, stream: int, layer: int, seq: int, c: int, heads: int, d: int, scale: float) -> np.ndarray:
    rng = np.random.default_rng([cfg_id, stream, layer, seq, c])
    u = np.frombuffer(rng.bytes(CHUNK * heads * d * 2), dtype=np.uint16)
    return normal_table(scale)[u].reshape(CHUNK, heads, d)


def rows(cfg_id: int, stream: int, layer: int, seq: int, lo: int, hi: int, heads: int, d: int,
         scale: float = 1.0) -> np.ndarray:
    """bf16 bits [hi - lo, heads, d] for token positions [lo, hi) of one sequence."""
    out = np.empty((max(hi - lo, 0), heads, d), dtype=np.uint16)
    if hi <= lo:
        return out
    for c in range(lo // CHUNK, (hi - 1) // CHUNK + 1):
        b = _block(cfg_id, stream, layer, seq, c, heads, d, scale)
        a0, a1 = max(lo, c * CHUNK), min(hi, (c + 1) * CHUNK)
        out[a0 - lo:a1 - lo] = b[a0 - c * CHUNK:a1 - c * CHUNK]
    return out


# ----------------------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Seq:
    """One sequence of a workload: ``context`` tokens are appended before the measured step;
    the step appends [context, context + new) and queries positions [q_lo, q_hi)."""
    context: int
    new: int
    q_lo: int
    q_hi: int

    @property
    def length(self) -> int:
        return self.context + self.new


@dataclass(frozen=True)
class Workload:
    cfg_id: int
    name: str
    layers: int
    hq: int
    hkv: int
    d: int
    page: int
    window: int
    ring_pages: int
    seqs: Tuple[Seq, ...]
    classes: Tuple[Tuple[int, ...], ...]      # [layers][hkv], 1 = global, 0 = local
    k_scale: float = 1.0
    decode: bool = False
    pool_slack: float = 1.25

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def max_seq_len(self) -> int:
        return max(s.length for s in self.seqs)

    @property
    def max_chunk(self) -> int:
        return max(max(s.new for s in self.seqs), 1)

    def class_array(self) -> np.ndarray:
        return np.asarray(self.classes, dtype=np.uint8).reshape(self.layers, self.hkv)

    def pages_needed(self) -> int:
        """Pool capacity the workload touches: a global head holds every page of its
        sequence, a local head at most ``ring_pages`` pages."""
        n = 0
        for l in range(self.layers):
            for s in self.seqs:
                full = -(-s.length // self.page)
                for h in range(self.hkv):
                    n += full if self.classes[l][h] else min(full, self.ring_pages)
        return n

    @property
    def num_pages(self) -> int:
        return int(math.ceil(self.pool_slack * self.pages_needed())) + 1

    def free_list(self) -> np.ndarray:
        """The caller-given free list: a seeded permutation of all physical page ids."""
        return np.random.default_rng([self.cfg_id, STREAM_PERM]).permutation(self.num_pages).astype(np.int32)

    # -- data ----------------------------------------------------------------
    def q(self, layer: int, seq: int, lo: int, hi: int) -> np.ndarray:
        return rows(self.cfg_id, STREAM_Q, layer, seq, lo, hi, self.hq, self.d)

    def k(self, layer: int, seq: int, lo: int, hi: int) -> np.ndarray:
        return rows(self.cfg_id, STREAM_K, layer, seq, lo, hi, self.hkv, self.d, self.k_scale)

    def v(self, layer: int, seq: int, lo: int, hi: int) -> np.ndarray:
        return rows(self.cfg_id, STREAM_V, layer, seq, lo, hi, self.hkv, self.d)

    def packed(self, which: str, layer: int, ranges: List[Tuple[int, int]]) -> np.ndarray:
        """Varlen-packed rows: the concatenation over sequences b of positions ranges[b]."""
        f = {"q": self.q, "k": self.k, "v": self.v}[which]
        parts = [f(layer, b, lo, hi) for b, (lo, hi) in enumerate(ranges)]
        return np.concatenate(parts, axis=0) if parts else np.zeros((0,), np.uint16)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _one_global(cfg_id: int, hkv: int, layer: Optional[int] = None) -> Tuple[int, ...]:
    seed = [cfg_id, STREAM_CLASS] if layer is None else [cfg_id, STREAM_CLASS, layer]
    g = int(np.random.default_rng(seed).integers(hkv))
    return tuple(1 if h == g else 0 for h in range(hkv))


def _tiny() -> Workload:
    L = 1024
    return Workload(1, "tiny_prefill_L1024_D64", 1, 8, 4, 64, 16, 128, L // 16,
                    (Seq(0, L, 0, L),), ((1, 0, 0, 0),))


def _mistral() -> Workload:
    L = 8192
    return Workload(2, "mistral7b_prefill_L8192", 1, 32, 8, 128, 64, 1024, L // 64,
                    (Seq(0, L, 0, L),), (_one_global(2, 8),), k_scale=1.0 / math.sqrt(128.0))


def _llama() -> Workload:
    lens = np.random.default_rng([3, STREAM_LEN]).integers(8192, 32768, endpoint=True, size=4)
    seqs = tuple(Seq(0, int(n), 0, int(n)) for n in lens)
    return Workload(3, "llama70b_varlen_prefill_4x4layers", 4, 64, 8, 128, 64, 2048, 32768 // 64,
                    seqs, tuple(_one_global(3, 8, l) for l in range(4)))


def _decode() -> Workload:
    ctx = 32767
    seqs = tuple(Seq(ctx, 1, ctx, ctx + 1) for _ in range(64))
    return Workload(4, "decode_64x32k", 1, 64, 8, 128, 64, 4096, 65, seqs, (_one_global(4, 8),), decode=True)


def _chunk128k() -> Workload:
    g = set(int(x) for x in np.random.default_rng([5, STREAM_CLASS]).choice(32, 4, replace=False))
    cls = tuple(1 if h in g else 0 for h in range(32))
    return Workload(5, "mha_chunked_prefill_128k", 1, 32, 32, 128, 64, 4096, 129,
                    (Seq(126976, 4096, 126976, 131072),), (cls,))


CONFIGS: Dict[str, Workload] = {w.name: w for w in (_tiny(), _mistral(), _llama(), _decode(), _chunk128k())}
BY_ID: Dict[int, Workload] = {w.cfg_id: w for w in CONFIGS.values()}


def random_small(seed: int, *, max_len: int = 64, d: int = 16) -> Workload:
    """A small random workload (for brute-force comparisons): random GQA group, page size,
    window, ring size, head classes, sequence count and lengths, query chunk."""
    rng = np.random.default_rng([1000, seed])
    hkv = int(rng.integers(1, 4))
    g = int(rng.choice([1, 2, 4]))
    page = int(rng.choice([2, 4, 8, 16]))
    window = int(rng.integers(1, max_len + 8))
    nseq = int(rng.integers(1, 4))
    seqs = []
    for _ in range(nseq):
        n = int(rng.integers(1, max_len + 1))
        ctx = int(rng.integers(0, n))
        new = n - ctx
        q_lo = ctx + int(rng.integers(0, new))
        seqs.append(Seq(ctx, new, q_lo, n))
    max_new = max(s.new for s in seqs)
    max_len_seen = max(s.length for s in seqs)
    ring = min(-(-max_len_seen // page), -(-(window + max_new - 1) // page) + 1 + int(rng.integers(0, 2)))
    cls = tuple(tuple(int(x) for x in rng.integers(0, 2, size=hkv)) for _ in range(1))
    return Workload(100 + seed, f"random_small_{seed}", 1, hkv * g, hkv, d, page, window, max(ring, 1),
                    tuple(seqs), cls)
