"""Replay of a workload's append/attention calls, shared by the oracle and GPU tests.

It decides only the order of calls (which tokens are appended by which call); every
number comes from head_wise_sparse_b200.workloads and every result from the side under
test.
"""
from __future__ import annotations

from typing import Iterator, List, Sequence, Tuple

import numpy as np

from head_wise_sparse_b200.workloads import Workload


def context_calls(w: Workload, ctx_chunk: int) -> Iterator[Tuple[List[int], List[int], List[int]]]:
    """Context appends: all sequences in each call, ``ctx_chunk`` tokens per call."""
    top = max(s.context for s in w.seqs)
    lo = 0
    while lo < top:
        hi = min(lo + ctx_chunk, top)
        ids, st, cnt = [], [], []
        for b, s in enumerate(w.seqs):
            a, e = min(lo, s.context), min(hi, s.context)
            if e > a:
                ids.append(b)
                st.append(a)
                cnt.append(e - a)
        if ids:
            yield ids, st, cnt
        lo = hi


def step_append(w: Workload) -> Tuple[List[int], List[int], List[int]]:
    ids = [b for b, s in enumerate(w.seqs) if s.new > 0]
    return ids, [w.seqs[b].context for b in ids], [w.seqs[b].new for b in ids]


def step_queries(w: Workload) -> Tuple[List[int], List[int], List[int]]:
    ids = [b for b, s in enumerate(w.seqs) if s.q_hi > s.q_lo]
    return ids, [w.seqs[b].q_lo for b in ids], [w.seqs[b].q_hi - w.seqs[b].q_lo for b in ids]


def kv_for_call(w: Workload, layer: int, ids: Sequence[int], st: Sequence[int], cnt: Sequence[int]):
    k = np.concatenate([w.k(layer, b, a, a + n) for b, a, n in zip(ids, st, cnt)], axis=0)
    v = np.concatenate([w.v(layer, b, a, a + n) for b, a, n in zip(ids, st, cnt)], axis=0)
    return k, v


def q_for_call(w: Workload, layer: int, ids, q_start, q_len):
    return np.concatenate([w.q(layer, b, a, a + n) for b, a, n in zip(ids, q_start, q_len)], axis=0)


def oracle_replay(w: Workload, layer: int, oracle, ctx_chunk: int = 4096) -> None:
    """Issue the workload's appends for ``layer`` on an oracle instance."""
    for ids, st, cnt in context_calls(w, ctx_chunk):
        k, v = kv_for_call(w, layer, ids, st, cnt)
        oracle.append(layer, ids, st, cnt, k, v)
    ids, st, cnt = step_append(w)
    if ids:
        k, v = kv_for_call(w, layer, ids, st, cnt)
        oracle.append(layer, ids, st, cnt, k, v)


# -- the CUDA side ------------------------------------------------------------------------
def to_dev(bits: np.ndarray, device="cuda"):
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on the device (bit-exact)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def bf16_to_f64(t) -> np.ndarray:
    import torch

    return t.detach().to("cpu").view(torch.int16).numpy().view(np.uint16).astype(np.uint32).__lshift__(16) \
        .view(np.float32).astype(np.float64)


def make_kv(w: Workload, free_list=None, max_seqs=None, ws_tokens=None, device="cuda"):
    from head_wise_sparse_b200.segkv import SegKV

    return SegKV(num_layers=w.layers, num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, page_size=w.page,
                 window=w.window, head_class=w.class_array(), num_pages=w.num_pages,
                 free_list=w.free_list() if free_list is None else free_list, max_seqs=max_seqs or len(w.seqs),
                 max_seq_len=w.max_seq_len, ring_pages=w.ring_pages, max_chunk=w.max_chunk,
                 ws_batch=max_seqs or len(w.seqs),
                 ws_tokens=ws_tokens or max(sum(s.q_hi - s.q_lo for s in w.seqs), 1), device=device)


def gpu_replay(w: Workload, layer: int, kv, ctx_chunk: int = 4096, step: bool = True) -> None:
    """Issue the workload's appends for ``layer`` through the library."""
    calls = list(context_calls(w, ctx_chunk))
    if step:
        calls.append(step_append(w))
    for ids, st, cnt in calls:
        if not ids:
            continue
        k, v = kv_for_call(w, layer, ids, st, cnt)
        kv.append(layer, ids, st, cnt, to_dev(k), to_dev(v))


def within_tolerance(out, ref, atol=8e-3, rtol=1e-2):
    """Elementwise |out - ref| <= atol + rtol |ref|; returns (ok, worst excess, index)."""
    err = np.abs(out - ref) - (atol + rtol * np.abs(ref))
    i = int(np.argmax(err))
    return bool(err.flat[i] <= 0), float(err.flat[i]), np.unravel_index(i, err.shape)
