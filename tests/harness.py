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
