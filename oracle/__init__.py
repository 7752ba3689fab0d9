"""fp64 CPU oracle for head-wise segmented paged attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package.  It shares no code with the CUDA library; the C source it wraps
(``segkv_oracle.c``) states what it computes and which passage each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "segkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsegkv_oracle.so")
_lib = None

ORC_OK, ORC_ERR_ARG, ORC_ERR_OUT_OF_PAGES, ORC_ERR_NOT_RESIDENT = 0, 1, 3, 4


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with the host C compiler (plain C11, pthreads, libm)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.orc_create.restype = P
        lib.orc_create.argtypes = [I] * 10 + [P, P]
        lib.orc_destroy.argtypes = [P]
        lib.orc_page_table.restype = P
        lib.orc_page_table.argtypes = [P]
        lib.orc_max_lp.argtypes = [P]
        lib.orc_cursor.argtypes = [P]
        lib.orc_seq_len.argtypes = [P, I, I]
        lib.orc_append.argtypes = [P, I, I, P, P, P, P, P]
        lib.orc_fork.argtypes = [P, I, I]
        lib.orc_attention.argtypes = [P, I, I, P, P, P, P, D, P, I64, P, P, P, I]
        lib.orc_router_scores.argtypes = [P, I, I, P, P, P, P, D, P, I]
        lib.orc_lpt_items.restype = I64
        lib.orc_lpt_items.argtypes = [I, P, P, I, P, I, I, I, P, I64]
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class Oracle:
    """Own page allocator, ring, pools and page tables; fp64 attention per query row."""

    def __init__(self, *, layers: int, hq: int, hkv: int, d: int, page: int, window: int, ring: int,
                 max_seqs: int, max_seq_len: int, num_pages: int, classes: np.ndarray, free_list: np.ndarray):
        self.lib = _load()
        self.hq, self.hkv, self.d, self.layers, self.max_seqs = hq, hkv, d, layers, max_seqs
        self._cls = np.ascontiguousarray(np.asarray(classes, dtype=np.uint8).reshape(layers, hkv))
        self._free = _i32(free_list)
        assert self._free.size == num_pages
        self.h = self.lib.orc_create(layers, hq, hkv, d, page, window, ring, max_seqs, max_seq_len, num_pages,
                                     _ptr(self._cls), _ptr(self._free))
        if not self.h:
            raise OracleError("orc_create rejected the configuration")

    @classmethod
    def for_workload(cls, w, max_seqs: Optional[int] = None, free_list: Optional[np.ndarray] = None) -> "Oracle":
        return cls(layers=w.layers, hq=w.hq, hkv=w.hkv, d=w.d, page=w.page, window=w.window, ring=w.ring_pages,
                   max_seqs=max_seqs or len(w.seqs), max_seq_len=w.max_seq_len, num_pages=w.num_pages,
                   classes=w.class_array(), free_list=w.free_list() if free_list is None else free_list)

    def __del__(self):
        if getattr(self, "h", None):
            self.lib.orc_destroy(self.h)
            self.h = None

    @property
    def max_lp(self) -> int:
        return self.lib.orc_max_lp(self.h)

    @property
    def cursor(self) -> int:
        return self.lib.orc_cursor(self.h)

    def seq_len(self, layer: int, seq: int) -> int:
        return self.lib.orc_seq_len(self.h, layer, seq)

    def page_table(self) -> np.ndarray:
        n = self.layers * self.max_seqs * self.hkv * self.max_lp
        buf = (ctypes.c_int32 * n).from_address(self.lib.orc_page_table(self.h))
        return np.frombuffer(buf, dtype=np.int32).copy().reshape(self.layers, self.max_seqs, self.hkv, self.max_lp)

    def append(self, layer: int, seq_ids: Sequence[int], start: Sequence[int], count: Sequence[int],
               k_new: np.ndarray, v_new: np.ndarray) -> None:
        k = np.ascontiguousarray(k_new, dtype=np.uint16)
        v = np.ascontiguousarray(v_new, dtype=np.uint16)
        s, st, c = _i32(seq_ids), _i32(start), _i32(count)
        assert k.size == int(c.sum()) * self.hkv * self.d and v.size == k.size
        rc = self.lib.orc_append(self.h, layer, len(s), _ptr(s), _ptr(st), _ptr(c), _ptr(k), _ptr(v))
        if rc:
            raise OracleError(f"orc_append failed with {rc}")

    def fork(self, src: int, dst: int) -> None:
        """The empty sequence dst takes src's pages (shared) and length in every layer."""
        rc = self.lib.orc_fork(self.h, src, dst)
        if rc != ORC_OK:
            raise OracleError(f"orc_fork failed: {rc}")

    def router_scores(self, layer: int, seq_ids: Sequence[int], q_start: Sequence[int], q_len: Sequence[int],
                      q: np.ndarray, scale: Optional[float] = None, threads: Optional[int] = None) -> np.ndarray:
        """Attention mass each token of the call's query range receives, summed over query
        heads and the call's queries (fp64 [sum(q_len)], packed like q)."""
        s, qs, ql = _i32(seq_ids), _i32(q_start), _i32(q_len)
        qq = np.ascontiguousarray(q, dtype=np.uint16)
        T = int(ql.sum())
        assert qq.size == T * self.hq * self.d
        out = np.zeros(max(T, 1))
        sc = float(scale) if scale is not None else 1.0 / np.sqrt(self.d)
        rc = self.lib.orc_router_scores(self.h, layer, len(s), _ptr(s), _ptr(qs), _ptr(ql), _ptr(qq), sc, _ptr(out),
                                        threads or host_threads())
        if rc:
            raise OracleError(f"orc_router_scores failed with {rc}")
        return out[:T]

    def attention(self, layer: int, seq_ids: Sequence[int], q_start: Sequence[int], q_len: Sequence[int],
                  q: np.ndarray, scale: Optional[float] = None, rows: Optional[np.ndarray] = None,
                  threads: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """Returns (out fp64 [T, hq, d], lse fp64 [T, hq], counts u64 [nseq, hq]).  With ``rows``
        (packed token * hq + q head) only those rows are computed and written; the other
        entries are NaN, except in outputs above 2^25 elements, where they are left unwritten
        (undefined) so that sampling a few rows of a large call does not cost a fill of the
        whole output."""
        s, qs, ql = _i32(seq_ids), _i32(q_start), _i32(q_len)
        qq = np.ascontiguousarray(q, dtype=np.uint16)
        T = int(ql.sum())
        assert qq.size == T * self.hq * self.d
        fill = rows is not None and T * self.hq * self.d <= (1 << 25)
        out = np.full((T, self.hq, self.d), np.nan) if fill else np.empty((T, self.hq, self.d))
        lse = np.full((T, self.hq), np.nan) if fill else np.empty((T, self.hq))
        counts = np.zeros((len(s), self.hq), dtype=np.uint64)
        rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
        sc = float(scale) if scale is not None else 1.0 / np.sqrt(self.d)
        rc = self.lib.orc_attention(self.h, layer, len(s), _ptr(s), _ptr(qs), _ptr(ql), _ptr(qq), sc, _ptr(rr),
                                    0 if rr is None else rr.size, _ptr(out), _ptr(lse), _ptr(counts),
                                    threads or host_threads())
        if rc:
            raise OracleError(f"orc_attention failed with {rc}")
        return out, lse, counts


def topk_rows(scores: np.ndarray, q_len: Sequence[int], k: Sequence[int]) -> np.ndarray:
    """Top-k routing over packed per-token scores (reading: the k highest scores of each
    sequence, equal scores by lower position first; rows returned ascending, sequences in
    call order).  Returns int32 packed rows."""
    out, off = [], 0
    for n, kk in zip(q_len, k):
        n, kk = int(n), int(kk)
        if not 0 <= kk <= n:
            raise OracleError("k outside [0, q_len]")
        s = np.asarray(scores[off:off + n])
        order = np.lexsort((np.arange(n), -s))  # score descending, then position ascending
        out.append(np.sort(order[:kk]) + off)
        off += n
    return np.concatenate(out).astype(np.int32) if out else np.zeros(0, np.int32)


def lpt_items(q_start, q_len, classes_layer, window: int, tile_pos: int, bn: int) -> np.ndarray:
    """Longest-processing-time-first work list: int32 rows (seq index, KV head, tile, cost)."""
    lib = _load()
    qs, ql = _i32(q_start), _i32(q_len)
    cls = np.ascontiguousarray(np.asarray(classes_layer, dtype=np.uint8))
    cap = int(sum(len(cls) * (-(-int(n) // tile_pos)) for n in ql))
    out = np.zeros((max(cap, 1), 4), dtype=np.int32)
    n = lib.orc_lpt_items(len(qs), _ptr(qs), _ptr(ql), len(cls), _ptr(cls), window, tile_pos, bn, _ptr(out), cap)
    if n < 0:
        raise OracleError("orc_lpt_items: capacity")
    return out[:n]
