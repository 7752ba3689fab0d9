"""Python binding of libsegkv.so (declared in include/segkv.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels.  PyTorch is used to own device
memory and to name the current stream.  There is no fallback: if the library is missing
or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsegkv.so")

SEGKV_OK = 0
STATUS = {
    0: "SEGKV_OK", 1: "SEGKV_ERR_INVALID_ARG", 2: "SEGKV_ERR_UNSUPPORTED", 3: "SEGKV_ERR_OUT_OF_PAGES",
    4: "SEGKV_ERR_RING_TOO_SMALL", 5: "SEGKV_ERR_WORKSPACE", 6: "SEGKV_ERR_CUDA", 7: "SEGKV_ERR_DEVICE_BOUNDS",
    8: "SEGKV_ERR_DEVICE_TIMEOUT",
}
EXPORTS = [
    "segkv_create", "segkv_destroy", "segkv_ring_pages", "segkv_max_lp", "segkv_seq_len", "segkv_pages_used",
    "segkv_workspace_bytes", "segkv_reset", "segkv_append", "segkv_prefill_attn", "segkv_plan_prefill",
    "segkv_decode_attn", "segkv_device_status", "segkv_strerror", "segkv_last_error",
    "segkv_decode_attn_noalloc", "segkv_relocate_q", "segkv_fork", "segkv_decode_step",
    "segkv_router_topk", "segkv_prefill_attn_2src", "segkv_prefill_append", "segkv_debug_set",
]

# keys of segkv_debug_set (test hooks; see include/segkv.h)
DEBUG_WAIT_LIMIT, DEBUG_STALL_NEXT_PREFILL, DEBUG_PREFILL_ORDER = 1, 2, 3


class SegkvError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("page_size", ctypes.c_int), ("window", ctypes.c_int),
        ("ring_pages", ctypes.c_int), ("max_seqs", ctypes.c_int), ("max_seq_len", ctypes.c_int),
        ("max_chunk", ctypes.c_int), ("head_class", ctypes.c_void_p), ("num_pages", ctypes.c_int),
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
        ("free_list", ctypes.c_void_p), ("state", ctypes.c_void_p),
    ]


_lib = None


def lib():
    """Loads libsegkv.so (raises if it is not built: there is no other implementation)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with `python -m head_wise_sparse_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.segkv_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(P)]
        L.segkv_destroy.argtypes = [P]
        L.segkv_destroy.restype = None
        L.segkv_ring_pages.argtypes = [P]
        L.segkv_max_lp.argtypes = [P]
        L.segkv_seq_len.argtypes = [P, I, I]
        L.segkv_pages_used.argtypes = [P]
        L.segkv_workspace_bytes.argtypes = [P, I, I]
        L.segkv_workspace_bytes.restype = SZ
        L.segkv_reset.argtypes = [P, P]
        L.segkv_append.argtypes = [P, I, I, P, P, P, P, P, P, SZ, P]
        L.segkv_prefill_attn.argtypes = [P, I, I, P, P, P, P, F, P, P, P, P, SZ, P]
        L.segkv_plan_prefill.argtypes = [P, I, I, P, P, P, I64, ctypes.POINTER(I64), ctypes.POINTER(I),
                                         ctypes.POINTER(I)]
        L.segkv_decode_attn.argtypes = [P, I, I, P, P, P, F, I, P, P, P, P, SZ, P]
        L.segkv_decode_attn_noalloc.argtypes = [P, I, I, P, P, P, F, I, P, P, P, P]
        L.segkv_relocate_q.argtypes = [P, I, I, P, P, P, F, I, P]
        L.segkv_fork.argtypes = [P, I, I, P]
        L.segkv_prefill_attn_2src.argtypes = [P, I, I, P, P, P, P, P, P, F, P, P, P, P, SZ, P]
        L.segkv_prefill_append.argtypes = [P, I, I, P, P, P, P, P, P, F, P, P, P, P, SZ, P]
        L.segkv_router_topk.argtypes = [P, I, I, P, P, P, P, P, F, P, P, P, P, SZ, P]
        L.segkv_decode_step.argtypes = [P, I, I, P, P, P, P, F, I, P, P, P, P, SZ, P]
        L.segkv_device_status.argtypes = [P, P]
        L.segkv_last_error.argtypes = [P]
        L.segkv_last_error.restype = ctypes.c_char_p
        L.segkv_debug_set.argtypes = [P, I, ctypes.c_longlong]
        L.segkv_strerror.argtypes = [I]
        L.segkv_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc: int, what: str, h=None) -> None:
    if rc != SEGKV_OK:
        detail = ""
        if h is not None and rc == 6:
            detail = " [" + lib().segkv_last_error(h).decode(errors="replace") + "]"
        raise SegkvError(rc, what + detail)


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a: np.ndarray) -> int:
    # the address as a plain int (data_as builds a ctypes object per call, several times
    # slower); the caller keeps `a` alive for the duration of the call
    return a.ctypes.data


def _dptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---------------------------------------------------------------------------- raw handle
class Handle:
    """A segkv_t.  Pointers may be torch tensors or raw integers (device addresses)."""

    def __init__(self, *, num_layers, num_q_heads, num_kv_heads, head_dim, page_size, window, ring_pages,
                 max_seqs, max_seq_len, max_chunk, head_class, num_pages, k_pool, v_pool, page_table, free_list,
                 state):
        self._cls = np.ascontiguousarray(np.asarray(head_class, dtype=np.uint8).reshape(-1))
        self.cfg = Config(num_layers, num_q_heads, num_kv_heads, head_dim, page_size, window, ring_pages, max_seqs,
                          max_seq_len, max_chunk, _p(self._cls), num_pages, _dptr(k_pool), _dptr(v_pool),
                          _dptr(page_table), _dptr(free_list), _dptr(state))
        self.h = ctypes.c_void_p()
        _check(lib().segkv_create(ctypes.byref(self.cfg), ctypes.byref(self.h)), "segkv_create")

    def close(self):
        if getattr(self, "h", None) and self.h.value:
            lib().segkv_destroy(self.h)
            self.h = ctypes.c_void_p()

    def __del__(self):
        self.close()

    @property
    def ring_pages(self) -> int:
        return lib().segkv_ring_pages(self.h)

    @property
    def max_lp(self) -> int:
        return lib().segkv_max_lp(self.h)

    @property
    def pages_used(self) -> int:
        return lib().segkv_pages_used(self.h)

    def seq_len(self, layer: int, seq: int) -> int:
        return lib().segkv_seq_len(self.h, layer, seq)

    def workspace_bytes(self, max_batch: int, max_tokens: int) -> int:
        return lib().segkv_workspace_bytes(self.h, max_batch, max_tokens)

    def reset(self, stream=None) -> None:
        _check(lib().segkv_reset(self.h, _stream(stream)), "segkv_reset", self.h)

    def append(self, layer, seq_ids, start, count, k_new, v_new, ws, ws_bytes, stream=None) -> int:
        s, st, c = _i32(seq_ids), _i32(start), _i32(count)
        return lib().segkv_append(self.h, layer, len(s), _p(s), _p(st), _p(c), _dptr(k_new), _dptr(v_new),
                                  _dptr(ws), ws_bytes, _stream(stream))

    def prefill(self, layer, seq_ids, q_start, q_len, q, scale, out, lse, visited, ws, ws_bytes, stream=None) -> int:
        s, qs, ql = _i32(seq_ids), _i32(q_start), _i32(q_len)
        return lib().segkv_prefill_attn(self.h, layer, len(s), _p(s), _p(qs), _p(ql), _dptr(q), float(scale),
                                        _dptr(out), _dptr(lse), _dptr(visited), _dptr(ws), ws_bytes, _stream(stream))

    def prefill_2src(self, layer, seq_ids, q_start, q_len, q, k_chunk, v_chunk, scale, out, lse, visited, ws,
                     ws_bytes, stream=None) -> int:
        s, qs, ql = _i32(seq_ids), _i32(q_start), _i32(q_len)
        return lib().segkv_prefill_attn_2src(self.h, layer, len(s), _p(s), _p(qs), _p(ql), _dptr(q), _dptr(k_chunk),
                                             _dptr(v_chunk), float(scale), _dptr(out), _dptr(lse), _dptr(visited),
                                             _dptr(ws), ws_bytes, _stream(stream))

    def prefill_append(self, layer, seq_ids, q_start, q_len, q, k_new, v_new, scale, out, lse, visited, ws,
                       ws_bytes, stream=None) -> int:
        s, qs, ql = _i32(seq_ids), _i32(q_start), _i32(q_len)
        return lib().segkv_prefill_append(self.h, layer, len(s), _p(s), _p(qs), _p(ql), _dptr(q), _dptr(k_new),
                                          _dptr(v_new), float(scale), _dptr(out), _dptr(lse), _dptr(visited),
                                          _dptr(ws), ws_bytes, _stream(stream))

    def decode(self, layer, seq_ids, q_pos, q, scale, num_splits, out, lse, visited, ws, ws_bytes,
               stream=None) -> int:
        s, qp = _i32(seq_ids), _i32(q_pos)
        return lib().segkv_decode_attn(self.h, layer, len(s), _p(s), _p(qp), _dptr(q), float(scale), int(num_splits),
                                       _dptr(out), _dptr(lse), _dptr(visited), _dptr(ws), ws_bytes, _stream(stream))

    def decode_step(self, layer, seq_ids, k_new, v_new, q, scale, num_splits, out, lse, visited, ws, ws_bytes,
                    stream=None) -> int:
        s = _i32(seq_ids)
        return lib().segkv_decode_step(self.h, layer, len(s), _p(s), _dptr(k_new), _dptr(v_new), _dptr(q),
                                       float(scale), int(num_splits), _dptr(out), _dptr(lse), _dptr(visited),
                                       _dptr(ws), ws_bytes, _stream(stream))

    def router_topk(self, layer, seq_ids, q_start, q_len, q, lse, scale, k, scores, rows_out, ws, ws_bytes,
                    stream=None) -> int:
        s, qs, ql, kk = _i32(seq_ids), _i32(q_start), _i32(q_len), _i32(k)
        return lib().segkv_router_topk(self.h, layer, len(s), _p(s), _p(qs), _p(ql), _dptr(q), _dptr(lse),
                                       float(scale), _p(kk), _dptr(scores), _dptr(rows_out), _dptr(ws), ws_bytes,
                                       _stream(stream))

    def decode_noalloc(self, layer, seq_ids, q_pos, q, scale, num_splits, out, lse, visited, stream=None) -> int:
        """segkv_decode_attn_noalloc: decode without a workspace, on the library's fixed scratch."""
        s, qp = _i32(seq_ids), _i32(q_pos)
        return lib().segkv_decode_attn_noalloc(self.h, layer, len(s), _p(s), _p(qp), _dptr(q), float(scale),
                                               int(num_splits), _dptr(out), _dptr(lse), _dptr(visited),
                                               _stream(stream))

    def fork(self, src_seq, dst_seq, stream=None) -> None:
        _check(lib().segkv_fork(self.h, int(src_seq), int(dst_seq), _stream(stream)), "segkv_fork", self.h)

    def relocate_q(self, layer, n_tokens, shift, q_in, q_out, theta_base, interleaved, stream=None) -> int:
        return lib().segkv_relocate_q(self.h, layer, int(n_tokens), _dptr(shift), _dptr(q_in), _dptr(q_out),
                                      float(theta_base), int(interleaved), _stream(stream))

    def plan_prefill(self, layer, q_start, q_len):
        """Longest-processing-time-first list as int32 rows (seq index, KV head, tile, cost)."""
        qs, ql = _i32(q_start), _i32(q_len)
        n = ctypes.c_int64()
        tp, kt = ctypes.c_int(), ctypes.c_int()
        lib().segkv_plan_prefill(self.h, layer, len(qs), _p(qs), _p(ql), None, 0, ctypes.byref(n), ctypes.byref(tp),
                                 ctypes.byref(kt))
        out = np.zeros((max(n.value, 1), 4), dtype=np.int32)
        _check(lib().segkv_plan_prefill(self.h, layer, len(qs), _p(qs), _p(ql), _p(out), n.value, ctypes.byref(n),
                                        ctypes.byref(tp), ctypes.byref(kt)), "segkv_plan_prefill")
        return out[:n.value], tp.value, kt.value

    def device_status(self, stream=None) -> int:
        return lib().segkv_device_status(self.h, _stream(stream))

    def debug_set(self, key: int, value: int) -> int:
        return lib().segkv_debug_set(self.h, key, value)


# ---------------------------------------------------------------------------- torch front end
class SegKV:
    """Owns the device buffers (through torch) of one segmented paged KV cache and calls the
    library on the current CUDA stream.  bf16 tensors are torch.bfloat16, contiguous."""

    def __init__(self, *, num_layers: int, num_q_heads: int, num_kv_heads: int, head_dim: int, page_size: int,
                 window: int, head_class, num_pages: int, free_list, max_seqs: int, max_seq_len: int,
                 ring_pages: int = 0, max_chunk: int = 0, ws_batch: Optional[int] = None,
                 ws_tokens: Optional[int] = None, device="cuda"):
        import torch

        self.torch = torch
        self.device = torch.device(device)
        self.num_layers, self.hq, self.hkv, self.d = num_layers, num_q_heads, num_kv_heads, head_dim
        self.page, self.num_pages = page_size, num_pages
        self.k_pool = torch.zeros((num_pages, page_size, head_dim), dtype=torch.bfloat16, device=self.device)
        self.v_pool = torch.zeros_like(self.k_pool)
        max_lp = -(-max_seq_len // page_size)
        self.page_table = torch.full((num_layers, max_seqs, num_kv_heads, max_lp), -1, dtype=torch.int32,
                                     device=self.device)
        fl = free_list if isinstance(free_list, torch.Tensor) else torch.from_numpy(_i32(free_list))
        self.free_list = fl.to(device=self.device, dtype=torch.int32).contiguous()
        self.state = torch.zeros(4, dtype=torch.int32, device=self.device)
        self.handle = Handle(num_layers=num_layers, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                             head_dim=head_dim, page_size=page_size, window=window, ring_pages=ring_pages,
                             max_seqs=max_seqs, max_seq_len=max_seq_len, max_chunk=max_chunk, head_class=head_class,
                             num_pages=num_pages, k_pool=self.k_pool, v_pool=self.v_pool,
                             page_table=self.page_table, free_list=self.free_list, state=self.state)
        nb = ws_batch or max_seqs
        nt = ws_tokens or max_seq_len * max(1, min(max_seqs, 4))
        self.ws_bytes = self.handle.workspace_bytes(nb, nt)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=self.device)

    def ensure_workspace(self, max_batch: int, max_tokens: int) -> None:
        need = self.handle.workspace_bytes(max_batch, max_tokens)
        if need > self.ws_bytes:
            self.ws = self.torch.zeros(need, dtype=self.torch.uint8, device=self.device)
            self.ws_bytes = need

    def reset(self) -> None:
        self.handle.reset()

    def append(self, layer: int, seq_ids: Sequence[int], start: Sequence[int], count: Sequence[int], k_new, v_new):
        _check(self.handle.append(layer, seq_ids, start, count, k_new, v_new, self.ws, self.ws_bytes),
               "segkv_append", self.handle.h)

    def prefill(self, layer: int, seq_ids, q_start, q_len, q, *, out=None, lse=None, visited=None,
                scale: float = 0.0):
        t = self.torch
        T = int(np.sum(q_len))
        out = out if out is not None else t.empty((T, self.hq, self.d), dtype=t.bfloat16, device=self.device)
        lse = lse if lse is not None else t.empty((T, self.hq), dtype=t.float32, device=self.device)
        _check(self.handle.prefill(layer, seq_ids, q_start, q_len, q, scale, out, lse, visited, self.ws,
                                   self.ws_bytes), "segkv_prefill_attn", self.handle.h)
        return out, lse

    def prefill_2src(self, layer: int, seq_ids, q_start, q_len, q, k_chunk, v_chunk, *, out=None, lse=None,
                     visited=None, scale: float = 0.0):
        """segkv_prefill_attn_2src: prefill of a chunk not yet appended; its keys come from
        k_chunk / v_chunk [sum(q_len), Hkv, D] (append the chunk afterwards)."""
        t = self.torch
        T = int(np.sum(q_len))
        out = out if out is not None else t.empty((T, self.hq, self.d), dtype=t.bfloat16, device=self.device)
        lse = lse if lse is not None else t.empty((T, self.hq), dtype=t.float32, device=self.device)
        _check(self.handle.prefill_2src(layer, seq_ids, q_start, q_len, q, k_chunk, v_chunk, scale, out, lse,
                                        visited, self.ws, self.ws_bytes), "segkv_prefill_attn_2src", self.handle.h)
        return out, lse

    def prefill_append(self, layer: int, seq_ids, q_start, q_len, q, k_new, v_new, *, out=None, lse=None,
                       visited=None, scale: float = 0.0):
        """segkv_prefill_append: appends k_new / v_new [sum(q_len), Hkv, D] at q_start and attends
        the range's queries, in one kernel (the kernel stores each page it loads)."""
        t = self.torch
        T = int(np.sum(q_len))
        out = out if out is not None else t.empty((T, self.hq, self.d), dtype=t.bfloat16, device=self.device)
        lse = lse if lse is not None else t.empty((T, self.hq), dtype=t.float32, device=self.device)
        _check(self.handle.prefill_append(layer, seq_ids, q_start, q_len, q, k_new, v_new, scale, out, lse, visited,
                                          self.ws, self.ws_bytes), "segkv_prefill_append", self.handle.h)
        return out, lse

    def decode(self, layer: int, seq_ids, q_pos, q, *, out=None, lse=None, visited=None, scale: float = 0.0,
               num_splits: int = 0):
        t = self.torch
        B = len(seq_ids)
        out = out if out is not None else t.empty((B, self.hq, self.d), dtype=t.bfloat16, device=self.device)
        lse = lse if lse is not None else t.empty((B, self.hq), dtype=t.float32, device=self.device)
        _check(self.handle.decode(layer, seq_ids, q_pos, q, scale, num_splits, out, lse, visited, self.ws,
                                  self.ws_bytes), "segkv_decode_attn", self.handle.h)
        return out, lse

    def decode_step(self, layer: int, seq_ids, k_new, v_new, q, *, out=None, lse=None, visited=None,
                    scale: float = 0.0, num_splits: int = 0):
        """segkv_decode_step: appends one token per sequence (k_new, v_new [B, Hkv, D]) and
        decodes its query q [B, Hq, D] at that position, in one decode pass."""
        t = self.torch
        B = len(seq_ids)
        out = out if out is not None else t.empty((B, self.hq, self.d), dtype=t.bfloat16, device=self.device)
        lse = lse if lse is not None else t.empty((B, self.hq), dtype=t.float32, device=self.device)
        _check(self.handle.decode_step(layer, seq_ids, k_new, v_new, q, scale, num_splits, out, lse, visited, self.ws,
                                       self.ws_bytes), "segkv_decode_step", self.handle.h)
        return out, lse

    def router_topk(self, layer: int, seq_ids, q_start, q_len, q, lse, k, *, scores=None, rows=None,
                    scale: float = 0.0):
        """segkv_router_topk: each token's received attention mass (fp32 [sum(q_len)]) and the
        packed rows of the k[b] highest-scoring tokens of every sequence (int32 [sum(k)])."""
        t = self.torch
        T, K = int(sum(q_len)), int(sum(k))
        scores = scores if scores is not None else t.empty((T,), dtype=t.float32, device=self.device)
        rows = rows if rows is not None else t.empty((max(K, 1),), dtype=t.int32, device=self.device)
        _check(self.handle.router_topk(layer, seq_ids, q_start, q_len, q, lse, scale, k, scores, rows, self.ws,
                                       self.ws_bytes), "segkv_router_topk", self.handle.h)
        return scores, rows[:K]

    def fork(self, src_seq: int, dst_seq: int) -> None:
        """segkv_fork: dst_seq (empty) shares src_seq's pages; appends copy shared pages first."""
        self.handle.fork(src_seq, dst_seq)

    def relocate_q(self, layer: int, q, shift, *, out=None, theta_base: float = 10000.0, interleaved: bool = False):
        """segkv_relocate_q: local heads' queries turned by the rotary angle of position -shift
        (shift: int32 per packed token, on the device); ``out`` may be ``q`` (in place)."""
        t = self.torch
        out = out if out is not None else t.empty_like(q)
        _check(self.handle.relocate_q(layer, q.shape[0], shift, q, out, theta_base, interleaved), "segkv_relocate_q",
               self.handle.h)
        return out

    def device_status(self) -> int:
        return self.handle.device_status()

    def debug_set(self, key: int, value: int) -> None:
        """segkv_debug_set (test hooks): the wait limit, a stalled prefill, the work-list order."""
        _check(self.handle.debug_set(key, value), "segkv_debug_set", self.handle.h)
