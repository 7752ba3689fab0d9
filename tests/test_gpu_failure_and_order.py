"""Failure detection and schedule independence of the prefill kernel (needs a B200).

- A prefill launch whose MMA thread waits on a barrier that nothing arrives on (a test hook,
  with a shortened wait limit) must end by itself: the wait runs out, every role leaves its
  loop, copies in flight drain, and the error word reads SEGKV_ERR_DEVICE_TIMEOUT.  The
  handle stays usable: the next call gives the same bits as before the stall.
- The longest-first work list is only a schedule: each item (or key-range chunk) is computed
  by one CTA in a fixed key order and chunks merge in a fixed order, so running the list
  reversed or shuffled gives identical output bits, lse bits and visited counts.
"""
import numpy as np
import pytest

from head_wise_sparse_b200 import segkv
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq, Workload
from tests.harness import gpu_replay, make_kv, q_for_call, step_queries, to_dev

pytestmark = pytest.mark.gpu

TIMEOUT = 8  # SEGKV_ERR_DEVICE_TIMEOUT


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def prefill(torch, kv, w, q):
    ids, qs, ql = step_queries(w)
    vis = torch.zeros((len(ids), w.hq), dtype=torch.int64, device="cuda")
    out, lse = kv.prefill(0, ids, qs, ql, q, visited=vis)
    torch.cuda.synchronize()
    return out, lse, vis


def test_stalled_prefill_times_out_and_the_handle_recovers(torch_cuda):
    torch = torch_cuda
    w = wl.CONFIGS["tiny_prefill_L1024_D64"]
    kv = make_kv(w)
    gpu_replay(w, 0, kv)
    ids, qs, ql = step_queries(w)
    q = to_dev(q_for_call(w, 0, ids, qs, ql))
    out_ref, lse_ref, vis_ref = prefill(torch, kv, w, q)
    assert kv.device_status() == 0
    table = kv.page_table.clone()

    kv.debug_set(segkv.DEBUG_WAIT_LIMIT, 2_000_000)  # about a millisecond
    kv.debug_set(segkv.DEBUG_STALL_NEXT_PREFILL, 1)
    prefill(torch, kv, w, q)
    assert kv.device_status() == TIMEOUT
    assert kv.device_status() == 0  # read and cleared

    kv.debug_set(segkv.DEBUG_WAIT_LIMIT, 0)
    out, lse, vis = prefill(torch, kv, w, q)
    assert kv.device_status() == 0
    assert torch.equal(out, out_ref) and torch.equal(lse, lse_ref) and torch.equal(vis, vis_ref)
    assert torch.equal(kv.page_table, table)


def test_debug_keys_are_checked(torch_cuda):
    w = wl.CONFIGS["tiny_prefill_L1024_D64"]
    kv = make_kv(w)
    for key, value in ((0, 1), (99, 1), (segkv.DEBUG_WAIT_LIMIT, -1), (segkv.DEBUG_STALL_NEXT_PREFILL, 2),
                       (segkv.DEBUG_PREFILL_ORDER, -5)):
        assert kv.handle.debug_set(key, value) == 1  # SEGKV_ERR_INVALID_ARG


CASES = {
    # one global head under 8 query heads: long items run as key-range chunks merged by the
    # combine kernel, beside whole items of a local head
    "key_chunks": Workload(320, "chunks", 1, 16, 2, 128, 64, 700, 64, (Seq(0, 4096, 0, 4096),), ((1, 0),)),
    # GQA 4, three ragged sequences, page 16, one global and one local head
    "ragged": Workload(304, "gqa", 1, 8, 2, 128, 64, 200, 16,
                       (Seq(0, 777, 0, 777), Seq(0, 300, 0, 300), Seq(0, 1000, 0, 1000)), ((1, 0),)),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_work_list_order_gives_identical_bits(torch_cuda, case):
    torch = torch_cuda
    w = CASES[case]
    ids, qs, ql = step_queries(w)
    q = to_dev(q_for_call(w, 0, ids, qs, ql))
    runs = []
    for order in (0, 1, 987654321):  # longest first, reversed, shuffled
        kv = make_kv(w)
        gpu_replay(w, 0, kv)
        kv.debug_set(segkv.DEBUG_PREFILL_ORDER, order)
        runs.append(prefill(torch, kv, w, q))
        assert kv.device_status() == 0
    for out, lse, vis in runs[1:]:
        assert torch.equal(out, runs[0][0]) and torch.equal(lse, runs[0][1]) and torch.equal(vis, runs[0][2])
