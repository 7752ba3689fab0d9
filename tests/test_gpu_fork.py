"""Fork and copy-on-write append on the CUDA path (needs a B200) against the oracle.

segkv_fork shares a sequence's pages with an empty one; an append that touches a shared
page first takes a private copy (hysenlabs.com write-up, "Experimental Features and Current
Limitations": a shared KV manager with forks and copy-on-write append).  After every call
the page table and allocation cursor must equal the oracle's bit for bit; attention over
every sequence must match the oracle within |out - ref| <= 8e-3 + 1e-2 |ref|, lse 1e-3.
"""
import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from tests.harness import bf16_to_f64, to_dev, within_tolerance

pytestmark = pytest.mark.gpu

HQ, HKV, D, P, W, R, SEQS, MAXLEN, PAGES = 8, 2, 128, 16, 40, 6, 4, 512, 160


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def bits(rng, shape):
    return wl.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def make_pair(torch):
    from head_wise_sparse_b200.segkv import SegKV

    free = np.random.default_rng(21).permutation(PAGES).astype(np.int32)
    cls = np.array([1, 0], dtype=np.uint8)
    kv = SegKV(num_layers=1, num_q_heads=HQ, num_kv_heads=HKV, head_dim=D, page_size=P, window=W, head_class=cls,
               num_pages=PAGES, free_list=free, max_seqs=SEQS, max_seq_len=MAXLEN, ring_pages=R, max_chunk=160,
               ws_batch=SEQS, ws_tokens=512)
    o = orc.Oracle(layers=1, hq=HQ, hkv=HKV, d=D, page=P, window=W, ring=R, max_seqs=SEQS, max_seq_len=MAXLEN,
                   num_pages=PAGES, classes=cls, free_list=free)
    return kv, o


def same_storage(torch, kv, o):
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    assert np.array_equal(kv.page_table.cpu().numpy(), o.page_table())
    assert int(kv.state[0].item()) == o.cursor


def test_fork_and_copy_on_write_match_the_oracle(torch_cuda):
    torch = torch_cuda
    kv, o = make_pair(torch)
    rng = np.random.default_rng(22)

    def append(seq_ids, starts, counts):
        n = int(sum(counts))
        k, v = bits(rng, (n, HKV, D)), bits(rng, (n, HKV, D))
        kv.append(0, seq_ids, starts, counts, to_dev(k), to_dev(v))
        o.append(0, seq_ids, starts, counts, k, v)
        same_storage(torch, kv, o)

    append([0], [0], [50])                # the fork point sits inside page 3
    kv.fork(0, 1)
    o.fork(0, 1)
    kv.fork(0, 2)
    o.fork(0, 2)
    same_storage(torch, kv, o)
    append([1], [50], [40])               # copies the shared page 3
    append([0, 2], [50, 50], [11, 1])     # seq 0 copies page 3; seq 2 then holds it alone
    append([2, 1], [51, 90], [149, 30])   # the local ring wraps over shared slots
    append([0], [61], [100])
    lens = {0: 161, 1: 120, 2: 200}
    for s, n in lens.items():
        # prefill over the last 24 positions (their windows lie in the ring's 96 tokens)
        q = bits(rng, (24, HQ, D))
        out, lse = kv.prefill(0, [s], [n - 24], [24], to_dev(q))
        torch.cuda.synchronize()
        ro, rl, _ = o.attention(0, [s], [n - 24], [24], q)
        ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
        assert ok, f"seq {s}: excess {worst} at {at}"
        assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-3
    qd = bits(rng, (3, HQ, D))
    out, lse = kv.decode(0, [0, 1, 2], [lens[0] - 1, lens[1] - 1, lens[2] - 1], to_dev(qd))
    torch.cuda.synchronize()
    ro, rl, _ = o.attention(0, [0, 1, 2], [lens[0] - 1, lens[1] - 1, lens[2] - 1], [1, 1, 1], qd)
    ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
    assert ok, f"decode: excess {worst} at {at}"
    assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-3
    assert kv.device_status() == 0


def test_fork_of_a_page_aligned_prefix_and_reset(torch_cuda):
    torch = torch_cuda
    kv, o = make_pair(torch)
    rng = np.random.default_rng(23)
    k, v = bits(rng, (64, HKV, D)), bits(rng, (64, HKV, D))
    kv.append(0, [0], [0], [64], to_dev(k), to_dev(v))
    o.append(0, [0], [0], [64], k, v)
    kv.fork(0, 3)
    o.fork(0, 3)
    k2, v2 = bits(rng, (5, HKV, D)), bits(rng, (5, HKV, D))
    kv.append(0, [3], [64], [5], to_dev(k2), to_dev(v2))
    o.append(0, [3], [64], [5], k2, v2)
    same_storage(torch, kv, o)
    q = bits(rng, (20, HQ, D))
    for s, n in ((0, 64), (3, 69)):
        out, lse = kv.prefill(0, [s], [n - 20], [20], to_dev(q))
        torch.cuda.synchronize()
        ro, rl, _ = o.attention(0, [s], [n - 20], [20], q)
        ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
        assert ok, f"seq {s}: excess {worst} at {at}"
    kv.reset()
    torch.cuda.synchronize()
    assert (kv.page_table.cpu().numpy() == -1).all() and kv.handle.pages_used == 0


def test_appends_after_every_shared_page_was_copied(torch_cuda):
    # Once the last shared page has been copied, appends no longer need a copy plan; the
    # page ids they take must still follow the oracle's allocation order exactly.
    torch = torch_cuda
    kv, o = make_pair(torch)
    rng = np.random.default_rng(24)

    def append(seq_ids, starts, counts):
        n = int(sum(counts))
        k, v = bits(rng, (n, HKV, D)), bits(rng, (n, HKV, D))
        kv.append(0, seq_ids, starts, counts, to_dev(k), to_dev(v))
        o.append(0, seq_ids, starts, counts, k, v)
        same_storage(torch, kv, o)

    append([0], [0], [10])
    kv.fork(0, 1)
    o.fork(0, 1)
    append([0, 1], [10, 10], [5, 3])        # seq 0 copies page 0, seq 1 then holds it alone
    append([1, 0, 2], [13, 15, 0], [120, 7, 33])
    append([0, 2, 1], [22, 33, 133], [1, 95, 1])
    for s, n in ((0, 23), (1, 134), (2, 128)):
        q = bits(rng, (8, HQ, D))
        out, lse = kv.prefill(0, [s], [n - 8], [8], to_dev(q))
        torch.cuda.synchronize()
        ro, rl, _ = o.attention(0, [s], [n - 8], [8], q)
        ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
        assert ok, f"seq {s}: excess {worst} at {at}"
        assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-3
