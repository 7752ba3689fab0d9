"""The fused decode step on the CUDA path (needs a B200).

segkv_decode_step appends one token per sequence inside the decode kernel and decodes its
query.  It must give, bit for bit, what segkv_append (one token) followed by
segkv_decode_attn gives -- outputs, lse, visited counts, page tables and the allocation
cursor -- across page starts, ring wraps of local heads and both head sizes, and match
the fp64 oracle within |out - ref| <= 8e-3 + 1e-2 |ref|, lse 1e-3 (per-head paged storage:
zhichai.net news item "What Happened", item 3).
"""
import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from tests.harness import bf16_to_f64, to_dev, within_tolerance

pytestmark = pytest.mark.gpu

HQ, HKV, P, W, R, SEQS, MAXLEN = 8, 2, 16, 40, 4, 4, 256


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def bits(rng, shape):
    return wl.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def make(d, pages, seed=31):
    from head_wise_sparse_b200.segkv import SegKV

    free = np.random.default_rng(seed).permutation(pages).astype(np.int32)
    cls = np.array([1, 0], dtype=np.uint8)
    kw = dict(num_layers=1, num_q_heads=HQ, num_kv_heads=HKV, head_dim=d, page_size=P, window=W, head_class=cls,
              num_pages=pages, free_list=free, max_seqs=SEQS, max_seq_len=MAXLEN, ring_pages=R, max_chunk=64,
              ws_batch=SEQS, ws_tokens=256)
    o = orc.Oracle(layers=1, hq=HQ, hkv=HKV, d=d, page=P, window=W, ring=R, max_seqs=SEQS, max_seq_len=MAXLEN,
                   num_pages=pages, classes=cls, free_list=free)
    return SegKV(**kw), SegKV(**kw), o


@pytest.mark.parametrize("d,splits", [(128, 0), (64, 3), (128, 2)])
def test_decode_step_equals_append_then_decode(torch_cuda, d, splits):
    torch = torch_cuda
    fused, pair, o = make(d, 200)
    rng = np.random.default_rng(32 + d + splits)
    ids = [0, 2, 3]
    ctx = [30, 47, 64]  # the next token ends a page, sits on its last row, starts a page
    k, v = bits(rng, (sum(ctx), HKV, d)), bits(rng, (sum(ctx), HKV, d))
    for kv in (fused, pair):
        kv.append(0, ids, [0, 0, 0], ctx, to_dev(k), to_dev(v))
    o.append(0, ids, [0, 0, 0], ctx, k, v)
    pos = list(ctx)
    for step in range(40):  # local heads wrap their 4-page ring several times
        kn, vn, q = bits(rng, (3, HKV, d)), bits(rng, (3, HKV, d)), bits(rng, (3, HQ, d))
        vis_f = torch.zeros((3, HQ), dtype=torch.int64, device="cuda")
        vis_p = torch.zeros((3, HQ), dtype=torch.int64, device="cuda")
        out_f, lse_f = fused.decode_step(0, ids, to_dev(kn), to_dev(vn), to_dev(q), visited=vis_f, num_splits=splits)
        pair.append(0, ids, pos, [1, 1, 1], to_dev(kn), to_dev(vn))
        out_p, lse_p = pair.decode(0, ids, pos, to_dev(q), visited=vis_p, num_splits=splits)
        o.append(0, ids, pos, [1, 1, 1], kn, vn)
        torch.cuda.synchronize()
        assert fused.device_status() == 0 and pair.device_status() == 0
        assert torch.equal(out_f, out_p) and torch.equal(lse_f, lse_p) and torch.equal(vis_f, vis_p), f"step {step}"
        assert torch.equal(fused.page_table, pair.page_table), f"step {step}"
        assert int(fused.state[0].item()) == int(pair.state[0].item()) == o.cursor
        assert fused.handle.pages_used == pair.handle.pages_used
        if step % 8 == 0 or step == 39:
            assert np.array_equal(fused.page_table.cpu().numpy(), o.page_table())
            ro, rl, rc = o.attention(0, ids, pos, [1, 1, 1], q)
            ok, worst, at = within_tolerance(bf16_to_f64(out_f), ro)
            assert ok, f"step {step}: excess {worst} at {at}"
            assert np.abs(lse_f.cpu().numpy() - rl).max() <= 1e-3
            assert np.array_equal(vis_f.cpu().numpy().astype(np.uint64), rc)
        pos = [p + 1 for p in pos]
    for b, n in zip(ids, pos):
        assert fused.handle.seq_len(0, b) == n


def test_decode_step_after_a_fork(torch_cuda):
    # while pages are shared the step takes the append's copy on write first
    torch = torch_cuda
    fused, _, o = make(128, 200, seed=33)
    rng = np.random.default_rng(34)
    k, v = bits(rng, (50, HKV, 128)), bits(rng, (50, HKV, 128))
    fused.append(0, [0], [0], [50], to_dev(k), to_dev(v))
    o.append(0, [0], [0], [50], k, v)
    fused.fork(0, 1)
    o.fork(0, 1)
    pos = [50, 50]
    for step in range(20):
        kn, vn, q = bits(rng, (2, HKV, 128)), bits(rng, (2, HKV, 128)), bits(rng, (2, HQ, 128))
        out, lse = fused.decode_step(0, [1, 0], to_dev(kn), to_dev(vn), to_dev(q))
        o.append(0, [1, 0], pos, [1, 1], kn, vn)
        torch.cuda.synchronize()
        assert fused.device_status() == 0
        assert np.array_equal(fused.page_table.cpu().numpy(), o.page_table()), f"step {step}"
        assert int(fused.state[0].item()) == o.cursor
        ro, rl, _ = o.attention(0, [1, 0], pos, [1, 1], q)
        ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
        assert ok, f"step {step}: excess {worst} at {at}"
        assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-3
        pos = [p + 1 for p in pos]


def test_decode_step_out_of_pages_changes_nothing(torch_cuda):
    from head_wise_sparse_b200.segkv import SegkvError

    torch = torch_cuda
    fused, _, _ = make(128, 8, seed=35)
    rng = np.random.default_rng(36)
    k, v = bits(rng, (64, HKV, 128)), bits(rng, (64, HKV, 128))
    fused.append(0, [0], [0], [64], to_dev(k), to_dev(v))  # 4 global + 4 local pages: the pool is full
    torch.cuda.synchronize()
    before = fused.page_table.clone()
    kn, vn, q = bits(rng, (1, HKV, 128)), bits(rng, (1, HKV, 128)), bits(rng, (1, HQ, 128))
    with pytest.raises(SegkvError) as e:
        fused.decode_step(0, [0], to_dev(kn), to_dev(vn), to_dev(q))
    assert e.value.code == 3
    torch.cuda.synchronize()
    assert fused.handle.seq_len(0, 0) == 64 and fused.handle.pages_used == 8
    assert torch.equal(before, fused.page_table)
