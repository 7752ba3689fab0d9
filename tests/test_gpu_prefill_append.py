"""Fused append + prefill on the CUDA path (needs a B200).

segkv_prefill_append stores each page of the appended range from shared memory into its pool
page while attending it.  It must equal segkv_append followed by segkv_prefill_attn bit for
bit -- outputs, lse, visited counts, page tables, cursor, lengths -- and the pages it stored
must serve later attention exactly like appended ones; against the fp64 oracle within
|out - ref| <= 8e-3 + 1e-2 |ref|, lse 1e-3, page tables bit-exact (per-head storage grown as
it is attended: zhichai.net news item "What Happened", item 3).
"""
import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from tests.harness import bf16_to_f64, to_dev, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def bits(rng, shape):
    return wl.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def make(hq, hkv, d, page, window, cls, ring, pages, max_len, seed):
    from head_wise_sparse_b200.segkv import SegKV

    free = np.random.default_rng(seed).permutation(pages).astype(np.int32)
    kw = dict(num_layers=1, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=page, window=window,
              head_class=np.array(cls, dtype=np.uint8), num_pages=pages, free_list=free, max_seqs=4,
              max_seq_len=max_len, ring_pages=ring, max_chunk=512, ws_batch=4, ws_tokens=1024)
    o = orc.Oracle(layers=1, hq=hq, hkv=hkv, d=d, page=page, window=window, ring=ring, max_seqs=4,
                   max_seq_len=max_len, num_pages=pages, classes=np.array(cls, dtype=np.uint8), free_list=free)
    return SegKV(**kw), SegKV(**kw), o


def check_same(torch, a, b):
    torch.cuda.synchronize()
    assert a.device_status() == 0 and b.device_status() == 0
    assert torch.equal(a.page_table, b.page_table)
    assert int(a.state[0].item()) == int(b.state[0].item())


@pytest.mark.parametrize("d,g,page,ring", [(128, 4, 16, 0), (64, 1, 64, 0), (128, 8, 32, 0), (128, 4, 16, 8)])
def test_fused_equals_append_then_prefill(torch_cuda, d, g, page, ring):
    # ring 8 with W 40 and 200 tokens of context: the local rings have wrapped, so the chunk
    # writes some of its pages in place; ring 0 keeps every page
    torch = torch_cuda
    hkv = 2
    hq = hkv * g
    window = 40
    ctx = [0, 2 * page, 200 // page * page if ring else 5 * page]
    chunk = [100, 37, 64]
    max_len = 1024
    ring = ring or max_len // page
    two, fused, o = make(hq, hkv, d, page, window, [1, 0], ring, 400, max_len, seed=60 + d + g)
    rng = np.random.default_rng(61 + d + g + ring)
    ids = [0, 1, 3]
    live = [(i, n) for i, n in zip(ids, ctx) if n]
    kc, vc = bits(rng, (sum(ctx), hkv, d)), bits(rng, (sum(ctx), hkv, d))
    for kv in (two, fused):
        kv.append(0, [i for i, _ in live], [0] * len(live), [n for _, n in live], to_dev(kc), to_dev(vc))
    o.append(0, [i for i, _ in live], [0] * len(live), [n for _, n in live], kc, vc)
    k, v, q = bits(rng, (sum(chunk), hkv, d)), bits(rng, (sum(chunk), hkv, d)), bits(rng, (sum(chunk), hq, d))
    vt = torch.zeros((3, hq), dtype=torch.int64, device="cuda")
    vf = torch.zeros((3, hq), dtype=torch.int64, device="cuda")
    two.append(0, ids, ctx, chunk, to_dev(k), to_dev(v))
    out_t, lse_t = two.prefill(0, ids, ctx, chunk, to_dev(q), visited=vt)
    out_f, lse_f = fused.prefill_append(0, ids, ctx, chunk, to_dev(q), to_dev(k), to_dev(v), visited=vf)
    o.append(0, ids, ctx, chunk, k, v)
    check_same(torch, two, fused)
    assert torch.equal(out_t, out_f) and torch.equal(lse_t, lse_f) and torch.equal(vt, vf)
    assert np.array_equal(fused.page_table.cpu().numpy(), o.page_table())
    assert int(fused.state[0].item()) == o.cursor
    for b, n in zip(ids, [c + m for c, m in zip(ctx, chunk)]):
        assert fused.handle.seq_len(0, b) == n
    ro, rl, _ = o.attention(0, ids, ctx, chunk, q)
    ok, worst, at = within_tolerance(bf16_to_f64(out_f), ro)
    assert ok, f"excess {worst} at {at}"
    assert np.abs(lse_f.cpu().numpy() - rl).max() <= 1e-3
    # the stored pages serve later attention exactly like appended ones: a one-source
    # prefill over the last 24 positions of every sequence, and one decode step
    ends = [c + m for c, m in zip(ctx, chunk)]
    q2 = bits(rng, (72, hq, d))
    r_t = two.prefill(0, ids, [e - 24 for e in ends], [24] * 3, to_dev(q2))
    r_f = fused.prefill(0, ids, [e - 24 for e in ends], [24] * 3, to_dev(q2))
    kd, vd, qd = bits(rng, (3, hkv, d)), bits(rng, (3, hkv, d)), bits(rng, (3, hq, d))
    d_t = two.decode_step(0, ids, to_dev(kd), to_dev(vd), to_dev(qd))
    d_f = fused.decode_step(0, ids, to_dev(kd), to_dev(vd), to_dev(qd))
    check_same(torch, two, fused)
    for x, y in zip(r_t + d_t, r_f + d_f):
        assert torch.equal(x, y)


def test_fused_after_a_fork_matches_the_oracle(torch_cuda):
    # while pages are shared the call runs as append (copy on write) then prefill
    torch = torch_cuda
    _, fused, o = make(8, 2, 128, 16, 40, [1, 0], 64, 200, 1024, seed=62)
    rng = np.random.default_rng(63)
    k, v = bits(rng, (64, 2, 128)), bits(rng, (64, 2, 128))
    fused.append(0, [0], [0], [64], to_dev(k), to_dev(v))
    o.append(0, [0], [0], [64], k, v)
    fused.fork(0, 1)
    o.fork(0, 1)
    k, v, q = bits(rng, (48, 2, 128)), bits(rng, (48, 2, 128)), bits(rng, (48, 8, 128))
    out, lse = fused.prefill_append(0, [1], [64], [48], to_dev(q), to_dev(k), to_dev(v))
    o.append(0, [1], [64], [48], k, v)
    torch.cuda.synchronize()
    assert fused.device_status() == 0
    assert np.array_equal(fused.page_table.cpu().numpy(), o.page_table())
    ro, rl, _ = o.attention(0, [1], [64], [48], q)
    ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
    assert ok, f"excess {worst} at {at}"
    assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-3


def test_fused_out_of_pages_changes_nothing(torch_cuda):
    from head_wise_sparse_b200.segkv import SegkvError

    torch = torch_cuda
    _, fused, _ = make(8, 2, 128, 16, 40, [1, 0], 64, 6, 1024, seed=64)
    rng = np.random.default_rng(65)
    k, v, q = bits(rng, (64, 2, 128)), bits(rng, (64, 2, 128)), bits(rng, (64, 8, 128))
    with pytest.raises(SegkvError) as e:  # 4 global + 4 local pages > 6
        fused.prefill_append(0, [0], [0], [64], to_dev(q), to_dev(k), to_dev(v))
    assert e.value.code == 3
    torch.cuda.synchronize()
    assert fused.handle.seq_len(0, 0) == 0 and fused.handle.pages_used == 0
    assert (fused.page_table.cpu().numpy() == -1).all()


def test_fused_full_size_mistral_shaped_equals_two_calls(torch_cuda):
    # the Mistral-shaped step at full size (8 192 tokens, Hq 32, Hkv 8, D 128, 1 global + 7
    # local W 1024): every CTA stores pages while it attends them
    torch = torch_cuda
    from head_wise_sparse_b200.segkv import SegKV

    w = wl.CONFIGS["mistral7b_prefill_L8192"]
    L = w.seqs[0].length
    kw = dict(num_layers=1, num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, page_size=w.page, window=w.window,
              head_class=w.class_array(), num_pages=w.num_pages, free_list=w.free_list(), max_seqs=1,
              max_seq_len=w.max_seq_len, ring_pages=w.ring_pages, max_chunk=L, ws_batch=1, ws_tokens=L)
    two, fused = SegKV(**kw), SegKV(**kw)
    g = torch.Generator(device="cuda")
    g.manual_seed(66)
    q = torch.randn((L, w.hq, w.d), generator=g, device="cuda").to(torch.bfloat16)
    k = (torch.randn((L, w.hkv, w.d), generator=g, device="cuda") / np.sqrt(w.d)).to(torch.bfloat16)
    v = torch.randn((L, w.hkv, w.d), generator=g, device="cuda").to(torch.bfloat16)
    vt = torch.zeros((1, w.hq), dtype=torch.int64, device="cuda")
    vf = torch.zeros((1, w.hq), dtype=torch.int64, device="cuda")
    two.append(0, [0], [0], [L], k, v)
    out_t, lse_t = two.prefill(0, [0], [0], [L], q, visited=vt)
    out_f, lse_f = fused.prefill_append(0, [0], [0], [L], q, k, v, visited=vf)
    check_same(torch, two, fused)
    assert torch.equal(out_t, out_f) and torch.equal(lse_t, lse_f) and torch.equal(vt, vf)
