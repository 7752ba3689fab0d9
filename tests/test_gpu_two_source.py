"""Two-source prefill on the CUDA path (needs a B200).

segkv_prefill_attn_2src attends a chunk that is not yet appended: the chunk's keys come
from its own K/V tensors, the earlier context from the pages.  Appended afterwards, it must
equal "append, then segkv_prefill_attn" bit for bit (outputs, lse, visited counts, page
tables), and it must let a local head's ring shrink to the W - 1 tokens before the chunk
(ceil((W - 1) / P) + 1 pages) while matching the fp64 oracle within |out - ref| <=
8e-3 + 1e-2 |ref|, lse 1e-3 (per-head storage holding only the tokens each head needs:
zhichai.net news item "What Happened", item 3).
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


def segkv(hq, hkv, d, page, window, cls, ring, pages, max_len, seed):
    from head_wise_sparse_b200.segkv import SegKV

    free = np.random.default_rng(seed).permutation(pages).astype(np.int32)
    return SegKV(num_layers=1, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=page, window=window,
                 head_class=np.array(cls, dtype=np.uint8), num_pages=pages, free_list=free, max_seqs=4,
                 max_seq_len=max_len, ring_pages=ring, max_chunk=256, ws_batch=4, ws_tokens=1024), free


@pytest.mark.parametrize("d,g,page", [(128, 4, 16), (64, 1, 64), (128, 8, 32)])
def test_two_source_equals_append_then_prefill(torch_cuda, d, g, page):
    torch = torch_cuda
    hkv = 2
    hq = hkv * g
    ctx, chunk = [0, 2 * page, 5 * page], [100, 37, 2 * page]
    max_len = 8 * page + 256
    ring = -(-max_len // page)
    a, _ = segkv(hq, hkv, d, page, 40, [1, 0], ring, 200, max_len, seed=50 + d)
    b, _ = segkv(hq, hkv, d, page, 40, [1, 0], ring, 200, max_len, seed=50 + d)
    rng = np.random.default_rng(51 + d + g)
    ids = [0, 1, 3]
    kc, vc = bits(rng, (sum(ctx), hkv, d)), bits(rng, (sum(ctx), hkv, d))
    live = [i for i, n in zip(ids, ctx) if n]
    for kv in (a, b):
        kv.append(0, live, [0] * len(live), [n for n in ctx if n], to_dev(kc), to_dev(vc))
    k, v, q = bits(rng, (sum(chunk), hkv, d)), bits(rng, (sum(chunk), hkv, d)), bits(rng, (sum(chunk), hq, d))
    va = torch.zeros((3, hq), dtype=torch.int64, device="cuda")
    vb = torch.zeros((3, hq), dtype=torch.int64, device="cuda")
    a.append(0, ids, ctx, chunk, to_dev(k), to_dev(v))
    out_a, lse_a = a.prefill(0, ids, ctx, chunk, to_dev(q), visited=va)
    out_b, lse_b = b.prefill_2src(0, ids, ctx, chunk, to_dev(q), to_dev(k), to_dev(v), visited=vb)
    b.append(0, ids, ctx, chunk, to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert a.device_status() == 0 and b.device_status() == 0
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b) and torch.equal(va, vb)
    assert torch.equal(a.page_table, b.page_table)


def test_two_source_runs_with_the_smallest_ring(torch_cuda):
    from head_wise_sparse_b200.segkv import SegkvError

    torch = torch_cuda
    hq, hkv, d, page, window = 8, 2, 128, 16, 40
    cls = [1, 0]
    ring = -(-(window - 1) // page) + 1  # 4 pages: the W - 1 tokens before a chunk
    total, step = 320, 64
    kv, free = segkv(hq, hkv, d, page, window, cls, ring, 120, total, seed=52)
    small, _ = segkv(hq, hkv, d, page, window, cls, ring, 120, total, seed=52)
    o = orc.Oracle(layers=1, hq=hq, hkv=hkv, d=d, page=page, window=window, ring=total // page, max_seqs=4,
                   max_seq_len=total, num_pages=120, classes=np.array(cls, dtype=np.uint8), free_list=free)
    rng = np.random.default_rng(53)
    for lo in range(0, total, step):
        k, v, q = bits(rng, (step, hkv, d)), bits(rng, (step, hkv, d)), bits(rng, (step, hq, d))
        out, lse = kv.prefill_2src(0, [0], [lo], [step], to_dev(q), to_dev(k), to_dev(v))
        kv.append(0, [0], [lo], [step], to_dev(k), to_dev(v))
        o.append(0, [0], [lo], [step], k, v)
        torch.cuda.synchronize()
        assert kv.device_status() == 0
        ro, rl, _ = o.attention(0, [0], [lo], [step], q)
        ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
        assert ok, f"chunk at {lo}: excess {worst} at {at}"
        assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-3
        # the one-source path needs the chunk's window inside the ring, which 4 pages cannot hold
        small.append(0, [0], [lo], [step], to_dev(k), to_dev(v))
        if lo > 0:
            with pytest.raises(SegkvError) as e:
                small.prefill(0, [0], [lo], [step], to_dev(q))
            assert e.value.code == 4
