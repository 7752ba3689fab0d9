"""Attention-as-router scores and top-k on the CUDA path (needs a B200) against the oracle.

segkv_router_topk scores every token of a prefill call by the attention mass it receives
from the call's queries, exp(scale q.k - lse) summed over query heads and queries, and
returns the k highest-scoring rows of each sequence (zhichai.net news item "What
Happened", item 2: dense FFN only on the top-k tokens by attention score).

Tolerance: a weight depends on lse through exp(-lse), so an lse within 1e-3 of the exact
one (the bound the prefill is held to) moves every weight, and so every score, by at most
a factor e^(+-1e-3): scores must satisfy |s - ref| <= 2e-3 |ref| + 1e-5.  The top-k rows
are a decision taken on the kernel's fp32 scores, so they are checked bit for bit against
the oracle's selection run on those same fp32 scores, and for validity (every chosen score
>= every other one) against the oracle's fp64 scores.
"""
import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from tests.harness import to_dev

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2e-3, 1e-5


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def bits(rng, shape, zero=False):
    if zero:
        return np.zeros(shape, dtype=np.uint16)
    return wl.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def build(hq, hkv, d, page, window, cls, ctx, chunk, seed, max_len=None, zero_q=False):
    """One handle and one oracle holding the same K/V; returns both plus the call's queries."""
    from head_wise_sparse_b200.segkv import SegKV

    rng = np.random.default_rng(seed)
    nseq = len(ctx)
    lens = [c + n for c, n in zip(ctx, chunk)]
    max_len = max_len or max(lens) + 8
    ring = -(-max_len // page)
    pages = nseq * hkv * (ring + 2) + 8
    free = rng.permutation(pages).astype(np.int32)
    cls = np.array(cls, dtype=np.uint8)
    kv = SegKV(num_layers=1, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, page_size=page, window=window,
               head_class=cls, num_pages=pages, free_list=free, max_seqs=nseq, max_seq_len=max_len,
               ring_pages=ring, max_chunk=max(lens), ws_batch=nseq, ws_tokens=sum(lens))
    o = orc.Oracle(layers=1, hq=hq, hkv=hkv, d=d, page=page, window=window, ring=ring, max_seqs=nseq,
                   max_seq_len=max_len, num_pages=pages, classes=cls, free_list=free)
    ids = list(range(nseq))
    k, v = bits(rng, (sum(lens), hkv, d)), bits(rng, (sum(lens), hkv, d))
    kv.append(0, ids, [0] * nseq, lens, to_dev(k), to_dev(v))
    o.append(0, ids, [0] * nseq, lens, k, v)
    q = bits(rng, (sum(chunk), hq, d), zero=zero_q)
    return kv, o, ids, list(ctx), list(chunk), q


def check(torch, kv, o, ids, qs, ql, q, k):
    qd = to_dev(q)
    _, lse = kv.prefill(0, ids, qs, ql, qd)
    scores, rows = kv.router_topk(0, ids, qs, ql, qd, lse, k)
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    s = scores.cpu().numpy().astype(np.float64)
    ref = o.router_scores(0, ids, qs, ql, q)
    err = np.abs(s - ref) - (RTOL * np.abs(ref) + ATOL)
    assert err.max() <= 0, f"score excess {err.max()} at {int(err.argmax())}"
    got = rows.cpu().numpy()
    assert np.array_equal(got, orc.topk_rows(s, ql, k))
    off, pos = 0, 0
    for n, kk in zip(ql, k):
        mine = got[pos:pos + kk]
        rest = np.setdiff1d(np.arange(off, off + n), mine)
        if kk and rest.size:  # within the score tolerance, the chosen rows are the top ones
            assert ref[mine].min() >= ref[rest].max() * (1 - 2 * RTOL) - 2 * ATOL
        off += n
        pos += kk
    return s, got


@pytest.mark.parametrize("d,g,page", [(128, 4, 16), (64, 2, 32), (128, 8, 64), (128, 1, 16)])
def test_router_scores_and_topk_match_the_oracle(torch_cuda, d, g, page):
    hkv = 2
    kv, o, ids, qs, ql, q = build(hkv * g, hkv, d, page, 40, [1, 0], ctx=[0, 37, 150], chunk=[300, 173, 64],
                                  seed=40 + d + g)
    check(torch_cuda, kv, o, ids, qs, ql, q, [75, 173, 0])


def test_router_window_one_ties_pick_the_first_positions(torch_cuda):
    # Q = 0 and every query sees only itself: each weight is exp(0 - 0) = 1 exactly, every
    # token scores exactly Hq, and position alone decides the top-k
    kv, o, ids, qs, ql, q = build(8, 2, 128, 16, 1, [0, 0], ctx=[0, 5], chunk=[200, 77], seed=41, zero_q=True)
    s, rows = check(torch_cuda, kv, o, ids, qs, ql, q, [17, 30])
    assert np.all(s == 8.0)
    assert rows.tolist() == list(range(17)) + list(range(200, 230))


def test_router_zero_queries_follow_the_harmonic_closed_form(torch_cuda):
    # with Q = 0 the weights are 1 / (keys seen); the oracle's pins fix that closed form
    kv, o, ids, qs, ql, q = build(8, 2, 128, 16, 40, [1, 0], ctx=[0], chunk=[640], seed=42, zero_q=True)
    check(torch_cuda, kv, o, ids, qs, ql, q, [160])


def test_router_mistral_shaped_chunk(torch_cuda):
    # 32 query heads over 8 KV heads (one global), D 128, pages of 64, window 1024: a 1 536-token
    # chunk after 700 tokens of context spans many key tiles and cuts long items into chunks
    cls = [0] * 8
    cls[3] = 1
    kv, o, ids, qs, ql, q = build(32, 8, 128, 64, 1024, cls, ctx=[700], chunk=[1536], seed=43)
    check(torch_cuda, kv, o, ids, qs, ql, q, [384])


def test_router_whole_sequence_mass_at_full_size(torch_cuda):
    # 8 192 tokens, Mistral-shaped: every query row's weights sum to 1 over the call's own
    # tokens, so the scores sum to Hq x L (a property at any size); top-k rows are valid
    from head_wise_sparse_b200.segkv import SegKV

    torch = torch_cuda
    w = wl.CONFIGS["mistral7b_prefill_L8192"]
    L = 8192
    kv = SegKV(num_layers=1, num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, page_size=w.page, window=w.window,
               head_class=w.class_array(), num_pages=w.num_pages, free_list=w.free_list(), max_seqs=1, max_seq_len=L,
               ring_pages=w.ring_pages, max_chunk=L, ws_batch=1, ws_tokens=L)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(44)
    k = torch.randn((L, w.hkv, w.d), generator=gen, device="cuda").to(torch.bfloat16) * (1.0 / np.sqrt(w.d))
    v = torch.randn((L, w.hkv, w.d), generator=gen, device="cuda").to(torch.bfloat16)
    q = torch.randn((L, w.hq, w.d), generator=gen, device="cuda").to(torch.bfloat16)
    kv.append(0, [0], [0], [L], k.contiguous(), v)
    _, lse = kv.prefill(0, [0], [0], [L], q)
    scores, rows = kv.router_topk(0, [0], [0], [L], q, lse, [L // 4])
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    s = scores.double().cpu().numpy()
    assert abs(s.sum() - w.hq * L) <= 1e-3 * w.hq * L
    r = rows.cpu().numpy()
    assert r.size == L // 4 and np.all(np.diff(r) > 0)
    rest = np.setdiff1d(np.arange(L), r)
    assert s[r].min() >= s[rest].max()
    assert np.array_equal(r, orc.topk_rows(scores.cpu().numpy().astype(np.float64), [L], [L // 4]))
