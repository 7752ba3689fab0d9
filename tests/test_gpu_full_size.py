"""Full-size workloads on the CUDA path (needs a B200), in the launch configuration the
benchmark times, plus edge cases.  The Mistral-shaped and 128K-chunk workloads are checked
on every (token, head) row against the oracle (seconds to about a minute of fp64 on the
host's cores); the Llama-shaped 4-layer workload (about 34 TFLOP in fp64) on sampled rows
the oracle computes one by one.

Tolerances as in test_gpu_parity: |out - ref| <= 8e-3 + 1e-2 |ref|, |lse - ref| <= 1e-3;
page tables and visited-pair counts bit-exact (counts against the closed forms in
tests/golden/visible_pairs.json).
"""
import json
import os

import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import segkv
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq
from tests.harness import (bf16_to_f64, context_calls, kv_for_call, make_kv, q_for_call, step_append, step_queries,
                           to_dev, within_tolerance)

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def dual_replay(w, layer, kv, o, ctx_chunk=4096):
    """Every append call's K/V is generated once and fed to both sides."""
    for ids, st, cnt in list(context_calls(w, ctx_chunk)) + [step_append(w)]:
        if not ids:
            continue
        k, v = kv_for_call(w, layer, ids, st, cnt)
        kv.append(layer, ids, st, cnt, to_dev(k), to_dev(v))
        o.append(layer, ids, st, cnt, k, v)


def sample_rows(w, q_len, n, seed):
    """Seeded uniform rows (packed token * hq + head) plus each sequence's first and last
    query token for every head."""
    total = int(sum(q_len))
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(total * w.hq, size=min(n, total * w.hq), replace=False).tolist())
    off = 0
    for n_b in q_len:
        for tok in (off, off + n_b - 1):
            rows.update(tok * w.hq + h for h in range(w.hq))
        off += n_b
    return np.array(sorted(rows), dtype=np.int64)


def compare_rows(w, out, lse, ro, rl, rows):
    go = bf16_to_f64(out).reshape(-1, w.d)[rows]
    gl = lse.cpu().numpy().astype(np.float64).reshape(-1)[rows]
    ok, worst, at = within_tolerance(go, ro.reshape(-1, w.d)[rows])
    assert ok, f"out mismatch: excess {worst} at row {rows[at[0]]}"
    err = np.abs(gl - rl.reshape(-1)[rows]).max()
    assert err <= 1e-3, f"lse mismatch {err}"


def closed_form_counts(w, layer, ids, qs, ql):
    want = np.zeros((len(ids), w.hq), dtype=np.uint64)
    for i, (a, n) in enumerate(zip(qs, ql)):
        p = np.arange(a, a + n, dtype=np.int64)
        for h in range(w.hq):
            want[i, h] = (p + 1).sum() if w.classes[layer][h // w.group] else np.minimum(p + 1, w.window).sum()
    return want


def prefill_full(torch, w, layer_list, n_rows, ctx_chunk=4096, golden=None):
    kv = make_kv(w)
    o = orc.Oracle.for_workload(w)  # one allocator for all layers, like the library's
    for layer in layer_list:
        dual_replay(w, layer, kv, o, ctx_chunk)
        ids, qs, ql = step_queries(w)
        q = q_for_call(w, layer, ids, qs, ql)
        vis = torch.zeros((len(ids), w.hq), dtype=torch.int64, device="cuda")
        out, lse = kv.prefill(layer, ids, qs, ql, to_dev(q), visited=vis)
        torch.cuda.synchronize()
        assert kv.device_status() == 0
        got = vis.cpu().numpy().astype(np.uint64)
        if n_rows is None:  # every row, and the oracle's own visited counts
            ro, rl, rc = o.attention(layer, ids, qs, ql, q)
            compare_rows(w, out, lse, ro, rl, np.arange(ro.reshape(-1, w.d).shape[0]))
            assert np.array_equal(got, rc)
        else:
            rows = sample_rows(w, ql, n_rows, seed=layer)
            ro, rl, _ = o.attention(layer, ids, qs, ql, q, rows=rows)
            compare_rows(w, out, lse, ro, rl, rows)
        assert np.array_equal(got, closed_form_counts(w, layer, ids, qs, ql))
        if golden:
            g = json.load(open(os.path.join(GOLDEN, "visible_pairs.json")))[golden]
            for h in range(w.hq):
                assert int(got[0, h]) == (g["global"] if w.classes[layer][h // w.group] else g["local"])
        assert np.array_equal(kv.page_table.cpu().numpy()[layer], o.page_table()[layer])
    assert int(kv.state[0].item()) == o.cursor
    return kv


def test_mistral7b_prefill_full_size_every_row(torch_cuda):
    prefill_full(torch_cuda, wl.CONFIGS["mistral7b_prefill_L8192"], [0], None, golden="mistral7b_prefill_L8192")


def test_chunked_128k_prefill_full_size_every_row(torch_cuda):
    prefill_full(torch_cuda, wl.CONFIGS["mha_chunked_prefill_128k"], [0], None, golden="mha_chunked_prefill_128k")


def test_llama70b_varlen_four_layers_full_size(torch_cuda):
    prefill_full(torch_cuda, wl.CONFIGS["llama70b_varlen_prefill_4x4layers"], [0, 1, 2, 3], 600)


def test_decode_64x32k_full_size_every_row(torch_cuda):
    torch = torch_cuda
    w = wl.CONFIGS["decode_64x32k"]
    kv = make_kv(w)
    o = orc.Oracle.for_workload(w)
    dual_replay(w, 0, kv, o, ctx_chunk=4096)
    ids = list(range(len(w.seqs)))
    qp = [s.q_lo for s in w.seqs]
    q = np.concatenate([w.q(0, b, p, p + 1) for b, p in zip(ids, qp)], axis=0)
    vis = torch.zeros((len(ids), w.hq), dtype=torch.int64, device="cuda")
    out, lse = kv.decode(0, ids, qp, to_dev(q), visited=vis)
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    ro, rl, rc = o.attention(0, ids, qp, [1] * len(ids), q)
    rows = np.arange(len(ids) * w.hq)
    compare_rows(w, out, lse, ro, rl, rows)
    assert np.array_equal(vis.cpu().numpy().astype(np.uint64), rc)
    g = json.load(open(os.path.join(GOLDEN, "visible_pairs.json")))["decode_64x32k"]
    for h in range(w.hq):
        assert int(rc[0, h]) == (g["global"] if w.classes[0][h // w.group] else g["local"])
    assert np.array_equal(kv.page_table.cpu().numpy(), o.page_table())
    assert int(kv.state[0].item()) == o.cursor
    # the same step with other split counts: each stays within tolerance of the oracle
    for splits in (1, 5):
        o2, l2 = kv.decode(0, ids, qp, to_dev(q), num_splits=splits)
        torch.cuda.synchronize()
        compare_rows(w, o2, l2, ro, rl, rows)


# -- edge cases ----------------------------------------------------------------------------
def test_decode_row_equals_prefill_row(torch_cuda):
    torch = torch_cuda
    w = wl.CONFIGS["decode_64x32k"].scaled(seqs=(Seq(0, 3000, 2999, 3000), Seq(0, 1234, 1233, 1234)), window=700,
                                           ring_pages=-(-3000 // 64))
    kv = make_kv(w)
    for ids, st, cnt in [step_append(w)]:
        k, v = kv_for_call(w, 0, ids, st, cnt)
        kv.append(0, ids, st, cnt, to_dev(k), to_dev(v))
    ids = [0, 1]
    qp = [2999, 1233]
    q = np.concatenate([w.q(0, b, p, p + 1) for b, p in zip(ids, qp)], axis=0)
    od, ld = kv.decode(0, ids, qp, to_dev(q))
    op, lp = kv.prefill(0, ids, qp, [1, 1], to_dev(q))
    torch.cuda.synchronize()
    a, b = bf16_to_f64(od), bf16_to_f64(op)
    ok, worst, _ = within_tolerance(a, b)
    assert ok, worst
    assert np.abs(ld.cpu().numpy() - lp.cpu().numpy()).max() < 1e-3


def test_ring_too_small_is_rejected_on_the_host(torch_cuda):
    w = wl.CONFIGS["tiny_prefill_L1024_D64"].scaled(seqs=(Seq(0, 1024, 0, 1024),), ring_pages=9)
    kv = make_kv(w)
    k, v = kv_for_call(w, 0, [0], [0], [1024])
    kv.append(0, [0], [0], [1024], to_dev(k), to_dev(v))
    q = w.q(0, 0, 0, 1024)
    with pytest.raises(segkv.SegkvError) as e:
        kv.prefill(0, [0], [0], [1024], to_dev(q))
    assert e.value.code == 4
    # the last 9 pages (144 tokens) still hold every key the last 16 queries need (W = 128)
    kv.prefill(0, [0], [1008], [16], to_dev(q[1008:]))
    assert kv.device_status() == 0


def test_corrupt_page_id_sets_the_error_word_without_faulting(torch_cuda):
    torch = torch_cuda
    w = wl.CONFIGS["tiny_prefill_L1024_D64"].scaled(seqs=(Seq(0, 512, 0, 512),), ring_pages=32)
    kv = make_kv(w)
    k, v = kv_for_call(w, 0, [0], [0], [512])
    kv.append(0, [0], [0], [512], to_dev(k), to_dev(v))
    q = to_dev(w.q(0, 0, 0, 512))
    good = kv.page_table[0, 0, 0, 3].item()
    kv.page_table[0, 0, 0, 3] = w.num_pages + 7  # global head, a page every late query reads
    kv.prefill(0, [0], [0], [512], q)
    assert kv.device_status() == 7
    kv.decode(0, [0], [511], q[511:512])
    assert kv.device_status() == 7
    kv.page_table[0, 0, 0, 3] = good
    kv.prefill(0, [0], [0], [512], q)
    assert kv.device_status() == 0


def test_empty_ranges_single_tokens_and_reset(torch_cuda):
    torch = torch_cuda
    w = wl.Workload(700, "edge", 1, 8, 2, 128, 16, 40, 64,
                    (Seq(0, 1, 0, 1), Seq(0, 300, 300, 300), Seq(0, 77, 0, 77)), ((1, 0),))
    kv = make_kv(w, ws_tokens=400)
    ids, st, cnt = step_append(w)
    k, v = kv_for_call(w, 0, ids, st, cnt)
    kv.append(0, ids, st, cnt, to_dev(k), to_dev(v))
    ids, qs, ql = [0, 1, 2], [0, 300, 0], [1, 0, 77]
    q = np.concatenate([w.q(0, 0, 0, 1), w.q(0, 2, 0, 77)], axis=0)
    out1, lse1 = kv.prefill(0, ids, qs, ql, to_dev(q))
    torch.cuda.synchronize()
    o = orc.Oracle.for_workload(w)
    o.append(0, *step_append(w), k, v)
    ro, rl, _ = o.attention(0, ids, qs, ql, q)
    compare_rows(w, out1, lse1, ro, rl, np.arange(78 * w.hq))
    # empty the cache and rebuild it: identical bits
    kv.reset()
    assert kv.handle.seq_len(0, 1) == 0 and kv.handle.pages_used == 0
    kv.append(0, *step_append(w), to_dev(k), to_dev(v))
    out2, lse2 = kv.prefill(0, ids, qs, ql, to_dev(q))
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    assert kv.device_status() == 0


def test_chunked_128k_two_source_full_size(torch_cuda):
    # The 4096-token chunk at 126 976 attended before it is appended (segkv_prefill_attn_2src),
    # with every local ring at ceil((W - 1) / P) + 1 = 65 pages instead of the 129 that the
    # one-source call needs; sampled rows against the oracle, counts against the closed form.
    torch = torch_cuda
    w = wl.CONFIGS["mha_chunked_prefill_128k"]
    small = w.scaled(ring_pages=-(-(w.window - 1) // w.page) + 1)
    kv = make_kv(small)
    o = orc.Oracle.for_workload(w)
    for ids, st, cnt in context_calls(w, 4096):
        k, v = kv_for_call(w, 0, ids, st, cnt)
        kv.append(0, ids, st, cnt, to_dev(k), to_dev(v))
        o.append(0, ids, st, cnt, k, v)
    ids, st, cnt = step_append(w)
    k, v = kv_for_call(w, 0, ids, st, cnt)
    o.append(0, ids, st, cnt, k, v)
    qids, qs, ql = step_queries(w)
    assert (qids, qs, ql) == (ids, st, cnt)  # the chunk is the query range
    q = q_for_call(w, 0, qids, qs, ql)
    vis = torch.zeros((len(qids), w.hq), dtype=torch.int64, device="cuda")
    out, lse = kv.prefill_2src(0, qids, qs, ql, to_dev(q), to_dev(k), to_dev(v), visited=vis)
    kv.append(0, ids, st, cnt, to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    rows = sample_rows(w, ql, 2000, seed=7)
    ro, rl, _ = o.attention(0, qids, qs, ql, q, rows=rows)
    compare_rows(w, out, lse, ro, rl, rows)
    assert np.array_equal(vis.cpu().numpy().astype(np.uint64), closed_form_counts(w, 0, qids, qs, ql))
