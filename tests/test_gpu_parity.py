"""CUDA path against the fp64 oracle, through the C ABI (needs a B200).

Tolerances: |out - ref| <= 8e-3 + 1e-2 |ref| elementwise on bf16 outputs,
|lse - ref| <= 1e-3; page tables, cursor and visited-pair counts bit-exact.
"""
import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq, Workload
from tests.harness import (bf16_to_f64, gpu_replay, make_kv, oracle_replay, q_for_call, step_queries, to_dev,
                           within_tolerance)

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def run_prefill_case(torch, w: Workload, layer=0, ctx_chunk=4096, free_list=None, visited=True):
    kv = make_kv(w, free_list=free_list)
    gpu_replay(w, layer, kv, ctx_chunk)
    ids, qs, ql = step_queries(w)
    q = q_for_call(w, layer, ids, qs, ql)
    vis = torch.zeros((len(ids), w.hq), dtype=torch.int64, device="cuda") if visited else None
    out, lse = kv.prefill(layer, ids, qs, ql, to_dev(q), visited=vis)
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    return kv, q, out, lse, vis


def check_against_oracle(w, layer, q, out, lse, vis, ids, qs, ql, ctx_chunk=4096, rows=None):
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, layer, o, ctx_chunk)
    ro, rl, rc = o.attention(layer, ids, qs, ql, q, rows=rows)
    go, gl = bf16_to_f64(out), lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        go = go.reshape(-1, w.d)[rows]
        ro = ro.reshape(-1, w.d)[rows]
        gl = gl.reshape(-1)[rows]
        rl = rl.reshape(-1)[rows]
    ok, worst, at = within_tolerance(go, ro)
    assert ok, f"out mismatch: excess {worst} at {at}"
    assert np.abs(gl - rl).max() <= LSE_TOL, f"lse mismatch {np.abs(gl - rl).max()}"
    if rows is None and vis is not None:
        assert np.array_equal(vis.cpu().numpy().astype(np.uint64), rc)
    return o


def test_tiny_config_full_parity(torch_cuda):
    w = wl.CONFIGS["tiny_prefill_L1024_D64"]
    kv, q, out, lse, vis = run_prefill_case(torch_cuda, w)
    ids, qs, ql = step_queries(w)
    o = check_against_oracle(w, 0, q, out, lse, vis, ids, qs, ql)
    assert np.array_equal(kv.page_table.cpu().numpy(), o.page_table())
    assert int(kv.state[0].item()) == o.cursor


@pytest.mark.parametrize("seed", range(12))
def test_random_small_parity(torch_cuda, seed):
    rng = np.random.default_rng([77, seed])
    base = wl.random_small(seed, max_len=300, d=int(rng.choice([64, 128])))
    page = int(rng.choice([16, 32, 64]))
    ring = min(-(-base.max_seq_len // page), -(-(base.window + base.max_chunk - 1) // page) + 1)
    w = base.scaled(page=page, ring_pages=ring)
    chunk = int(rng.integers(20, 200))
    kv, q, out, lse, vis = run_prefill_case(torch_cuda, w, ctx_chunk=chunk)
    ids, qs, ql = step_queries(w)
    o = check_against_oracle(w, 0, q, out, lse, vis, ids, qs, ql, ctx_chunk=chunk)
    assert np.array_equal(kv.page_table.cpu().numpy(), o.page_table())


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_gqa_groups_and_ragged_lengths(torch_cuda, g):
    hkv = 2
    w = Workload(300 + g, "gqa", 1, hkv * g, hkv, 128, 64, 200, 16,
                 (Seq(0, 777, 0, 777), Seq(0, 300, 0, 300), Seq(0, 1000, 0, 1000)), ((1, 0),))
    kv, q, out, lse, vis = run_prefill_case(torch_cuda, w)
    ids, qs, ql = step_queries(w)
    check_against_oracle(w, 0, q, out, lse, vis, ids, qs, ql)


# edge configurations: a window of one key (each query sees only itself on a local head), 16
# query heads a KV head (8 positions a 128-row tile), a layer whose heads are all local and
# one whose heads are all global; ragged lengths that end mid-tile and mid-page
@pytest.mark.parametrize("name,g,window,cls", [("w1", 2, 1, (1, 0)), ("g16", 16, 100, (0, 1)),
                                               ("all_local", 4, 64, (0, 0)), ("all_global", 4, 64, (1, 1))])
def test_edge_windows_groups_and_classes(torch_cuda, name, g, window, cls):
    hkv = 2
    seqs = (Seq(0, 333, 0, 333), Seq(0, 70, 0, 70), Seq(0, 1, 0, 1))
    w = Workload(340 + g + window, name, 1, hkv * g, hkv, 128, 16, window, 64, seqs, (cls,))
    kv, q, out, lse, vis = run_prefill_case(torch_cuda, w)
    ids, qs, ql = step_queries(w)
    o = check_against_oracle(w, 0, q, out, lse, vis, ids, qs, ql)
    assert np.array_equal(kv.page_table.cpu().numpy(), o.page_table())


def test_mistral_shape_scaled_length(torch_cuda):
    w = wl.CONFIGS["mistral7b_prefill_L8192"].scaled(seqs=(Seq(0, 2048, 0, 2048),), ring_pages=32)
    kv, q, out, lse, vis = run_prefill_case(torch_cuda, w)
    ids, qs, ql = step_queries(w)
    check_against_oracle(w, 0, q, out, lse, vis, ids, qs, ql)


def test_long_items_cut_into_key_chunks(torch_cuda):
    # one global KV head under 8 query heads: 128 items of 1..32 key tiles against a per-SM
    # share of about 15, so the longer items run as several key-range chunks merged by the
    # combine kernel; a local head beside it keeps whole items
    w = Workload(320, "chunks", 1, 16, 2, 128, 64, 700, 64, (Seq(0, 4096, 0, 4096),), ((1, 0),))
    kv, q, out, lse, vis = run_prefill_case(torch_cuda, w)
    ids, qs, ql = step_queries(w)
    check_against_oracle(w, 0, q, out, lse, vis, ids, qs, ql)


def test_chunked_prefill_at_offset_with_ring(torch_cuda):
    w = wl.CONFIGS["mha_chunked_prefill_128k"].scaled(
        seqs=(Seq(6000, 1000, 6000, 7000),), ring_pages=-(-(4096 + 1000 - 1) // 64) + 1)
    kv, q, out, lse, vis = run_prefill_case(torch_cuda, w, ctx_chunk=1500)
    ids, qs, ql = step_queries(w)
    check_against_oracle(w, 0, q, out, lse, vis, ids, qs, ql, ctx_chunk=1500)


def test_page_permutation_gives_identical_bits(torch_cuda):
    w = wl.CONFIGS["tiny_prefill_L1024_D64"]
    a = run_prefill_case(torch_cuda, w, free_list=np.random.default_rng(11).permutation(w.num_pages))
    b = run_prefill_case(torch_cuda, w, free_list=np.random.default_rng(12).permutation(w.num_pages))
    assert not torch_cuda.equal(a[0].page_table, b[0].page_table)
    assert torch_cuda.equal(a[2], b[2]) and torch_cuda.equal(a[3], b[3])


# -- decode -----------------------------------------------------------------------------------
def run_decode_case(torch, w: Workload, ctx_chunk=4096, num_splits=0):
    kv = make_kv(w)
    gpu_replay(w, 0, kv, ctx_chunk)
    ids = list(range(len(w.seqs)))
    qp = [s.q_lo for s in w.seqs]
    q = np.concatenate([w.q(0, b, s.q_lo, s.q_lo + 1) for b, s in enumerate(w.seqs)], axis=0)
    vis = torch.zeros((len(ids), w.hq), dtype=torch.int64, device="cuda")
    out, lse = kv.decode(0, ids, qp, to_dev(q), visited=vis, num_splits=num_splits)
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o, ctx_chunk)
    ro, rl, rc = o.attention(0, ids, qp, [1] * len(ids), q)
    ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
    assert ok, f"out mismatch: excess {worst} at {at}"
    assert np.abs(lse.cpu().numpy() - rl).max() <= LSE_TOL
    assert np.array_equal(vis.cpu().numpy().astype(np.uint64), rc)
    assert np.array_equal(kv.page_table.cpu().numpy(), o.page_table())
    return out, lse


@pytest.mark.parametrize("splits", [0, 1, 3])
def test_decode_small_parity(torch_cuda, splits):
    w = wl.CONFIGS["decode_64x32k"].scaled(
        seqs=tuple(Seq(1500 + 97 * i, 1, 1500 + 97 * i, 1501 + 97 * i) for i in range(5)), window=512,
        ring_pages=-(-512 // 64) + 1)
    run_decode_case(torch_cuda, w, ctx_chunk=700, num_splits=splits)
