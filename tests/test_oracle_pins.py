"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test names what fixes the expected value: a library routine (torch SDPA), a closed
form, brute force without paging, or a hand-worked golden file.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq, Workload, bf16_bits_to_f32
from tests import brute
from tests.harness import oracle_replay, q_for_call, step_queries

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _small(L=96, hq=4, hkv=2, d=16, page=8, window=8, classes=((1, 0),), cfg_id=900, ring=None, ctx=0,
           q_lo=0):
    ring = ring or -(-L // page)
    return Workload(cfg_id, "pin", 1, hq, hkv, d, page, window, ring, (Seq(ctx, L - ctx, q_lo, L),), classes)


def _run(w, q_override=None, k_fn=None, v_fn=None, free_list=None, rows=None, ctx_chunk=4096):
    o = orc.Oracle.for_workload(w, free_list=free_list)
    if k_fn or v_fn:
        from tests import harness

        # appends with substituted K/V values
        for ids, st, cnt in list(harness.context_calls(w, ctx_chunk)) + [harness.step_append(w)]:
            if not ids:
                continue
            k, v = harness.kv_for_call(w, 0, ids, st, cnt)
            k = k_fn(k) if k_fn else k
            v = v_fn(v) if v_fn else v
            o.append(0, ids, st, cnt, k, v)
    else:
        oracle_replay(w, 0, o, ctx_chunk)
    ids, qs, ql = step_queries(w)
    q = q_for_call(w, 0, ids, qs, ql) if q_override is None else q_override
    out, lse, cnt = o.attention(0, ids, qs, ql, q, rows=rows)
    return o, q, out, lse, cnt


# -- a library routine ------------------------------------------------------------------
def test_all_global_equals_torch_sdpa():
    """All-global heads are plain causal attention: torch SDPA (is_causal) in fp64."""
    w = _small(L=96, hq=4, hkv=2, classes=((1, 1),))
    _, q, out, lse, _ = _run(w)
    qt = torch.from_numpy(bf16_bits_to_f32(q).astype(np.float64)).permute(1, 0, 2)       # [Hq, L, D]
    k = torch.from_numpy(bf16_bits_to_f32(w.k(0, 0, 0, 96)).astype(np.float64)).permute(1, 0, 2)
    v = torch.from_numpy(bf16_bits_to_f32(w.v(0, 0, 0, 96)).astype(np.float64)).permute(1, 0, 2)
    k = k.repeat_interleave(2, dim=0)
    v = v.repeat_interleave(2, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(qt[None], k[None], v[None], is_causal=True)[0]
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    # lse: logsumexp of the scaled causal scores
    s = (qt @ k.transpose(1, 2)) / np.sqrt(16.0)
    s = s.masked_fill(torch.triu(torch.ones(96, 96, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).T.numpy(), rtol=0, atol=1e-12)


# -- closed forms ------------------------------------------------------------------------
def test_local_with_window_covering_everything_is_global():
    a = _run(_small(L=80, window=80, classes=((0, 0),)))
    b = _run(_small(L=80, window=80, classes=((1, 1),)))
    assert np.array_equal(a[2], b[2]) and np.array_equal(a[3], b[3]) and np.array_equal(a[4], b[4])
    c = _run(_small(L=80, window=79, classes=((0, 0),)))
    assert not np.array_equal(a[2], c[2])  # a window one short must differ


def test_window_one_returns_own_value():
    w = _small(L=64, window=1, classes=((0, 0),))
    _, q, out, lse, cnt = _run(w)
    k = bf16_bits_to_f32(w.k(0, 0, 0, 64)).astype(np.float64)
    v = bf16_bits_to_f32(w.v(0, 0, 0, 64)).astype(np.float64)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    for h in range(4):
        np.testing.assert_array_equal(out[:, h, :], v[:, h // 2, :])
        np.testing.assert_allclose(lse[:, h], (qf[:, h, :] * k[:, h // 2, :]).sum(-1) / 4.0, rtol=0, atol=1e-13)
    assert (cnt == 64).all()


def test_zero_query_is_mean_of_visible_values():
    w = _small(L=72, window=10, classes=((1, 0),))
    q0 = np.zeros((72, 4, 16), np.uint16)
    _, _, out, lse, _ = _run(w, q_override=q0)
    v = bf16_bits_to_f32(w.v(0, 0, 0, 72)).astype(np.float64)
    for p in range(72):
        lo_local = max(0, p - 10 + 1)
        for h in range(4):
            lo = 0 if h < 2 else lo_local
            np.testing.assert_allclose(out[p, h], v[lo:p + 1, h // 2].mean(0), rtol=0, atol=1e-13)
            assert abs(lse[p, h] - np.log(p + 1 - lo)) < 1e-13


def test_constant_values_pass_through():
    w = _small(L=70, window=9, classes=((0, 1),))
    c = wl.f32_to_bf16_bits(np.float32(0.8125))
    _, _, out, _, _ = _run(w, v_fn=lambda v: np.full_like(v, c))
    np.testing.assert_allclose(out, 0.8125, rtol=0, atol=1e-14)


def test_visible_pair_counts_tiny_config_match_closed_form():
    """Full tiny prefill (L=1024, D=64, W=128): per-head counts against the golden closed forms."""
    w = wl.CONFIGS["tiny_prefill_L1024_D64"]
    g = _load("visible_pairs.json")[w.name]
    _, _, out, lse, cnt = _run(w)
    G = w.group
    for h in range(w.hq):
        want = g["global"] if w.classes[0][h // G] else g["local"]
        assert int(cnt[0, h]) == want
    assert np.isfinite(out).all() and np.isfinite(lse).all()


def test_sampled_row_counts_follow_closed_form_at_full_size():
    """Rows sampled from the 128K chunked config: count = p + 1 (global) or W (local)."""
    w = wl.CONFIGS["mha_chunked_prefill_128k"].scaled(seqs=(Seq(4096 + 64, 64, 4096, 4096 + 128),))
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(128 * w.hq, 40, replace=False)).astype(np.int64)
    o, q, out, lse, _ = _run(w, rows=rows)
    ids, qs, ql = step_queries(w)
    assert np.isfinite(out.reshape(-1, w.d)[rows]).all() and np.isnan(lse.reshape(-1)[np.setdiff1d(np.arange(128 * w.hq), rows)]).all()
    for r in rows[:8]:
        _, _, c = o.attention(0, ids, qs, ql, q, rows=np.array([r]))
        p = 4096 + r // w.hq
        want = (p + 1) if w.classes[0][r % w.hq] else min(p + 1, w.window)
        assert int(c.sum()) == want


# -- brute force without paging ----------------------------------------------------------
@pytest.mark.parametrize("seed", range(24))
def test_random_small_cases_match_dense_brute_force(seed):
    w = wl.random_small(seed)
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o, ctx_chunk=int(np.random.default_rng(seed).integers(1, 40)))
    ids, qs, ql = step_queries(w)
    q = q_for_call(w, 0, ids, qs, ql)
    out, lse, cnt = o.attention(0, ids, qs, ql, q)
    row = 0
    for i, b in enumerate(ids):
        s = w.seqs[b]
        kb, vb = w.k(0, b, 0, s.length), w.v(0, b, 0, s.length)
        qb = q[row:row + ql[i]]
        bo, bl, bc = brute.dense_masked_attention(qb, kb, vb, np.arange(s.q_lo, s.q_hi), w.classes[0],
                                                  w.window, 1.0 / np.sqrt(w.d))
        np.testing.assert_allclose(out[row:row + ql[i]], bo, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[row:row + ql[i]], bl, rtol=0, atol=1e-12)
        assert np.array_equal(cnt[i].astype(np.int64), bc.astype(np.int64))
        row += ql[i]


# -- storage: page tables, permutation, ring ----------------------------------------------
def test_page_table_matches_hand_worked_example():
    g = _load("page_table_small.json")
    o = orc.Oracle(layers=1, hq=g["hq"], hkv=g["hkv"], d=g["d"], page=g["page"], window=g["window"],
                   ring=g["ring"], max_seqs=g["max_seqs"], max_seq_len=g["max_seq_len"],
                   num_pages=len(g["free_list"]), classes=np.array(g["classes"]), free_list=np.array(g["free_list"]))
    rng = np.random.default_rng(0)
    for call, cur in zip(g["calls"], g["cursor_after"]):
        n = sum(call["count"])
        k = rng.integers(0, 1 << 14, size=(n, 2, 4)).astype(np.uint16)
        o.append(0, call["seq_ids"], call["start"], call["count"], k, k)
        assert o.cursor == cur
    assert np.array_equal(o.page_table(), np.array(g["page_table"], dtype=np.int32))
    pr = g["resident_probe"]
    q = np.zeros((1, 2, 4), np.uint16)
    # the ring dropped position 3 of the local head: only the wide window reaches it
    o2 = orc.Oracle(layers=1, hq=2, hkv=2, d=4, page=4, window=pr["window_ok"], ring=2, max_seqs=2,
                    max_seq_len=16, num_pages=10, classes=np.array(g["classes"]), free_list=np.array(g["free_list"]))
    o3 = orc.Oracle(layers=1, hq=2, hkv=2, d=4, page=4, window=pr["window_evicted"], ring=2, max_seqs=2,
                    max_seq_len=16, num_pages=10, classes=np.array(g["classes"]), free_list=np.array(g["free_list"]))
    for oo in (o2, o3):
        for call in g["calls"]:
            n = sum(call["count"])
            k = rng.integers(0, 1 << 14, size=(n, 2, 4)).astype(np.uint16)
            oo.append(0, call["seq_ids"], call["start"], call["count"], k, k)
    o2.attention(0, [pr["seq"]], [pr["q_pos"]], [1], q)
    with pytest.raises(orc.OracleError):
        o3.attention(0, [pr["seq"]], [pr["q_pos"]], [1], q)


def test_page_table_invariants_on_a_chunked_workload():
    w = wl.CONFIGS["decode_64x32k"].scaled(seqs=tuple(Seq(1000 + 37 * i, 1, 1000 + 37 * i, 1001 + 37 * i)
                                                      for i in range(6)), window=256, ring_pages=5)
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o, ctx_chunk=300)
    pt = o.page_table()
    ids = pt[pt >= 0]
    assert len(np.unique(ids)) == ids.size == o.cursor
    assert set(ids.tolist()) == set(w.free_list()[:o.cursor].tolist())
    g = w.classes[0].index(1)
    for b, s in enumerate(w.seqs):
        n = -(-s.length // w.page)
        assert (pt[0, b, g, :n] >= 0).all() and (pt[0, b, g, n:] == -1).all()
        for h in range(w.hkv):
            if h != g:
                assert (pt[0, b, h, :5] >= 0).all() and (pt[0, b, h, 5:] == -1).all()


def test_physical_page_permutation_does_not_change_results():
    w = _small(L=120, page=8, window=20, classes=((1, 0),))
    a = _run(w, free_list=np.random.default_rng(1).permutation(w.num_pages))
    b = _run(w, free_list=np.random.default_rng(2).permutation(w.num_pages))
    assert not np.array_equal(a[0].page_table(), b[0].page_table())
    assert np.array_equal(a[2], b[2]) and np.array_equal(a[3], b[3])


def test_ring_keeps_window_across_chunked_appends():
    """Appending the same tokens in many small calls (ring wraps several times) gives the
    same result as one call into unwrapped storage."""
    base = _small(L=200, page=8, window=24, classes=((0, 1),), ctx=150, q_lo=170)
    ringed = base.scaled(ring_pages=-(-(24 + 50 - 1) // 8) + 1)
    a = _run(base)
    b = _run(ringed, ctx_chunk=13)
    assert np.array_equal(a[2], b[2]) and np.array_equal(a[3], b[3])
    assert b[0].cursor < a[0].cursor


def test_lpt_order_matches_hand_worked_example():
    g = _load("lpt_small.json")
    items = orc.lpt_items(g["q_start"], g["q_len"], g["classes"], g["window"], g["tile_pos"], g["bn"])
    assert items.tolist() == g["items"]
