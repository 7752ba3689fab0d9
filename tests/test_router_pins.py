"""Pins of the oracle's attention-as-router scores and top-k selection (CPU only).

Reading (zhichai.net news item "What Happened", item 2; hysenlabs.com write-up, "The Three
Core Mechanisms in Detail", second mechanism): a token's score is the attention mass it
receives -- the softmax weights of every query head and every query of the call that sees
it -- and the FFN runs on the k highest-scoring tokens of each sequence.
"""
import json
import os

import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq, Workload
from tests import brute
from tests.harness import oracle_replay, q_for_call, step_queries

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _small(L=96, hq=4, hkv=2, d=16, page=8, window=8, classes=((1, 0),), ctx=0, q_lo=0):
    return Workload(901, "router-pin", 1, hq, hkv, d, page, window, -(-L // page), (Seq(ctx, L - ctx, q_lo, L),),
                    classes)


def _scores(w, q=None):
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o)
    ids, qs, ql = step_queries(w)
    q = q_for_call(w, 0, ids, qs, ql) if q is None else q
    return o.router_scores(0, ids, qs, ql, q), q


# -- brute force without paging ----------------------------------------------------------
@pytest.mark.parametrize("seed", range(12))
def test_scores_match_dense_brute_force(seed):
    w = wl.random_small(seed)
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o, ctx_chunk=int(np.random.default_rng(seed).integers(1, 40)))
    ids, qs, ql = step_queries(w)
    q = q_for_call(w, 0, ids, qs, ql)
    sc = o.router_scores(0, ids, qs, ql, q)
    row = 0
    for i, b in enumerate(ids):
        s = w.seqs[b]
        ref = brute.dense_received_attention(q[row:row + ql[i]], w.k(0, b, 0, s.length), np.arange(s.q_lo, s.q_hi),
                                             s.q_lo, s.q_hi, w.classes[0], w.window, 1.0 / np.sqrt(w.d))
        np.testing.assert_allclose(sc[row:row + ql[i]], ref, rtol=1e-12, atol=1e-12)
        row += ql[i]


def test_chunk_at_an_offset_scores_only_its_own_tokens():
    w = _small(L=80, ctx=37, q_lo=37, window=12)
    sc, q = _scores(w)
    ref = brute.dense_received_attention(q, w.k(0, 0, 0, 80), np.arange(37, 80), 37, 80, w.classes[0], w.window,
                                         1.0 / np.sqrt(w.d))
    np.testing.assert_allclose(sc, ref, rtol=1e-12, atol=1e-12)


# -- invariants and closed forms --------------------------------------------------------------
def test_scores_of_a_whole_sequence_sum_to_heads_times_queries():
    # every query row's weights sum to 1 and every key it sees lies in the range
    w = _small(L=96)
    sc, _ = _scores(w)
    assert abs(sc.sum() - w.hq * 96) < 1e-9


def test_zero_queries_give_harmonic_sums():
    # Q = 0: a query spreads its weight evenly, 1 / (number of keys it sees)
    L, W = 96, 8
    w = _small(L=L, window=W)
    T = L
    sc, _ = _scores(w, q=np.zeros((T, w.hq, w.d), dtype=np.uint16))
    G = w.hq // w.hkv
    ref = np.zeros(L)
    for j in range(L):
        glob = sum(1.0 / (i + 1) for i in range(j, L))
        loc = sum(1.0 / min(i + 1, W) for i in range(j, min(j + W, L)))
        ref[j] = G * glob + G * loc  # KV head 0 global, KV head 1 local
    np.testing.assert_allclose(sc, ref, rtol=1e-13, atol=0)


def test_window_one_gives_every_token_one_per_head():
    w = _small(L=64, window=1, classes=((0, 0),))
    sc, _ = _scores(w)
    np.testing.assert_allclose(sc, np.full(64, float(w.hq)), rtol=0, atol=1e-13)


def test_global_heads_alone_first_token_receives_most():
    # with Q = 0 a global head's first key is seen by every query with weight 1/(i+1)
    w = _small(L=32, classes=((1, 1),))
    sc, _ = _scores(w, q=np.zeros((32, w.hq, w.d), dtype=np.uint16))
    assert np.all(np.diff(sc) < 0)
    assert abs(sc[-1] - w.hq / 32.0) < 1e-15


# -- top-k selection ------------------------------------------------------------------------
def test_topk_matches_hand_worked_cases():
    with open(os.path.join(GOLDEN, "router_topk_small.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        rows = orc.topk_rows(np.array(case["scores"]), case["q_len"], case["k"])
        assert rows.tolist() == case["rows"], case


def test_topk_rejects_k_outside_the_sequence():
    with pytest.raises(orc.OracleError):
        orc.topk_rows(np.zeros(4), [4], [5])


def test_topk_keeps_the_highest_scores_of_each_sequence():
    rng = np.random.default_rng(7)
    s = rng.random(300)
    q_len, k = [100, 150, 50], [10, 150, 0]
    rows = orc.topk_rows(s, q_len, k)
    off = 0
    picked = set(rows.tolist())
    for n, kk in zip(q_len, k):
        mine = [r for r in range(off, off + n) if r in picked]
        assert len(mine) == kk
        rest = [r for r in range(off, off + n) if r not in picked]
        if mine and rest:
            assert min(s[mine]) >= max(s[rest])
        off += n
    assert rows.tolist() == sorted(rows.tolist())
