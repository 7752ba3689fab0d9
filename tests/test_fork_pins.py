"""Pins of the oracle's fork and copy-on-write append (CPU only).

The reading (hysenlabs.com write-up, "Experimental Features and Current Limitations": a
shared KV manager with forks and copy-on-write append): a fork gives an empty sequence the
source's page-table rows and length, sharing the pages; an append that touches a slot whose
page another sequence shares takes a fresh page, in the usual allocation order, after the
shared content is copied into it.  Pinned by a hand-worked page table and by equivalence
with sequences built without any sharing (same tokens, fresh pages).
"""
import json
import os

import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(rng, shape):
    return wl.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def test_page_tables_match_hand_worked_fork():
    g = json.load(open(os.path.join(GOLDEN, "fork_small.json")))
    o = orc.Oracle(layers=g["layers"], hq=g["hq"], hkv=g["hkv"], d=g["d"], page=g["page"], window=g["window"],
                   ring=g["ring"], max_seqs=g["max_seqs"], max_seq_len=g["max_seq_len"],
                   num_pages=len(g["free_list"]), classes=np.array(g["classes"]), free_list=np.array(g["free_list"]))
    rng = np.random.default_rng(3)
    for st in g["steps"]:
        if st["op"] == "fork":
            o.fork(st["src"], st["dst"])
        else:
            n = st["count"]
            o.append(0, [st["seq"]], [st["start"]], [n], bits(rng, (n, g["hkv"], g["d"])),
                     bits(rng, (n, g["hkv"], g["d"])))
    pt = o.page_table()[0]
    assert pt[0].tolist() == g["page_table"]["seq0"]
    assert pt[1].tolist() == g["page_table"]["seq1"]
    assert o.cursor == g["cursor"]


def make(hkv=2, g=2, d=16, page=4, window=9, ring=4, max_seqs=3, max_len=64, classes=(1, 0), seed=0, n_pages=96):
    free = np.random.default_rng([77, seed]).permutation(n_pages)
    return orc.Oracle(layers=1, hq=hkv * g, hkv=hkv, d=d, page=page, window=window, ring=ring, max_seqs=max_seqs,
                      max_seq_len=max_len, num_pages=n_pages, classes=np.array(classes), free_list=free)


def attend(o, seq, lo, hi, q):
    out, lse, cnt = o.attention(0, [seq], [lo], [hi - lo], q)
    return out, lse


@pytest.mark.parametrize("fork_at", [6, 8, 13])
def test_forked_sequences_equal_sequences_built_alone(fork_at):
    hkv, g, d = 2, 2, 16
    rng = np.random.default_rng([5, fork_at])
    prefix_k, prefix_v = bits(rng, (fork_at, hkv, d)), bits(rng, (fork_at, hkv, d))
    a_k, a_v = bits(rng, (11, hkv, d)), bits(rng, (11, hkv, d))
    b_k, b_v = bits(rng, (7, hkv, d)), bits(rng, (7, hkv, d))
    shared = make(seed=fork_at)
    shared.append(0, [0], [0], [fork_at], prefix_k, prefix_v)
    shared.fork(0, 1)
    q0 = bits(rng, (fork_at, hkv * g, d))
    # the fork reads exactly like its source before either changes
    o0, l0 = attend(shared, 0, 0, fork_at, q0)
    o1, l1 = attend(shared, 1, 0, fork_at, q0)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    # diverge: seq 1 first (copy on write of the shared tail page), then seq 0
    shared.append(0, [1], [fork_at], [7], b_k, b_v)
    shared.append(0, [0], [fork_at], [11], a_k, a_v)
    alone = make(seed=fork_at + 100)
    alone.append(0, [0], [0], [fork_at], prefix_k, prefix_v)
    alone.append(0, [0], [fork_at], [11], a_k, a_v)
    alone.append(0, [1], [0], [fork_at], prefix_k, prefix_v)
    alone.append(0, [1], [fork_at], [7], b_k, b_v)
    for seq, n in ((0, fork_at + 11), (1, fork_at + 7)):
        # the last 3 positions: their windows (9 keys) lie in the 4 pages the ring keeps
        q = bits(rng, (3, hkv * g, d))
        o_s, l_s = attend(shared, seq, n - 3, n, q)
        o_a, l_a = attend(alone, seq, n - 3, n, q)
        assert np.array_equal(o_s, o_a) and np.array_equal(l_s, l_a)


def test_appends_to_a_fork_never_change_the_source():
    hkv, g, d = 2, 2, 16
    rng = np.random.default_rng(9)
    o = make(seed=9)
    o.append(0, [0], [0], [10], bits(rng, (10, hkv, d)), bits(rng, (10, hkv, d)))
    o.fork(0, 2)
    q = bits(rng, (10, hkv * g, d))
    before = attend(o, 0, 0, 10, q)
    for start in range(10, 30, 5):
        o.append(0, [2], [start], [5], bits(rng, (5, hkv, d)), bits(rng, (5, hkv, d)))
    after = attend(o, 0, 0, 10, q)
    assert np.array_equal(before[0], after[0]) and np.array_equal(before[1], after[1])
    pt = o.page_table()[0]
    # the global head's first two pages are still shared (never written after the fork) ...
    assert pt[2, 0, 0] == pt[0, 0, 0] and pt[2, 0, 1] == pt[0, 0, 1]
    # ... the page holding the fork point (position 10 on page 2) was copied for the fork
    assert pt[2, 0, 2] != pt[0, 0, 2]


def test_fork_rejects_a_non_empty_destination():
    o = make(seed=1)
    rng = np.random.default_rng(1)
    o.append(0, [0], [0], [3], bits(rng, (3, 2, 16)), bits(rng, (3, 2, 16)))
    o.append(0, [1], [0], [2], bits(rng, (2, 2, 16)), bits(rng, (2, 2, 16)))
    with pytest.raises(orc.OracleError):
        o.fork(0, 1)
    with pytest.raises(orc.OracleError):
        o.fork(0, 0)
