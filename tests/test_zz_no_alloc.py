"""The allocation-free decode entry point (segkv_decode_attn_noalloc), through the C ABI, on
a B200: against the regular decode entry point and against the fp64 oracle.

Some callers cannot give the library device memory: an engine that reserved the whole
GPU for its own allocator, or code under a fixed memory budget.  For them the library
decodes on a fixed scratch array of its own (reserved when the handle is created).  This
file runs last (pytest collects it after the others) so that a failure here never hides
another test's result; it passes both alone in a fresh process and after the rest of the
suite.
"""
import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import segkv
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq
from tests.harness import bf16_to_f64, gpu_replay, make_kv, oracle_replay, to_dev, within_tolerance

pytestmark = pytest.mark.gpu

INVALID_ARG, WORKSPACE = 1, 5


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def noalloc(torch, kv, ids, qp, q, num_splits=0):
    out = torch.full((len(ids), kv.hq, kv.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((len(ids), kv.hq), float("nan"), dtype=torch.float32, device="cuda")
    rc = kv.handle.decode_noalloc(0, ids, qp, q, 0.0, num_splits, out, lse, None)
    torch.cuda.synchronize()
    return rc, out, lse


def test_noalloc_decode_matches_the_workspace_decode_and_the_oracle(torch_cuda):
    torch = torch_cuda
    # decode workload shape (Hq 64, Hkv 8, D 128, one global head, local W=4096 rings of 65
    # pages), 16 sequences of 5000-8750 tokens, context appended in 2048-token calls
    base = wl.CONFIGS["decode_64x32k"]
    seqs = tuple(Seq(5000 + 250 * i, 1, 5000 + 250 * i, 5001 + 250 * i) for i in range(16))
    w = base.scaled(seqs=seqs)
    kv = make_kv(w)
    gpu_replay(w, 0, kv, ctx_chunk=2048)
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o, ctx_chunk=2048)
    # call 1: every sequence at its last position; call 2: another subset, in another order,
    # at other positions (halfway into each sequence's last page, which its ring still covers)
    ids1 = list(range(len(seqs)))
    qp1 = [s.q_lo for s in seqs]
    ids2 = [15, 2, 9, 4, 11]
    qp2 = [qp1[b] - (qp1[b] % w.page) // 2 for b in ids2]
    assert qp2 != [qp1[b] for b in ids2]
    for call, (ids, qp) in enumerate(((ids1, qp1), (ids2, qp2))):
        qh = np.concatenate([w.q(0, b, p, p + 1) for b, p in zip(ids, qp)], axis=0)
        q = to_dev(qh)
        ref_out, ref_lse = kv.decode(0, ids, qp, q)
        torch.cuda.synchronize()
        assert kv.device_status() == 0
        rc, out, lse = noalloc(torch, kv, ids, qp, q)
        assert rc == 0, segkv.lib().segkv_last_error(kv.handle.h)
        assert kv.device_status() == 0
        ok, worst, at = within_tolerance(bf16_to_f64(out), bf16_to_f64(ref_out))
        assert ok, f"call {call}: out differs from the workspace decode by {worst} beyond tolerance at {at}"
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= 1e-3, f"call {call}: lse"
        # the oracle on a few rows (sequence, query head)
        ro, rl, _ = o.attention(0, ids, qp, [1] * len(ids), qh)
        rows = np.random.default_rng(call).choice(len(ids) * w.hq, 24, replace=False)
        go = bf16_to_f64(out).reshape(-1, w.d)[rows]
        ok, worst, at = within_tolerance(go, ro.reshape(-1, w.d)[rows])
        assert ok, f"call {call}: out differs from the oracle by {worst} beyond tolerance at {at}"
        assert np.abs(lse.cpu().numpy().reshape(-1)[rows] - rl.reshape(-1)[rows]).max() <= 1e-3

    # a repeated sequence id is refused before anything is enqueued, and leaves the check's
    # bitmap clear for the next call
    rc, _, _ = noalloc(torch, kv, [0, 1, 0], [qp1[0], qp1[1], qp1[0]], to_dev(
        np.concatenate([w.q(0, b, qp1[b], qp1[b] + 1) for b in (0, 1, 0)], axis=0)))
    assert rc == INVALID_ARG
    q = to_dev(np.concatenate([w.q(0, b, qp1[b], qp1[b] + 1) for b in (0, 1)], axis=0))
    ref_out, _ = kv.decode(0, [0, 1], qp1[:2], q)
    rc, out, _ = noalloc(torch, kv, [0, 1], qp1[:2], q)
    assert rc == 0 and kv.device_status() == 0
    assert within_tolerance(bf16_to_f64(out), bf16_to_f64(ref_out))[0]


def test_noalloc_decode_refuses_a_call_beyond_its_scratch(torch_cuda):
    torch = torch_cuda
    # 64 sequences queried at position 4095 (64 pages a head) split 32 ways: the fp32
    # partials alone are 64 x 64 heads x 32 splits x 128 x 4 B = 64 MiB, more than the fixed
    # scratch holds
    base = wl.CONFIGS["decode_64x32k"]
    n, ctx = 64, 4095
    w = base.scaled(seqs=tuple(Seq(ctx, 1, ctx, ctx + 1) for _ in range(n)))
    kv = make_kv(w)
    ids = list(range(n))
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    k = torch.randn((n * (ctx + 1), w.hkv, w.d), generator=g, device="cuda").to(torch.bfloat16)
    kv.append(0, ids, [0] * n, [ctx + 1] * n, k, k)
    q = torch.randn((n, w.hq, w.d), generator=g, device="cuda").to(torch.bfloat16)
    rc, _, _ = noalloc(torch, kv, ids, [ctx] * n, q, num_splits=32)
    assert rc == WORKSPACE
    msg = segkv.lib().segkv_last_error(kv.handle.h).decode()
    assert "scratch" in msg and "67108864" in msg, msg
    # the same call with the default split count fits and runs
    ref_out, _ = kv.decode(0, ids, [ctx] * n, q)
    rc, out, _ = noalloc(torch, kv, ids, [ctx] * n, q)
    assert rc == 0 and kv.device_status() == 0
    assert within_tolerance(bf16_to_f64(out), bf16_to_f64(ref_out))[0]
