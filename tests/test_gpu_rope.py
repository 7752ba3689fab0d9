"""Query relocation on the CUDA path (needs a B200) against the fp64 oracle.

segkv_relocate_q turns the queries of local heads by the rotary angle of position -shift
(RedKnot-MLA review, Summary: local-head KV prefilled at canonical position zero is reused
by rotating the queries by the negative position offset).  Tolerance as for attention
outputs: |out - ref| <= 8e-3 + 1e-2 |ref| (one bf16 rounding of an fp32 rotation).
"""
import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq, Workload
from oracle import rope
from tests.harness import bf16_to_f64, make_kv, to_dev, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def bf16_bits(x: np.ndarray) -> np.ndarray:
    return wl.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# hq 8: several tokens a CTA with a ragged last block (8 tokens a block at D 128, 16 at D 64);
# hq 64 at D 128: one token a block; hq 128 at D 128: two passes of 512 16-byte units a token
@pytest.mark.parametrize("d,interleaved,inplace,hkv,g", [(128, False, False, 4, 2), (128, True, True, 4, 2),
                                                         (64, False, True, 4, 2), (64, True, False, 4, 2),
                                                         (128, False, False, 8, 8), (128, True, True, 16, 8)])
def test_relocation_matches_oracle(torch_cuda, d, interleaved, inplace, hkv, g):
    torch = torch_cuda
    cls = tuple(int(k % 3 == 0) for k in range(hkv))  # globals among locals, first head global
    w = Workload(400 + d, "rope", 1, hkv * g, hkv, d, 64, 256, 8, (Seq(0, 64, 0, 64),), (cls,))
    kv = make_kv(w)
    rng = np.random.default_rng([41, d, int(interleaved), hkv])
    T = 777 if hkv * g <= 8 else 131
    q_bits = bf16_bits(rng.standard_normal((T, w.hq, d)))
    shift = rng.integers(-500000, 500000, size=T).astype(np.int32)
    q = to_dev(q_bits)
    sh = torch.from_numpy(shift).cuda()
    out = kv.relocate_q(0, q, sh, out=q if inplace else None, theta_base=500000.0, interleaved=interleaved)
    torch.cuda.synchronize()
    got = bf16_to_f64(out)
    x = wl.bf16_bits_to_f32(q_bits).astype(np.float64)
    ref = rope.relocate(x, shift[:, None], 500000.0, interleaved)
    for h in range(w.hq):
        if w.classes[0][h // g]:  # global head: copied bit for bit
            assert np.array_equal(got[:, h], x[:, h])
        else:
            ok, worst, at = within_tolerance(got[:, h], ref[:, h])
            assert ok, f"head {h}: excess {worst} at {at}"


def test_relocated_queries_over_canonical_keys_match_true_positions(torch_cuda):
    # A document of L tokens sits at offset delta of the serving context.  Local heads keep
    # K computed at canonical positions 0..L-1 (reused from an offline prefill); global heads
    # keep K at the true positions delta + j.  Queries arrive rotated to their true
    # positions; segkv_relocate_q moves the local heads' queries back by delta.  The result
    # must equal attention with every head at its true positions (the oracle, fp64).
    torch = torch_cuda
    L, d, hkv, g, delta, base = 1536, 128, 2, 4, 100000, 10000.0
    w = Workload(420, "rope_e2e", 1, hkv * g, hkv, d, 64, 512, 24, (Seq(0, L, 0, L),), ((1, 0),))
    rng = np.random.default_rng(42)
    k_raw = rng.standard_normal((L, hkv, d)) / np.sqrt(d)
    v = rng.standard_normal((L, hkv, d))
    q_raw = rng.standard_normal((L, w.hq, d))
    j = np.arange(L, dtype=np.float64)
    k_true = rope.rotate(k_raw, (j + delta)[:, None], base)
    k_canon = rope.rotate(k_raw, j[:, None], base)
    k_cache = np.where(np.array([1, 0], dtype=bool)[None, :, None], k_true, k_canon)  # head 0 global
    q_true = rope.rotate(q_raw, (j + delta)[:, None], base)
    kb, vb, qb = bf16_bits(k_cache), bf16_bits(v), bf16_bits(q_true)
    kv = make_kv(w)
    kv.append(0, [0], [0], [L], to_dev(kb), to_dev(vb))
    q_dev = to_dev(qb)
    sh = torch.full((L,), delta, dtype=torch.int32, device="cuda")
    q_rel = kv.relocate_q(0, q_dev, sh, theta_base=base)
    out, lse = kv.prefill(0, [0], [0], [L], q_rel)
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    # oracle: every head at its true positions, from the same bf16 inputs
    kt = bf16_bits(k_true)
    o = orc.Oracle.for_workload(w)
    o.append(0, [0], [0], [L], kt, vb)
    ro, rl, _ = o.attention(0, [0], [0], [L], qb)
    ok, worst, at = within_tolerance(bf16_to_f64(out), ro)
    assert ok, f"out mismatch: excess {worst} at {at}"
    # lse: the relocated query is rounded to bf16 once more, so allow its effect on s*q.k
    assert np.abs(lse.cpu().numpy() - rl).max() <= 2e-2
