"""The allocation-free decode entry point (segkv_decode_attn_noalloc) against the regular
decode entry point, through the C ABI, on a B200.

Some callers cannot give the library device memory: an engine that reserved the whole
GPU for its own allocator, or code under a fixed memory budget.  For them the library
decodes on a fixed scratch array of its own.  This file runs last (pytest collects it
after the others) so that a failure here never hides another test's result; it passes
both alone in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest

from head_wise_sparse_b200 import segkv
from head_wise_sparse_b200 import workloads as wl
from head_wise_sparse_b200.workloads import Seq
from tests.harness import bf16_to_f64, gpu_replay, make_kv, to_dev, within_tolerance

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_the_workspace_decode_twice_in_a_row():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # decode workload shape (Hq 64, Hkv 8, D 128, one global head, local W=4096 rings of 65
    # pages), 16 sequences of 5000-9000 tokens, context appended in 2048-token calls
    base = wl.CONFIGS["decode_64x32k"]
    seqs = tuple(Seq(5000 + 250 * i, 1, 5000 + 250 * i, 5001 + 250 * i) for i in range(16))
    w = base.scaled(seqs=seqs)
    kv = make_kv(w)
    gpu_replay(w, 0, kv, ctx_chunk=2048)
    ids = list(range(len(seqs)))
    qp = [s.q_lo for s in seqs]
    q = to_dev(np.concatenate([w.q(0, b, p, p + 1) for b, p in zip(ids, qp)], axis=0))
    ref_out, ref_lse = kv.decode(0, ids, qp, q)
    torch.cuda.synchronize()
    assert kv.device_status() == 0
    ref_o, ref_l = bf16_to_f64(ref_out), ref_lse.cpu().numpy()
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = kv.handle.decode_noalloc(0, ids, qp, q, 0.0, 0, out, lse, None)
        assert rc == 0, segkv.lib().segkv_last_error(kv.handle.h)
        torch.cuda.synchronize()
        assert kv.device_status() == 0
        ok, worst, at = within_tolerance(bf16_to_f64(out), ref_o)
        assert ok, f"call {call}: out differs by {worst} beyond tolerance at {at}"
        assert np.abs(lse.cpu().numpy() - ref_l).max() <= 1e-3, f"call {call}: lse"
