"""Host-side tests of libsegkv.so (CPU only): exported symbols, argument validation before
any enqueue, and the longest-processing-time-first plan against the oracle's."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as orc
from head_wise_sparse_b200 import segkv
from head_wise_sparse_b200 import workloads as wl

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "segkv.h")
FAKE = 1 << 40  # a device address the host never dereferences


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(segkv_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = segkv.lib()
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(segkv.EXPORTS) == names


def handle(**kw):
    args = dict(num_layers=1, num_q_heads=8, num_kv_heads=4, head_dim=128, page_size=64, window=256, ring_pages=0,
                max_seqs=4, max_seq_len=4096, max_chunk=512, head_class=[1, 0, 0, 0], num_pages=1000,
                k_pool=FAKE, v_pool=FAKE, page_table=FAKE, free_list=FAKE, state=FAKE)
    args.update(kw)
    return segkv.Handle(**args)


@pytest.mark.parametrize("bad,code", [
    (dict(head_dim=96), 2), (dict(page_size=8), 2), (dict(num_q_heads=6), 1), (dict(num_q_heads=24, num_kv_heads=4), 2),
    (dict(window=0), 1), (dict(k_pool=0), 1), (dict(k_pool=FAKE + 8), 1), (dict(num_pages=0), 1),
])
def test_create_rejects_bad_configurations(bad, code):
    with pytest.raises(segkv.SegkvError) as e:
        handle(**bad)
    assert e.value.code == code


def test_default_ring_size_and_row_length():
    h = handle()
    # min(ceil(4096/64), ceil((256 + 512 - 1)/64) + 1) = min(64, 13)
    assert h.ring_pages == 13 and h.max_lp == 64
    assert handle(ring_pages=5).ring_pages == 5
    assert handle(ring_pages=500).ring_pages == 64


def test_append_validation_happens_before_any_enqueue():
    h = handle(num_pages=20)
    ws = FAKE
    big = 1 << 20
    # start must equal the current length (0)
    assert h.append(0, [0], [5], [10], FAKE, FAKE, ws, big, stream=0) == 1
    # duplicate sequence ids, bad layer, bad seq id
    assert h.append(0, [1, 1], [0, 0], [1, 1], FAKE, FAKE, ws, big, stream=0) == 1
    assert h.append(1, [0], [0], [1], FAKE, FAKE, ws, big, stream=0) == 1
    assert h.append(0, [4], [0], [1], FAKE, FAKE, ws, big, stream=0) == 1
    # past max_seq_len
    assert h.append(0, [0], [0], [4097], FAKE, FAKE, ws, big, stream=0) == 1
    # 1000 tokens: global head 16 pages + 3 local heads x min(16, 13) pages = 55 > 20
    assert h.append(0, [0], [0], [1000], FAKE, FAKE, ws, big, stream=0) == 3
    # workspace too small / misaligned
    assert h.append(0, [0], [0], [10], FAKE, FAKE, ws, 8, stream=0) == 5
    assert h.append(0, [0], [0], [10], FAKE, FAKE, ws + 16, big, stream=0) == 5
    assert h.seq_len(0, 0) == 0 and h.pages_used == 0


def test_fork_validation_happens_before_any_enqueue():
    h = handle()
    for src, dst in ((0, 0), (-1, 1), (0, 4), (4, 0)):
        with pytest.raises(segkv.SegkvError) as e:
            h.fork(src, dst, stream=0)
        assert e.value.code == 1
    assert h.seq_len(0, 1) == 0


def test_attention_validation_happens_before_any_enqueue():
    h = handle()
    big = 1 << 20
    # nothing appended: any query is past the sequence's length
    assert h.prefill(0, [0], [0], [1], FAKE, 0.0, FAKE, FAKE, None, FAKE, big, stream=0) == 1
    assert h.decode(0, [0], [0], FAKE, 0.0, 0, FAKE, FAKE, None, FAKE, big, stream=0) == 1
    # an empty query range is a no-op
    assert h.prefill(0, [0], [0], [0], FAKE, 0.0, FAKE, FAKE, None, FAKE, big, stream=0) == 0
    assert h.decode(0, [0], [0], FAKE, 0.0, -1, FAKE, FAKE, None, FAKE, big, stream=0) == 1


def test_workspace_size_grows_with_batch_and_tokens():
    h = handle()
    a = h.workspace_bytes(1, 1024)
    b = h.workspace_bytes(4, 1024)
    c = h.workspace_bytes(4, 8192)
    assert a % 256 == 0 and a <= b <= c


def test_strerror_names_every_status():
    lib = segkv.lib()
    for code in range(9):
        assert lib.segkv_strerror(code)
    assert b"unknown" in lib.segkv_strerror(99)


@pytest.mark.parametrize("name", ["tiny_prefill_L1024_D64", "mistral7b_prefill_L8192",
                                  "llama70b_varlen_prefill_4x4layers", "mha_chunked_prefill_128k"])
def test_plan_matches_oracle_lpt_order(name):
    w = wl.CONFIGS[name]
    qs = [s.q_lo for s in w.seqs]
    ql = [s.q_hi - s.q_lo for s in w.seqs]
    h = handle(num_layers=w.layers, num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, page_size=w.page,
               window=w.window, ring_pages=w.ring_pages, max_seqs=len(w.seqs), max_seq_len=w.max_seq_len,
               head_class=w.class_array())
    for layer in range(w.layers):
        got, tile_pos, key_tile = h.plan_prefill(layer, qs, ql)
        want = orc.lpt_items(qs, ql, w.classes[layer], w.window, tile_pos, key_tile)
        assert tile_pos == 256 // w.group and key_tile == 128
        assert np.array_equal(got, want)


@pytest.mark.parametrize("seed", range(8))
def test_plan_matches_oracle_on_random_varlen_batches(seed):
    rng = np.random.default_rng([55, seed])
    hkv = int(rng.integers(1, 9))
    g = int(rng.choice([1, 2, 4, 8, 16]))
    nseq = int(rng.integers(1, 9))
    qs = rng.integers(0, 5000, size=nseq)
    ql = rng.integers(0, 3000, size=nseq)
    cls = rng.integers(0, 2, size=hkv)
    W = int(rng.integers(1, 3000))
    h = handle(num_q_heads=hkv * g, num_kv_heads=hkv, head_class=cls, window=W, max_seqs=nseq, max_seq_len=9000)
    got, tile_pos, key_tile = h.plan_prefill(0, qs, ql)
    want = orc.lpt_items(qs, ql, cls, W, tile_pos, key_tile)
    assert np.array_equal(got, want)


def test_decode_step_validation_happens_before_any_enqueue():
    h = handle(max_seq_len=64)
    big = 1 << 20
    # bad pointers (null K/V or query), bad layer, duplicate ids, negative splits
    assert h.decode_step(0, [0], 0, FAKE, FAKE, 0.0, 0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.decode_step(0, [0], FAKE, FAKE, 0, 0.0, 0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.decode_step(1, [0], FAKE, FAKE, FAKE, 0.0, 0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.decode_step(0, [2, 2], FAKE, FAKE, FAKE, 0.0, 0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.decode_step(0, [0], FAKE, FAKE, FAKE, 0.0, -1, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.decode_step(0, [0], FAKE + 8, FAKE, FAKE, 0.0, 0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.seq_len(0, 0) == 0 and h.pages_used == 0


def test_router_validation_happens_before_any_enqueue():
    h = handle()
    big = 1 << 20
    # queries beyond the sequence (length 0), k above q_len, negative k, misaligned lse
    assert h.router_topk(0, [0], [0], [4], FAKE, FAKE, 0.0, [1], FAKE, FAKE, FAKE, big, stream=0) == 1
    assert h.router_topk(0, [0], [0], [0], FAKE, FAKE, 0.0, [1], FAKE, FAKE, FAKE, big, stream=0) == 1
    assert h.router_topk(0, [0], [0], [0], FAKE, FAKE, 0.0, [-1], FAKE, FAKE, FAKE, big, stream=0) == 1
    assert h.router_topk(0, [0, 0], [0, 0], [0, 0], FAKE, FAKE, 0.0, [0, 0], FAKE, FAKE, FAKE, big, stream=0) == 1
    # an empty call (no query tokens) is a no-op
    assert h.router_topk(0, [0], [0], [0], FAKE, FAKE, 0.0, [0], FAKE, FAKE, FAKE, big, stream=0) == 0


def test_two_source_prefill_validation_happens_before_any_enqueue():
    h = handle()
    big = 1 << 20
    # the chunk must start at the sequence's end (0) and on a page boundary
    assert h.prefill_2src(0, [0], [64], [10], FAKE, FAKE, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    # missing chunk tensors, misaligned chunk tensor
    assert h.prefill_2src(0, [0], [0], [10], FAKE, 0, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.prefill_2src(0, [0], [0], [10], FAKE, FAKE + 4, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    # past max_seq_len
    assert h.prefill_2src(0, [0], [0], [4097], FAKE, FAKE, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1


def test_fused_prefill_append_validation_happens_before_any_enqueue():
    h = handle()
    big = 1 << 20
    # not at the sequence's end, not page-aligned, missing or misaligned K/V, past max_seq_len
    assert h.prefill_append(0, [0], [64], [10], FAKE, FAKE, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.prefill_append(0, [0], [0], [10], FAKE, 0, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.prefill_append(0, [0], [0], [10], FAKE, FAKE, FAKE + 4, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    assert h.prefill_append(0, [0], [0], [4097], FAKE, FAKE, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 1
    # the default ring (13 pages of 64) cannot hold a 1000-token chunk's windows after it
    assert h.prefill_append(0, [0], [0], [1000], FAKE, FAKE, FAKE, 0.0, FAKE, FAKE, 0, FAKE, big, stream=0) == 4
    assert h.seq_len(0, 0) == 0 and h.pages_used == 0


def test_binding_argument_counts_match_the_header():
    # every declaration's parameter count equals the binding's ctypes signature, so a change
    # to include/segkv.h that the binding missed fails here rather than on a GPU
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    lib = segkv.lib()
    for name, params in re.findall(r"\b(segkv_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        argtypes = getattr(lib, name).argtypes
        if argtypes is not None:
            assert len(argtypes) == n, (name, len(argtypes), n)


LOG_SCRIPT = """
import sys
sys.path.insert(0, {root!r})
from tests.test_abi_host import handle, FAKE
h = handle(num_pages=20)
print("rc", h.append(0, [0], [5], [10], FAKE, FAKE, FAKE, 1 << 20, stream=0))
print("rc", h.seq_len(0, 0))
print("rc", h.append(1, [0], [0], [1], FAKE, FAKE, FAKE, 1 << 20, stream=0))
"""


def run_logged(env_value, nvtx=False):
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ)
    env.pop("SEGKV_LOG", None)
    env.pop("SEGKV_NVTX", None)
    if env_value is not None:
        env["SEGKV_LOG"] = env_value
    if nvtx:
        env["SEGKV_NVTX"] = "1"  # ranges are pushed and popped; without a profiler they cost nothing
    r = subprocess.run([sys.executable, "-c", LOG_SCRIPT.format(root=root)], capture_output=True, text=True, env=env,
                       timeout=120)
    assert r.returncode == 0, r.stderr
    return r.stdout, [l for l in r.stderr.splitlines() if l.startswith("[segkv]")]


def test_log_switch_reports_failed_calls_and_every_call():
    out, lines = run_logged(None)  # default: silent
    assert "rc 1" in out and lines == []
    out, lines = run_logged("1")  # failures only: an append past the stored length, one on a bad layer
    assert len(lines) == 2 and all(l.startswith("[segkv] segkv_append -> 1 (invalid argument") for l in lines)
    for nvtx in (False, True):
        out, lines = run_logged("2", nvtx)  # every logged entry point, in order (seq_len is a plain query)
        assert out.split() == ["rc", "1", "rc", "0", "rc", "1"]
        assert [l.split()[1] for l in lines] == ["segkv_create", "segkv_append", "segkv_append"]
        assert lines[0].startswith("[segkv] segkv_create -> 0 (ok")
        assert all("us on the host" in l for l in lines)
