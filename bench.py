#!/usr/bin/env python
"""Benchmark of the segmented paged attention hot path on B200.

One step = the Llama-3.3-70B-shaped varlen prefill over 4 layers (4 sequences of seeded
lengths in [8192, 32768], Hq 64, Hkv 8, D 128, per layer one global KV head and seven local
heads with W = 2048, 64-token pages, shuffled physical pages): empty the cache, append every
layer's K/V into each head's own pages (page-table build + scatter), and run the causal
varlen prefill of every layer over those pages.  Metric: TFLOP/s over visible (q, k) pairs,
FLOPs = 4 * D * sum of visible pairs over the 4 layers.

The same JSON line carries the other workloads as sub-objects, each with its own roofline:
the Mistral-7B-shaped single-layer prefill, the 128K-context chunked prefill (one-source and
two-source), the tiny prefill, the KV append on three shapes, the batched decode step (64
sequences at 32K, KV GB/s), attention as a router, query relocation and copy on write.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl segkv|reference]

Under torchrun every rank runs its own replica (weak scaling, no collective on the data
path); rank 0 prints one JSON line with the whole-job throughput (max time over ranks).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from head_wise_sparse_b200 import workloads as wl  # noqa: E402

METRIC = "prefill TFLOP/s over visible (q,k) pairs (% BF16 peak); decode KV GB/s (% HBM)"
HEADLINE = "llama70b_varlen_prefill_4x4layers"
PREFILL = "mistral7b_prefill_L8192"
TINY = "tiny_prefill_L1024_D64"
DECODE = "decode_64x32k"
CHUNKED = "mha_chunked_prefill_128k"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_SOURCES = ["head_wise_sparse_b200/csrc/prefill_sm100.cu", "head_wise_sparse_b200/csrc/device_common.cuh"]
DECODE_SOURCES = ["head_wise_sparse_b200/csrc/decode.cu", "head_wise_sparse_b200/csrc/device_common.cuh"]
ROUTER_SOURCES = ["head_wise_sparse_b200/csrc/router_sm100.cu", "head_wise_sparse_b200/csrc/device_common.cuh"]
APPEND_SOURCES = ["head_wise_sparse_b200/csrc/storage.cu", "head_wise_sparse_b200/csrc/device_common.cuh"]
RELOCATE_SOURCES = ["head_wise_sparse_b200/csrc/rope.cu", "head_wise_sparse_b200/csrc/device_common.cuh"]


# ---------------------------------------------------------------------------- helpers
def visible_pairs(w: wl.Workload, layer: int = 0) -> int:
    """Visible (q, k) pairs of the workload's queries: p + 1 (global head) or min(p + 1, W)."""
    n = 0
    for s in w.seqs:
        p = np.arange(s.q_lo, s.q_hi, dtype=np.int64)
        glob = int((p + 1).sum())
        loc = int(np.minimum(p + 1, w.window).sum())
        for h in range(w.hq):
            n += glob if w.classes[layer][h // w.group] else loc
    return n


def rank_tools(torch, dist, device):
    """(barrier, max_over_ranks) for one process per GPU: a no-op and the identity on one
    rank; else a process-group barrier and an all-reduce MAX of a float64 on `device` (the
    GPU under NCCL, the CPU under gloo).  Every multi-GPU time is the slowest rank's."""
    if dist is None:
        return (lambda: None), (lambda x: x)

    def barrier():
        dist.barrier()

    def max_over_ranks(x: float) -> float:
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def whole_job(units_per_rank: float, world: int, t_max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (t_max_ms * 1e-3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK), "fallback"


def sources_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(summary: str, paths):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    kernel source (the summary records the source hash); else None."""
    path = os.path.join(ROOT, "profiles", summary)
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    t = re.search(r"dram_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
    if not m or not t or m.group(1) != sources_hash(paths):
        return None
    return float(t.group(1))


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        self.windows = []

    def mark(self):
        return time.time()

    def stop(self):
        if self.p:
            self.p.terminate()
            try:
                self.p.wait(5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(", ") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        return rows

    def summary(self, t0: float, t1: float):
        rows = self.stop()
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sel, allr = [], []
        for r in rows:
            if len(r) < 10 or (self.uuid and self.uuid not in r[1]):
                continue
            try:
                ts = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            allr.append((ts, r))
            if t0 - 0.05 <= ts <= t1 + 0.05:
                sel.append(r)
        if not sel and allr:  # timed region shorter than the sampling period: nearest samples
            mid = 0.5 * (t0 + t1)
            sel = [min(allr, key=lambda x: abs(x[0] - mid))[1]]
        if not sel:
            return out
        try:
            out["sm_mhz"] = statistics.median(float(r[2]) for r in sel)
            out["sm_max_mhz"] = max(float(r[3]) for r in sel)
        except ValueError:
            pass
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in sel:
            for n, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        out["reasons"] = sorted(reasons)
        out["samples"] = len(sel)
        return out


# ---------------------------------------------------------------------------- oracle (CPU)
def cpu_baseline(w: wl.Workload, budget_s: float, min_s: float):
    """The fp64 oracle timed on this host's cores over a seeded sample of query rows of the
    same workload; returns (TFLOP/s over visible pairs, threads, description)."""
    import oracle as orc
    from tests.harness import oracle_replay, q_for_call, step_queries

    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o)
    ids, qs, ql = step_queries(w)
    q = q_for_call(w, 0, ids, qs, ql)
    total_rows = int(sum(ql)) * w.hq
    rng = np.random.default_rng(12345)
    order = rng.permutation(total_rows)
    done, pairs, t_used, batch = 0, 0, 0.0, 256
    while t_used < min_s and done < total_rows:
        rows = np.sort(order[done:done + batch]).astype(np.int64)
        t = time.perf_counter()
        _, _, cnt = o.attention(0, ids, qs, ql, q, rows=rows)
        t_used += time.perf_counter() - t
        pairs += int(cnt.sum())
        done += len(rows)
        if t_used > 0 and t_used < min_s:
            batch = int(min(max(batch, len(rows) * (min_s - t_used) / max(t_used, 1e-3) * 0.5), 8192))
        if t_used > budget_s:
            break
    tflops = 4.0 * w.d * pairs / t_used / 1e12
    desc = (f"{done} of {total_rows} query rows (seeded uniform sample) of {w.name}, "
            f"{pairs} visible pairs, {t_used:.1f} s")
    return tflops, orc.host_threads(), desc


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle as orc
    from tests.harness import oracle_replay, q_for_call, step_queries

    w = wl.CONFIGS[HEADLINE]
    o = orc.Oracle.for_workload(w)
    oracle_replay(w, 0, o)
    ids, qs, ql = step_queries(w)
    q = q_for_call(w, 0, ids, qs, ql)
    rng = np.random.default_rng(54321)
    total_rows = int(sum(ql)) * w.hq
    rows_per_step = 256
    times, pairs = [], 0
    for step in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(total_rows, rows_per_step, replace=False)).astype(np.int64)
        t = time.perf_counter()
        _, _, cnt = o.attention(0, ids, qs, ql, q, rows=rows)
        dt = time.perf_counter() - t
        if step >= args.warmup:
            times.append(dt)
            pairs += int(cnt.sum())
    total_t = sum(times)
    value = 4.0 * w.d * pairs / total_t / 1e12
    sample = (f"{rows_per_step} seeded random query rows of {w.name} per step "
              f"({pairs} visible pairs over {args.steps} timed steps)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE, "sample": "rows"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": orc.host_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- GPU arm
def new_handle(w: wl.Workload, dev, *, ring=None, max_chunk=None, ws_batch=None, ws_tokens=None, max_seqs=None,
               free_list=None, num_pages=None, max_seq_len=None):
    from head_wise_sparse_b200.segkv import SegKV

    return SegKV(num_layers=w.layers, num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, page_size=w.page,
                 window=w.window, head_class=w.class_array(), num_pages=num_pages or w.num_pages,
                 free_list=w.free_list() if free_list is None else free_list, max_seqs=max_seqs or len(w.seqs),
                 max_seq_len=max_seq_len or w.max_seq_len, ring_pages=ring or w.ring_pages,
                 max_chunk=max_chunk or w.max_chunk, ws_batch=ws_batch or len(w.seqs),
                 ws_tokens=ws_tokens or max(sum(s.q_hi - s.q_lo for s in w.seqs), 1), device=dev)


def events(torch, n, k):
    return [[torch.cuda.Event(enable_timing=True) for _ in range(k)] for _ in range(n)]


def mean_ms(evs, a, b):
    return sum(e[a].elapsed_time(e[b]) for e in evs) / len(evs)


def roofline(achieved, peak, unit, bound, kernel, traffic=None, **extra):
    r = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
         "traffic": traffic, "kernel": kernel}
    r.update(extra)
    return r


def append_bytes(w: wl.Workload, tokens: int) -> int:
    """Algorithmic bytes of appending `tokens` tokens: K and V rows read and written once."""
    return 2 * 2 * tokens * w.hkv * w.d * 2


def bench_headline(args, torch, dev, stream, barrier, max_over_ranks, world, pk, sampler):
    """The Llama-3.3-70B-shaped varlen prefill over 4 layers: reset + 4 appends + 4 prefills."""
    w = wl.CONFIGS[HEADLINE]
    lens = [s.length for s in w.seqs]
    ids, starts, T = list(range(len(lens))), [0] * len(lens), int(sum(lens))
    gen = torch.Generator(device=dev)
    gen.manual_seed(3)
    # seeded N(0, 1) inputs drawn on the device (the workload's distribution; the parity tests
    # use the workload's own bit patterns)
    q = [torch.randn((T, w.hq, w.d), generator=gen, device=dev).to(torch.bfloat16) for _ in range(w.layers)]
    k = [torch.randn((T, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16) for _ in range(w.layers)]
    v = [torch.randn((T, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16) for _ in range(w.layers)]
    out = [torch.empty((T, w.hq, w.d), dtype=torch.bfloat16, device=dev) for _ in range(w.layers)]
    lse = [torch.empty((T, w.hq), dtype=torch.float32, device=dev) for _ in range(w.layers)]
    vis = torch.zeros((w.layers, len(ids), w.hq), dtype=torch.int64, device=dev)
    kv = new_handle(w, dev, ws_tokens=T, max_chunk=max(lens))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    pairs = [visible_pairs(w, l) for l in range(w.layers)]
    flops = 4.0 * w.d * sum(pairs)
    L = w.layers

    def step(ev=None, with_vis=False):
        if ev:
            ev[0].record(stream)
        kv.handle.reset(stream)
        for l in range(L):
            kv.append(l, ids, starts, lens, k[l], v[l])
        if ev:
            ev[1].record(stream)
        for l in range(L):
            kv.prefill(l, ids, starts, lens, q[l], out=out[l], lse=lse[l], visited=vis[l] if with_vis else None)
            if ev:
                ev[2 + l].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during warm-up")
    ev = events(torch, args.steps, 2 + L)
    vis.zero_()
    barrier()
    torch.cuda.synchronize()
    t0 = sampler.mark()
    for s in range(args.steps):
        flush.fill_(s & 0xFF)  # evict L2 between timed steps (not timed)
        step(ev[s], with_vis=True)
    torch.cuda.synchronize()
    barrier()
    t1 = sampler.mark()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the timed steps")
    # the kernel's own count of visited pairs (columns its masks kept) must equal the closed form
    got = vis.sum(dim=(1, 2)).cpu().numpy()
    for l in range(L):
        if int(got[l]) != args.steps * pairs[l]:
            raise RuntimeError(f"layer {l}: visited pairs {int(got[l])} != {args.steps} x {pairs[l]}")
    t_step = max_over_ranks(mean_ms(ev, 0, 2 + L - 1))
    t_app = max_over_ranks(mean_ms(ev, 0, 1))
    t_pre = max_over_ranks(sum(mean_ms(ev, 1 + l, 2 + l) for l in range(L)))
    achieved = flops / (t_pre * 1e-3) / 1e12
    app_b = L * append_bytes(w, T)

    # ------------------------------------------------------------------ query relocation
    # one layer's queries a call (1.4 GB read, 1.4 GB written: no call finds its operands in
    # L2), each layer's in turn with that layer's head classes, seeded offsets in [0, 2^20);
    # calls back to back after a sleep kernel lets the host queue them ahead of the GPU
    shift = torch.randint(0, 1 << 20, (T,), generator=gen, device=dev, dtype=torch.int32)
    for l in range(L):
        kv.relocate_q(l, q[l], shift, out=out[l])
    n_rel = max(args.steps, 12)
    evr = events(torch, n_rel, 2)
    torch.cuda.synchronize()
    torch.cuda._sleep(4_000_000)
    for i, e in enumerate(evr):
        e[0].record(stream)
        kv.relocate_q(i % L, q[i % L], shift, out=out[i % L])
        e[1].record(stream)
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the relocation calls")
    t_rel = max_over_ranks(mean_ms(evr, 0, 1))
    rel_b = 2 * q[0].numel() * 2
    relocate = {"metric": "query relocation GB/s", "value": world * rel_b / (t_rel * 1e-3) / 1e9, "unit": "GB/s",
                "ms_per_call": t_rel, "bytes_per_call": rel_b, "calls": n_rel,
                "queries": f"{T} tokens x {w.hq} heads x {w.d} (one layer of {HEADLINE})",
                "l2": "operands of 2.8 GB a call, calls back to back",
                "roofline": roofline(rel_b / (t_rel * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s", "hbm",
                                     "relocate_q_kernel (events around each segkv_relocate_q)",
                                     profiled_traffic("relocate_llama70b_layer.md", RELOCATE_SOURCES))}

    # ------------------------------------------------------------------ end to end, host buffers
    # every step copies all 4 layers' Q, K and V in from pinned host memory and every layer's
    # output and lse back out.  Layer by layer on three streams, as a serving loop would: the
    # copy in of layer l + 1 and the copy out of layer l - 1 overlap the append + prefill of
    # layer l (PCIe carries both directions at once).  The layers are independent, so append
    # and prefill per layer compute what the reset + 4 appends + 4 prefills step computes.
    q_h = [t.to("cpu").pin_memory() for t in q]
    k_h = [t.to("cpu").pin_memory() for t in k]
    v_h = [t.to("cpu").pin_memory() for t in v]
    out_h = [torch.empty((T, w.hq, w.d), dtype=torch.bfloat16).pin_memory() for _ in range(L)]
    lse_h = [torch.empty((T, w.hq), dtype=torch.float32).pin_memory() for _ in range(L)]
    e2e_steps = max(3, min(args.steps, 8))
    ev2 = events(torch, e2e_steps, 2)
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    barrier()
    torch.cuda.synchronize()
    for s in range(e2e_steps):
        flush.fill_(s & 0xFF)
        ev2[s][0].record(stream)
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(stream)
        ev_in = [torch.cuda.Event() for _ in range(L)]
        ev_done = [torch.cuda.Event() for _ in range(L)]
        with torch.cuda.stream(s_in):
            for l in range(L):
                q[l].copy_(q_h[l], non_blocking=True)
                k[l].copy_(k_h[l], non_blocking=True)
                v[l].copy_(v_h[l], non_blocking=True)
                ev_in[l].record(s_in)
        with torch.cuda.stream(s_cmp):
            kv.handle.reset(s_cmp)
            for l in range(L):
                s_cmp.wait_event(ev_in[l])
                kv.append(l, ids, starts, lens, k[l], v[l])
                kv.prefill(l, ids, starts, lens, q[l], out=out[l], lse=lse[l])
                ev_done[l].record(s_cmp)
        with torch.cuda.stream(s_out):
            for l in range(L):
                s_out.wait_event(ev_done[l])
                out_h[l].copy_(out[l], non_blocking=True)
                lse_h[l].copy_(lse[l], non_blocking=True)
        for st in (s_in, s_cmp, s_out):
            stream.wait_stream(st)
        ev2[s][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the end-to-end steps")
    # the last end-to-end step's outputs, read back through the host, equal the device-timed
    # step's (same inputs, same kernels)
    step()
    torch.cuda.synchronize()
    for l in range(L):
        if not torch.equal(out_h[l], out[l].cpu()):
            raise RuntimeError(f"layer {l}: end-to-end output differs from the device step's")
    t_e2e = max_over_ranks(mean_ms(ev2, 0, 1))
    h2d = sum(t.numel() * t.element_size() for t in q_h + k_h + v_h)
    d2h = sum(t.numel() * t.element_size() for t in out_h + lse_h)
    e2e = {"value": world * flops / (t_e2e * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": t_e2e, "steps": e2e_steps,
           "overlap": "per layer on three streams: copy in, append + prefill, copy out"}
    res = {
        "value": world * flops / (t_step * 1e-3) / 1e12, "ms_per_step": t_step, "prefill_kernel_ms": t_pre,
        "append_ms": t_app, "flops_per_step": flops, "visible_pairs_per_layer": pairs, "e2e": e2e,
        "relocate": relocate,
        "roofline": roofline(achieved, pk["bf16_tflops"], "TFLOP/s", "tensor",
                             "prefill_kernel<128> (events around the 4 segkv_prefill_attn calls of a step)",
                             profiled_traffic("prefill_llama70b_varlen.md", PREFILL_SOURCES),
                             peak_source="measured bf16 burst (cuBLAS)",
                             frac_of_sustained=achieved / pk["bf16_tflops_sustained"]),
        "append": {"bytes": app_b, "ms": t_app, "GB/s": app_b / (t_app * 1e-3) / 1e9,
                   "roofline": roofline(app_b / (t_app * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s", "hbm",
                                        "reset_kernel + append_kernel x 4 (events around reset + the 4 segkv_append calls)",
                                        profiled_traffic("append_llama70b_layer.md", APPEND_SOURCES),
                                        traffic_per="append_kernel launch (one layer)")},
        "config": {"workload": HEADLINE, "layers": L, "seq_lens": lens, "q_heads": w.hq, "kv_heads": w.hkv,
                   "head_dim": w.d, "page_size": w.page, "window": w.window,
                   "global_kv_heads_per_layer": [int(sum(c)) for c in w.classes],
                   "step": "reset + append of 4 layers (page ids + scatter) + prefill of 4 layers",
                   "l2": "inputs larger than L2 (1.4 GB of Q a layer); L2 also flushed between timed steps "
                         "(256 MiB write, outside the events)",
                   "parallelism": f"replicas x{world}", "global_batch": len(lens), "seq_len": max(lens)},
        "gpu_launches": (1 + 2 * L) * args.steps,
        "clock_window": (t0, t1),
    }
    del kv, q, k, v, out, lse, q_h, k_h, v_h, out_h, lse_h, flush
    torch.cuda.empty_cache()
    return res


def bench_mistral(args, torch, dev, stream, max_over_ranks, world, pk):
    """The Mistral-7B-shaped single-layer step (reset + append + prefill), the same work as one
    fused call, and the router and query relocation on the same queries."""
    w = wl.CONFIGS[PREFILL]
    L = w.seqs[0].length
    dev_bf16 = lambda bits: torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
    q_d, k_d, v_d = dev_bf16(w.q(0, 0, 0, L)), dev_bf16(w.k(0, 0, 0, L)), dev_bf16(w.v(0, 0, 0, L))
    kv = new_handle(w, dev, ws_tokens=L, max_chunk=L)
    out = torch.empty((L, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((L, w.hq), dtype=torch.float32, device=dev)
    visited = torch.zeros((1, w.hq), dtype=torch.int64, device=dev)
    flops = 4.0 * w.d * visible_pairs(w)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        kv.handle.reset(stream)
        kv.append(0, [0], [0], [L], k_d, v_d)

    for _ in range(args.warmup):
        step()
        kv.prefill(0, [0], [0], [L], q_d, out=out, lse=lse, visited=visited)
    torch.cuda.synchronize()
    ev = events(torch, args.steps, 4)
    visited.zero_()
    for s in range(args.steps):
        flush.fill_(s & 0xFF)
        ev[s][0].record(stream)
        kv.handle.reset(stream)
        ev[s][1].record(stream)
        kv.append(0, [0], [0], [L], k_d, v_d)
        ev[s][2].record(stream)
        kv.prefill(0, [0], [0], [L], q_d, out=out, lse=lse, visited=visited)
        ev[s][3].record(stream)
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the Mistral-shaped steps")
    if int(visited.sum().item()) != args.steps * visible_pairs(w):
        raise RuntimeError("Mistral-shaped visited pairs differ from the closed form")
    t_step = max_over_ranks(mean_ms(ev, 0, 3))
    t_app = max_over_ranks(mean_ms(ev, 1, 2))
    t_pre = max_over_ranks(mean_ms(ev, 2, 3))
    app_b = append_bytes(w, L)
    # the same work as one fused call: reset, then segkv_prefill_append
    for _ in range(args.warmup):
        kv.handle.reset(stream)
        kv.prefill_append(0, [0], [0], [L], q_d, k_d, v_d, out=out, lse=lse)
    evf = events(torch, args.steps, 2)
    for s in range(args.steps):
        flush.fill_(s & 0xFF)
        kv.handle.reset(stream)
        evf[s][0].record(stream)
        kv.prefill_append(0, [0], [0], [L], q_d, k_d, v_d, out=out, lse=lse)
        evf[s][1].record(stream)
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the fused calls")
    t_fused = max_over_ranks(mean_ms(evf, 0, 1))
    res = {
        "workload": PREFILL, "value": world * flops / (t_step * 1e-3) / 1e12, "unit": "TFLOP/s",
        "ms_per_step": t_step, "prefill_kernel_ms": t_pre, "append_ms": t_app,
        "step": "reset + append (page ids + scatter) + prefill",
        "roofline": roofline(flops / (t_pre * 1e-3) / 1e12, pk["bf16_tflops"], "TFLOP/s", "tensor",
                             "prefill_kernel<128> (events around segkv_prefill_attn: metadata upload + kernel)",
                             profiled_traffic("prefill_mistral7b_L8192.md", PREFILL_SOURCES)),
        "append": {"bytes": app_b, "ms": t_app,
                   "roofline": roofline(app_b / (t_app * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s", "hbm",
                                        "append_kernel (events around segkv_append)",
                                        profiled_traffic("append_mistral7b_L8192.md", APPEND_SOURCES))},
        "fused_append_prefill": {"ms_per_call": t_fused, "value": world * flops / (t_fused * 1e-3) / 1e12,
                                 "unit": "TFLOP/s", "two_call_ms": t_app + t_pre,
                                 "step": "segkv_prefill_append (the prefill kernel stores the K/V pages it loads)"},
        "gpu_launches": 3 * args.steps,
    }
    # query relocation: local heads turned by -delta, the global head copied (one read + one
    # write of every query element).  Calls run back to back, as a serving loop issues them,
    # over three (input, output) pairs in turn: 402 MB, so no call finds its operands in L2,
    # and each call writes back the lines the call before it left dirty, as a copy in steady
    # state does.  A sleep kernel first lets the host queue the calls ahead of the GPU, so the
    # events time the GPU's work, not the host's call overhead.
    sets = [(q_d if i == 0 else q_d.clone(), torch.empty_like(q_d)) for i in range(3)]
    shift = torch.full((L,), 100000, dtype=torch.int32, device=dev)
    for i in range(max(args.warmup, 3)):
        kv.relocate_q(0, sets[i % 3][0], shift, out=sets[i % 3][1])
    n_rel = max(args.steps, 30)
    evr = events(torch, n_rel, 2)
    torch.cuda.synchronize()
    torch.cuda._sleep(4_000_000)
    for i, e in enumerate(evr):
        e[0].record(stream)
        kv.relocate_q(0, sets[i % 3][0], shift, out=sets[i % 3][1])
        e[1].record(stream)
    torch.cuda.synchronize()
    t_rel = max_over_ranks(mean_ms(evr, 0, 1))
    rel_b = 2 * q_d.numel() * 2
    res["relocate"] = {"metric": "query relocation GB/s", "value": world * rel_b / (t_rel * 1e-3) / 1e9,
                       "unit": "GB/s", "ms_per_call": t_rel, "bytes_per_call": rel_b, "calls": n_rel,
                       "l2": "three operand sets in turn (402 MB), calls back to back",
                       "roofline": roofline(rel_b / (t_rel * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s", "hbm",
                                            "relocate_q_kernel (events around each segkv_relocate_q)",
                                            profiled_traffic("relocate_mistral7b_8192.md", RELOCATE_SOURCES))}
    del sets
    # attention as a router: every token's received attention mass and the top quarter
    k_top = [L // 4]
    rt_scores = torch.empty((L,), dtype=torch.float32, device=dev)
    rt_rows = torch.empty((L // 4,), dtype=torch.int32, device=dev)
    for _ in range(args.warmup):
        kv.router_topk(0, [0], [0], [L], q_d, lse, k_top, scores=rt_scores, rows=rt_rows)
    evt = events(torch, min(args.steps, 50), 2)
    for e in evt:
        flush.fill_(2)
        e[0].record(stream)
        kv.router_topk(0, [0], [0], [L], q_d, lse, k_top, scores=rt_scores, rows=rt_rows)
        e[1].record(stream)
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the router benchmark")
    t_rt = max_over_ranks(mean_ms(evt, 0, 1))
    pairs = visible_pairs(w)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mufu_peak = 16 * sms * 1965.0 * 1e6 / 1e9  # G exponentials per second at the maximum SM clock
    res["router"] = {"metric": "router visible pairs/s", "value": world * pairs / (t_rt * 1e-3) / 1e9,
                     "unit": "Gpair/s", "ms_per_call": t_rt, "pairs_per_call": pairs, "k": k_top[0],
                     "step": "segkv_router_topk: received attention mass of 8192 tokens (32 query heads) + top 2048",
                     "roofline": roofline(pairs / (t_rt * 1e-3) / 1e9, mufu_peak, "Gexp/s", "alu",
                                          "router_kernel<128> + score_sum_kernel + topk_kernel (events around "
                                          "segkv_router_topk)",
                                          profiled_traffic("router_mistral7b_L8192.md", ROUTER_SOURCES),
                                          peak_source=f"MUFU ex2: 16 per clock per SM x {sms} SMs x 1965 MHz "
                                                      "(the maximum SM clock)"),
                     "gpu_launches": 3 * len(evt)}
    del kv, flush
    torch.cuda.empty_cache()
    return res


def bench_tiny(args, torch, dev, stream, max_over_ranks, world, pk):
    """The tiny prefill (L 1024, Hq 8, Hkv 4, D 64, page 16): a correctness-sized workload whose
    whole run is shorter than a kernel launch's fixed costs."""
    w = wl.CONFIGS[TINY]
    L = w.seqs[0].length
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    k = torch.randn((L, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    q = torch.randn((L, w.hq, w.d), generator=gen, device=dev).to(torch.bfloat16)
    kv = new_handle(w, dev, ws_tokens=L, max_chunk=L)
    kv.append(0, [0], [0], [L], k, k)
    out = torch.empty((L, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((L, w.hq), dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        kv.prefill(0, [0], [0], [L], q, out=out, lse=lse)
    ev = events(torch, args.steps, 2)
    for e in ev:
        e[0].record(stream)
        kv.prefill(0, [0], [0], [L], q, out=out, lse=lse)
        e[1].record(stream)
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the tiny prefill")
    t = max_over_ranks(mean_ms(ev, 0, 1))
    flops = 4.0 * w.d * visible_pairs(w)
    del kv
    return {"workload": TINY, "value": world * flops / (t * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_call": t,
            "roofline": roofline(flops / (t * 1e-3) / 1e12, pk["bf16_tflops"], "TFLOP/s", "tensor",
                                 "prefill_kernel<64> (events around segkv_prefill_attn); launch- and latency-bound"),
            "gpu_launches": len(ev)}


def bench_headline_slice(args, torch, dev, stream, max_over_ranks, world, pk):
    """The headline's prefill kernel on a slice small enough for a full ncu capture (the
    profiling leg): one layer of the Llama-shaped heads (Hq 64, Hkv 8, D 128, W 2048, layer
    0's head classes) over one sequence of 8 192 tokens -- 134 MB of Q, more than L2, under
    1 GB on the device."""
    base = wl.CONFIGS[HEADLINE]
    w = base.scaled(layers=1, classes=base.classes[:1], seqs=(wl.Seq(0, 8192, 0, 8192),))
    L = 8192
    gen = torch.Generator(device=dev)
    gen.manual_seed(17)
    q = torch.randn((L, w.hq, w.d), generator=gen, device=dev).to(torch.bfloat16)
    k = torch.randn((L, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((L, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((L, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((L, w.hq), dtype=torch.float32, device=dev)
    kv = new_handle(w, dev, ws_tokens=L, max_chunk=L)
    kv.append(0, [0], [0], [L], k, v)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    for i in range(args.warmup + args.steps):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kv.prefill(0, [0], [0], [L], q, out=out, lse=lse)
        e1.record(stream)
        if i >= args.warmup:
            times.append((e0, e1))
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the headline slice")
    t = max_over_ranks(sum(a.elapsed_time(b) for a, b in times) / len(times))
    flops = 4.0 * w.d * visible_pairs(w)
    del kv, q, k, v, out, lse, flush
    torch.cuda.empty_cache()
    return {"workload": "llama70b_layer0_heads_one_sequence_8192", "ms": t, "TFLOP/s": flops / (t * 1e-3) / 1e12,
            "frac": flops / (t * 1e-3) / 1e12 / pk["bf16_tflops"]}


def bench_append_layer(args, torch, dev, stream, max_over_ranks, world, pk):
    """The append of one Llama-shaped layer (4 sequences of the seeded lengths, Hkv 8, D 128,
    181 MB of K/V read and written) into an emptied handle, alone (the profiling leg)."""
    w = wl.CONFIGS[HEADLINE].scaled(layers=1, classes=wl.CONFIGS[HEADLINE].classes[:1])
    lens = [s.length for s in w.seqs]
    ids, T = list(range(len(lens))), int(sum(lens))
    gen = torch.Generator(device=dev)
    gen.manual_seed(13)
    k = torch.randn((T, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((T, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    kv = new_handle(w, dev, ws_tokens=T, max_chunk=max(lens))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    for i in range(args.warmup + args.steps):
        kv.handle.reset(stream)
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kv.append(0, ids, [0] * len(lens), lens, k, v)
        e1.record(stream)
        if i >= args.warmup:
            times.append((e0, e1))
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the append leg")
    t = max_over_ranks(sum(a.elapsed_time(b) for a, b in times) / len(times))
    b = append_bytes(w, T)
    del kv, k, v, flush
    torch.cuda.empty_cache()
    return {"workload": "llama70b_one_layer_append", "bytes": b, "ms": t,
            "roofline": roofline(b / (t * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s", "hbm",
                                 "append_kernel (events around segkv_append)",
                                 profiled_traffic("append_llama70b_layer.md", APPEND_SOURCES))}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="segkv", choices=["segkv", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--only", default="", choices=["", "headline", "mistral", "chunked", "tiny", "fork", "decode",
                                                   "append", "headline_slice"],
                    help="run one leg alone (for profiling): the headline step, or one sub-workload; 'append' is the "
                         "append of one Llama-shaped layer (181 MB of K/V, about 1 GB on the device); "
                         "'headline_slice' the headline's prefill kernel on one 8 192-token sequence of its heads")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    barrier, max_over_ranks = rank_tools(torch, dist if world > 1 else None, dev)
    pk, pk_src = peaks()
    stream = torch.cuda.current_stream()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(str(getattr(props, "uuid", "")))
    time.sleep(0.3)

    if args.only and args.only != "headline":
        legs = {"mistral": lambda: bench_mistral(args, torch, dev, stream, max_over_ranks, world, pk),
                "chunked": lambda: bench_chunked(args, torch, dev, stream, max_over_ranks, world, pk),
                "tiny": lambda: bench_tiny(args, torch, dev, stream, max_over_ranks, world, pk),
                "fork": lambda: bench_fork(args, torch, dev, stream, max_over_ranks, world, pk),
                "decode": lambda: bench_decode(args, torch, dev, stream, barrier, max_over_ranks, world, pk),
                "append": lambda: bench_append_layer(args, torch, dev, stream, max_over_ranks, world, pk),
                "headline_slice": lambda: bench_headline_slice(args, torch, dev, stream, max_over_ranks, world, pk)}
        res = legs[args.only]()
        sampler.stop()
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"only": args.only, **res}), flush=True)
        return 0
    head = bench_headline(args, torch, dev, stream, barrier, max_over_ranks, world, pk, sampler)
    t0, t1 = head.pop("clock_window")
    clocks = sampler.summary(t0, t1)
    line = {
        "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) drawn on the device)",
        "config": head["config"], "prefill_kernel_ms": head["prefill_kernel_ms"], "append_ms": head["append_ms"],
        "roofline": head["roofline"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": clocks,
        "peaks": {"source": pk_src, **pk},
    }
    appends = {"llama70b_4_layers": head["append"]}
    line["relocate"] = head["relocate"]
    if not args.only:
        mis = bench_mistral(args, torch, dev, stream, max_over_ranks, world, pk)
        appends["mistral7b"] = mis.pop("append")
        line["relocate"]["mistral7b_8192"] = mis.pop("relocate")
        line["router"] = mis.pop("router")
        line["fused_append_prefill"] = mis.pop("fused_append_prefill")
        line["mistral7b"] = mis
        chunk = bench_chunked(args, torch, dev, stream, max_over_ranks, world, pk)
        appends["chunk_128k"] = chunk.pop("append")
        line["chunked_128k"] = chunk
        line["tiny"] = bench_tiny(args, torch, dev, stream, max_over_ranks, world, pk)
        line["fork"] = bench_fork(args, torch, dev, stream, max_over_ranks, world, pk)
        if not args.no_decode:
            line["decode"] = bench_decode(args, torch, dev, stream, barrier, max_over_ranks, world, pk)
    line["append"] = appends
    if rank == 0 and world == 1 and not args.no_cpu:
        v_cpu, cores, desc = cpu_baseline(wl.CONFIGS[HEADLINE], budget_s=3 * args.cpu_seconds, min_s=args.cpu_seconds)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def bench_chunked(args, torch, dev, stream, max_over_ranks, world, pk):
    """Chunked prefill of the 128K-context MHA workload (4096 queries at 126976, W 4096, P 64,
    4 global + 28 local KV heads): segkv_prefill_attn after the chunk is appended (local rings
    of 129 pages), segkv_prefill_attn_2src before it is appended (rings of
    ceil((W - 1) / P) + 1 = 65 pages: same keys, same FLOPs), and the append of the 4096-token
    chunk itself (into an emptied handle, so every page is a new one)."""
    w = wl.CONFIGS[CHUNKED]
    s = w.seqs[0]
    ctx, C = s.context, s.new
    r_two = -(-(w.window - 1) // w.page) + 1
    handles = {name: new_handle(w, dev, ring=ring, max_chunk=C, ws_tokens=C)
               for name, ring in (("one", w.ring_pages), ("two", r_two))}
    gen = torch.Generator(device=dev)
    gen.manual_seed(12)
    for lo in range(0, ctx, 4096):
        n = min(4096, ctx - lo)
        k = torch.randn((n, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
        v = torch.randn((n, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
        for kv in handles.values():
            kv.append(0, [0], [lo], [n], k, v)
        del k, v
    kc = torch.randn((C, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    vc = torch.randn((C, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    q = torch.randn((C, w.hq, w.d), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((C, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((C, w.hq), dtype=torch.float32, device=dev)
    handles["one"].append(0, [0], [ctx], [C], kc, vc)  # the one-source call needs the chunk stored first
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls = {"one": lambda: handles["one"].prefill(0, [0], [ctx], [C], q, out=out, lse=lse),
             "two": lambda: handles["two"].prefill_2src(0, [0], [ctx], [C], q, kc, vc, out=out, lse=lse)}
    ms = {}
    for name, call in calls.items():
        for _ in range(args.warmup):
            call()
        ev = events(torch, min(args.steps, 20), 2)
        for e in ev:
            flush.fill_(3)
            e[0].record(stream)
            call()
            e[1].record(stream)
        torch.cuda.synchronize()
        ms[name] = max_over_ranks(mean_ms(ev, 0, 1))
    handles["two"].append(0, [0], [ctx], [C], kc, vc)
    torch.cuda.synchronize()
    for kv in handles.values():
        if kv.device_status() != 0:
            raise RuntimeError("device error word set during the chunked-prefill benchmark")
    del handles
    # the chunk's append: 4096 tokens x 32 heads into new pages of an emptied handle
    kv = new_handle(w, dev, ring=w.ring_pages, max_chunk=C, ws_tokens=C)
    app = []
    for i in range(args.warmup + min(args.steps, 20)):
        kv.handle.reset(stream)
        flush.fill_(4)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kv.append(0, [0], [0], [C], kc, vc)
        e1.record(stream)
        if i >= args.warmup:
            app.append((e0, e1))
    torch.cuda.synchronize()
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the chunk append")
    t_app = max_over_ranks(sum(a.elapsed_time(b) for a, b in app) / len(app))
    app_b = append_bytes(w, C)
    del kv, flush
    torch.cuda.empty_cache()
    flops = 4.0 * w.d * visible_pairs(w)
    n_local = int(w.hkv - sum(w.classes[0]))
    page_bytes = 2 * w.page * w.d * 2
    return {
        "workload": CHUNKED, "value": world * flops / (ms["one"] * 1e-3) / 1e12, "unit": "TFLOP/s",
        "ms_per_call": ms["one"],
        "roofline": roofline(flops / (ms["one"] * 1e-3) / 1e12, pk["bf16_tflops"], "TFLOP/s", "tensor",
                             "prefill_kernel<128> + prefill_combine_kernel (events around segkv_prefill_attn)"),
        "two_source": {"metric": "two-source chunked prefill TFLOP/s", "unit": "TFLOP/s",
                       "value": world * flops / (ms["two"] * 1e-3) / 1e12, "ms_per_call": ms["two"],
                       "ring_pages": {"two_source": r_two, "one_source": w.ring_pages},
                       "local_ring_bytes_saved_per_sequence": n_local * (w.ring_pages - r_two) * page_bytes,
                       "roofline": roofline(flops / (ms["two"] * 1e-3) / 1e12, pk["bf16_tflops"], "TFLOP/s",
                                            "tensor", "prefill_kernel<128>, chunk pages from the call's K/V "
                                                      "(events around segkv_prefill_attn_2src)")},
        "append": {"bytes": app_b, "ms": t_app,
                   "roofline": roofline(app_b / (t_app * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s", "hbm",
                                        "append_kernel (events around segkv_append of the 4096-token chunk)",
                                        profiled_traffic("append_chunk128k.md", APPEND_SOURCES))},
        "gpu_launches": 2 * min(args.steps, 20) * 2,
    }


def bench_fork(args, torch, dev, stream, max_over_ranks, world, pk):
    """Copy on write after a fork: 64 sequences of 1000 tokens (Mistral-shaped heads) are
    forked into 8 groups of 64 empty slots; each timed call appends one token to every fork
    of one group, so each of the 8 heads of each fork first copies its shared, partly filled
    last page (the rows before the new token) into a fresh page.  The 8 calls of a step run
    back to back after a sleep kernel lets the host queue them (the events time the GPU's
    work); one call on an idle GPU, host planning included, is reported beside it.  Bytes:
    the copied rows plus the new rows, read and written."""
    from head_wise_sparse_b200.segkv import SegKV

    w = wl.CONFIGS[PREFILL]
    B, ctx, P, NG = 64, 1000, w.page, 8
    n_pages = B * w.hkv * ((ctx // P + 2) + NG) + 64
    free = np.random.default_rng(7).permutation(n_pages).astype(np.int32)
    kv = SegKV(num_layers=1, num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, page_size=P, window=w.window,
               head_class=w.class_array(), num_pages=n_pages, free_list=free, max_seqs=(NG + 1) * B,
               max_seq_len=ctx + 8, ring_pages=-(-(ctx + 8) // P), max_chunk=ctx, ws_batch=B, ws_tokens=B * ctx,
               device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    k = torch.randn((B * ctx, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    k1 = torch.randn((B, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    src = list(range(B))
    groups = [list(range((g + 1) * B, (g + 2) * B)) for g in range(NG)]
    queued, idle = [], []
    for it in range(args.warmup + max(3, min(args.steps, 10))):
        kv.reset()
        kv.append(0, src, [0] * B, [ctx] * B, k, k)
        for grp in groups:
            for a, b in zip(src, grp):
                kv.fork(a, b)
        torch.cuda.synchronize()
        # one group on an idle GPU, host planning and upload inside the events
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kv.append(0, groups[0], [ctx] * B, [1] * B, k1, k1)
        e1.record(stream)
        torch.cuda.synchronize()
        # the other groups back to back, queued behind a sleep kernel
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in groups[1:]]
        torch.cuda._sleep(2_000_000)
        for (a, b), grp in zip(evs, groups[1:]):
            a.record(stream)
            kv.append(0, grp, [ctx] * B, [1] * B, k1, k1)
            b.record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            idle.append(e0.elapsed_time(e1))
            queued.extend(a.elapsed_time(b) for a, b in evs)
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during the fork benchmark")
    t = max_over_ranks(statistics.median(queued))
    t_idle = max_over_ranks(statistics.median(idle))
    moved = B * w.hkv * ((ctx % P) + 1) * w.d * 2 * 2 * 2  # K and V: copied rows read + written, new row
    del kv, k, k1
    torch.cuda.empty_cache()
    return {"metric": "copy-on-write append GB/s", "value": world * moved / (t * 1e-3) / 1e9, "unit": "GB/s",
            "ms_per_call": t, "ms_per_call_idle_gpu": t_idle, "bytes_per_call": moved, "pages_copied": B * w.hkv,
            "step": "append 1 token to 64 forks of 1000-token sequences (8 heads each: 512 shared pages copied); "
                    "calls back to back over 8 fork groups",
            "roofline": {"bound": "hbm", "achieved": moved / (t * 1e-3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": moved / (t * 1e-3) / 1e9 / pk["hbm_gbs"], "traffic": None,
                         "kernel": "append_kernel with the copy on write folded in (events around each segkv_append)"}}


def bench_decode(args, torch, dev, stream, barrier, max_over_ranks, world, pk):
    """Batched decode: 64 sequences, context 32767 (+1 new token per step).  The step runs
    first as the fused segkv_decode_step (the split kernel appends the token itself; split +
    combine), which gives the line's value, then as two calls (segkv_append of the token,
    then segkv_decode_attn: append kernel, split kernel, combine kernel) for comparison."""
    from head_wise_sparse_b200.segkv import SegKV

    w = wl.CONFIGS[DECODE]
    B = len(w.seqs)
    ctx = w.seqs[0].context
    steps = min(args.steps, 100)
    warm = args.warmup
    nsteps = warm + steps
    max_len = ctx + 2 * nsteps + 64
    wmax = w.scaled(seqs=tuple(wl.Seq(ctx, 2 * nsteps + 1, ctx, ctx + 1) for _ in range(B)))
    kv = SegKV(num_layers=1, num_q_heads=w.hq, num_kv_heads=w.hkv, head_dim=w.d, page_size=w.page, window=w.window,
               head_class=w.class_array(), num_pages=wmax.num_pages, free_list=wmax.free_list(), max_seqs=B,
               max_seq_len=max_len, ring_pages=w.ring_pages, max_chunk=1, ws_batch=B, ws_tokens=B * 2048, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)
    chunk = 2048
    ids = list(range(B))
    for lo in range(0, ctx, chunk):
        n = min(chunk, ctx - lo)
        k = torch.randn((B * n, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
        v = torch.randn((B * n, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
        kv.append(0, ids, [lo] * B, [n] * B, k, v)
        del k, v
    k_new = torch.randn((2 * nsteps, B, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    v_new = torch.randn((2 * nsteps, B, w.hkv, w.d), generator=gen, device=dev).to(torch.bfloat16)
    q = torch.randn((2 * nsteps, B, w.hq, w.d), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((B, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, w.hq), dtype=torch.float32, device=dev)
    n_glob = int(sum(w.classes[0]))

    def kv_bytes(p):  # algorithmic KV bytes of one decode step with the query at position p
        keys = n_glob * (p + 1) + (w.hkv - n_glob) * min(p + 1, w.window)
        return B * keys * w.d * 2 * 2

    def run(fused, s0):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        total_bytes = 0
        for i in range(nsteps):
            s = s0 + i
            p = ctx + s
            timed = i >= warm
            if timed and i == warm:
                barrier()
                torch.cuda.synchronize()
            if timed:
                ev[i - warm][0].record(stream)
            if fused:
                kv.decode_step(0, ids, k_new[s], v_new[s], q[s], out=out, lse=lse)
                if timed:
                    ev[i - warm][1].record(stream)
            else:
                kv.append(0, ids, [p] * B, [1] * B, k_new[s], v_new[s])
                if timed:
                    ev[i - warm][1].record(stream)
                kv.decode(0, ids, [p] * B, q[s], out=out, lse=lse)
            if timed:
                ev[i - warm][2].record(stream)
                total_bytes += kv_bytes(p)
        torch.cuda.synchronize()
        barrier()
        t_step = max_over_ranks(sum(e[0].elapsed_time(e[2]) for e in ev) / steps)
        t_dec = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / steps)
        return t_step, t_dec, total_bytes / steps

    t_step, _, per_step = run(True, 0)  # the fused step first, at the configured context
    t_pair, t_pair_dec, b_pair = run(False, nsteps)
    if kv.device_status() != 0:
        raise RuntimeError("device error word set during decode")
    achieved = per_step / (t_step * 1e-3) / 1e9
    res = {
        "workload": DECODE, "metric": "decode KV GB/s", "value": world * per_step / (t_step * 1e-3) / 1e9,
        "unit": "GB/s", "ms_per_step": t_step, "steps": steps, "kv_bytes_per_step": per_step,
        "step": "segkv_decode_step: the split kernel appends each sequence's token, then split-K decode + combine",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": profiled_traffic("decode_64x32k.md", DECODE_SOURCES),
                     "kernel": "decode_split_kernel<128> with the step's append + lse_combine "
                               "(events around segkv_decode_step)"},
        "two_calls": {"value": world * b_pair / (t_pair * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": t_pair,
                      "decode_ms": t_pair_dec, "step": "segkv_append (1 token) + segkv_decode_attn",
                      "gpu_launches": 3 * steps},
        "gpu_launches": 2 * steps, "data": "synthetic (seeded torch generator on the device)",
    }
    del kv
    torch.cuda.empty_cache()
    return res


if __name__ == "__main__":
    sys.exit(main())
