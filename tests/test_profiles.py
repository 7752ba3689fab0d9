"""The ncu summaries bench.py reads its DRAM-traffic figures from (CPU only): every summary it
names exists, gives the command that made it, and was taken on the kernel sources as they are
now (the summary records their hash; bench.py reports no traffic for a stale one)."""
import importlib.util
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def summaries_read_by_bench():
    text = open(os.path.join(ROOT, "bench.py")).read()
    return sorted(set(re.findall(r'profiled_traffic\("([^"]+)", ([A-Z_]+)\)', text)))


def test_bench_reads_traffic_from_several_summaries():
    assert len(summaries_read_by_bench()) >= 8


@pytest.mark.parametrize("name,sources", summaries_read_by_bench())
def test_summary_matches_current_kernel_sources(name, sources):
    bench = load_bench()
    path = os.path.join(ROOT, "profiles", name)
    assert os.path.exists(path), name
    text = open(path).read()
    assert "--clock-control none" in text and "python bench.py" in text, "the capture command is recorded"
    traffic = bench.profiled_traffic(name, getattr(bench, sources))
    assert traffic is not None and traffic > 0, f"{name}: hash does not match {sources} or no DRAM bytes"
