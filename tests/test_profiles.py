"""The committed profiler summaries that bench.py reads its roofline traffic from: each names an
existing kernel source, a 64-digit source hash and, where it gives one, an integer byte count; the
traffic bench.py reports is that count exactly when the hash matches the source as it is."""
import hashlib
import importlib.util
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fields(path):
    out = {}
    for line in open(path):
        if ":" in line and not line.startswith(("|", " ", "#")):
            k, v = line.split(":", 1)
            out[k.strip()] = v.strip()
    return out


def _summaries():
    d = os.path.join(ROOT, "profiles")
    return sorted(os.path.join(d, f) for f in os.listdir(d) if f.endswith(".md"))


def test_profiles_are_text_summaries():
    for p in os.listdir(os.path.join(ROOT, "profiles")):
        assert p.endswith((".md", ".txt")), p          # no raw reports in the repository
        assert os.path.getsize(os.path.join(ROOT, "profiles", p)) < 64 * 1024, p


@pytest.mark.parametrize("path", _summaries(), ids=os.path.basename)
def test_summary_fields(path):
    f = _fields(path)
    text = open(path).read()
    assert "ncu" in text and "--clock-control none" in text, "the command that made it"
    if "kernel_source" not in f:
        return
    assert os.path.isfile(os.path.join(ROOT, f["kernel_source"])), f["kernel_source"]
    if "source_sha256" in f or "traffic_bytes_per_launch" in f:   # a capture of one kernel version
        assert re.fullmatch(r"[0-9a-f]{64}", f.get("source_sha256", "")), "source hash"
    if "traffic_bytes_per_launch" in f:
        assert int(f["traffic_bytes_per_launch"]) > 0


def test_bench_reads_traffic_only_for_the_source_captured():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    for path in _summaries():
        name = os.path.basename(path)[:-3]
        m = re.fullmatch(r"(attention_tc_kernel|attention_bwd_kernel|candidate_attention)_(\w+)", name)
        if not m:
            continue
        f = _fields(path)
        src = open(os.path.join(ROOT, f["kernel_source"]), "rb").read()
        current = hashlib.sha256(src).hexdigest() == f["source_sha256"]
        got = bench.profiled_traffic(m.group(2), m.group(1))
        assert got == (int(f["traffic_bytes_per_launch"]) if current else None), name
