"""Host-side pieces of bench.py that need no GPU: the kernel-code hash that
keys the committed DRAM counters, and the lookup of those counters."""
import json
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join("transformer_decode_persistent_b200", "csrc")


@pytest.fixture()
def bench_in(tmp_path, monkeypatch):
    """bench.py pointed at a private copy of the kernel sources and profiles."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.makedirs(tmp_path / CSRC)
    for f in ("monokernel.cu", "kie_internal.h"):
        shutil.copy(os.path.join(ROOT, CSRC, f), tmp_path / CSRC / f)
    os.makedirs(tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return bench, tmp_path


def test_kernel_hash_ignores_comments_and_whitespace(bench_in):
    bench, root = bench_in
    h0 = bench._kernel_hash()
    p = root / CSRC / "monokernel.cu"
    src = p.read_text()
    p.write_text("// a new comment line\n/* and a\n block */\n" + src.replace("\n", "\n\n"))
    assert bench._kernel_hash() == h0


def test_kernel_hash_follows_code_changes(bench_in):
    bench, root = bench_in
    h0 = bench._kernel_hash()
    p = root / CSRC / "kie_internal.h"
    p.write_text(p.read_text().replace("kPartFloats = ", "kPartFloats = 1 + "))
    assert bench._kernel_hash() != h0


def test_traffic_lookup_needs_matching_code(bench_in):
    bench, root = bench_in
    tj = root / "profiles" / "traffic.json"
    assert bench._traffic_per_token("dense2b") is None  # no counters yet
    tj.write_text(json.dumps({"dense2b": {"dram_bytes_per_token": 4.25e9,
                                          "kernel_hash": bench._kernel_hash()}}))
    assert bench._traffic_per_token("dense2b") == pytest.approx(4.25e9)
    assert bench._traffic_per_token("moe") is None  # no entry for that workload
    tj.write_text(json.dumps({"dense2b": {"dram_bytes_per_token": 4.25e9, "kernel_hash": "0" * 16}}))
    assert bench._traffic_per_token("dense2b") is None  # counters of other code

