"""Host-side pieces of bench.py that need no GPU: the kernel-code hash that
keys the committed DRAM counters, and the lookup of those counters."""
import json
import os
import shutil

import numpy as np

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
    for f in ("monokernel.cuh", "kie_internal.h"):
        shutil.copy(os.path.join(ROOT, CSRC, f), tmp_path / CSRC / f)
    os.makedirs(tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return bench, tmp_path


def test_kernel_hash_ignores_comments_and_whitespace(bench_in):
    bench, root = bench_in
    h0 = bench._kernel_hash()
    p = root / CSRC / "monokernel.cuh"
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



def test_phase_trace_summary_on_synthetic_records():
    # Two layers, three steps: every phase waits 1 us for its input, runs 2 us
    # of tiles and 0.5 us of epilogue (the LM head 3 us of tiles); the step
    # barrier waits 4 us. Step time = 6 phases * 3.5 us + 2.5 + 0.5 extra
    # for the LM head + 4 us barrier.
    import bench
    L, G, steps = 2, 3, 3
    rps = 5 * L + 2
    t = np.zeros((G, steps * rps, 4), dtype=np.int64)
    now = 0
    for st in range(steps):
        for ph in range(5 * L + 1):
            tiles = 3000 if ph == 5 * L else 2000
            rec = t[:, st * rps + ph]
            rec[:, 0] = now
            rec[:, 1] = now + 1000
            rec[:, 2] = now + 1000 + tiles
            rec[:, 3] = now + 1500 + tiles
            now += 1500 + tiles
        t[:, st * rps + rps - 1] = [now, now + 4000, now + 4000, now + 4000]
        now += 4000
    out = bench.summarize_phase_trace(t, L)
    step_us = (10 * 3.5 + 4.5 + 4.0)
    assert out["steps"] == steps and abs(out["step_us"] - step_us) < 1e-9
    p = out["per_token_us"]
    assert p["qkv"] == {"input_wait": 2.0, "tiles": 4.0, "epilogue": 1.0}
    assert p["lm_head"] == {"input_wait": 1.0, "tiles": 3.0, "epilogue": 0.5}
    assert p["step_barrier"]["wait"] == 4.0
    assert abs(out["flag_wait_share"] - 11.0 / step_us) < 1e-12
    assert abs(out["barrier_wait_share"] - 4.0 / step_us) < 1e-12
