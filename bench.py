#!/usr/bin/env python
"""Batch-1 decode benchmark of the persistent decode kernel on B200.

Metric: decode tokens/s of one request (batch 1) on the 2.2B FP16 decoder
(26 layers, d 2560, 20 x 128 MHA, SwiGLU 6912, V 32000, untied), prompt 256,
1024 greedy tokens; plus achieved HBM GB/s of the decode kernel against the
measured B200 copy bandwidth.

One step = one 1024-token greedy decode (one persistent launch) from the same
prefilled 256-token state (the context is rewound to the prompt between
steps; the prompt's KV entries stay resident). Weights stream from HBM every
token (4.3 GB > 126 MB L2), so no L2 flush is needed between steps.

`e2e` times the user's path through the C ABI with host buffers: reset,
prefill of the prompt from host memory, and the decode into a pinned host
buffer, per step.

`--impl reference` times the fp64 CPU oracle (a bounded sample of decode
steps of the same workload) on the host cores; under torchrun only rank 0
runs it.

Multi-GPU: replicas only -- each rank decodes its own request on its own GPU;
the value is all ranks' tokens divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 decode tokens/s at 2.2B FP16; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _kernel_hash() -> str:
    """Hash of the decode kernel's code (comments and whitespace removed), so
    DRAM counters stay attached to the code they were taken on."""
    h = hashlib.sha256()
    for f in ("monokernel.cuh", "kie_internal.h"):
        with open(os.path.join(ROOT, "transformer_decode_persistent_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", " ", src).strip().encode())
    return h.hexdigest()[:16]


def _traffic_per_token(workload: str):
    """DRAM bytes per decoded token of the decode kernel from the committed ncu
    summary, or None when the kernel source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_hash") != _kernel_hash():
        return None
    return float(e["dram_bytes_per_token"])


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.f = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        self.p = None
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "200"]
            if uuid:
                cmd[1:1] = ["-i", uuid]
            self.p = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [l.split(",") for l in self.f.read().splitlines() if l.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        load = [s for s in sm if mx is None or s > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device="cuda"):
    """Element-wise maximum over all ranks (the slowest rank's times)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_value(tokens_per_rank: int, world_size: int, elapsed_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world_size / (elapsed_ms / 1000.0)


def cpu_oracle_sample(shape, weights, budget_s: float, max_steps: int):
    """Time the oracle (as it stands) decoding steps of the workload from an
    empty context; returns (tokens/s, steps, seconds, threads)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    m = O.Decoder(shape, weights, cache_f64=False)
    cache = m.new_cache(max_steps + 1)
    tok = 0
    steps, t0 = 0, time.perf_counter()
    while steps < max_steps:
        lg = m.step(tok, cache)
        tok = O.argmax_lowest(lg)
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return steps / dt, steps, dt, threads


def run_reference(args, shape):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    import synthetic as S
    weights = S.make_weights(shape, seed=0)
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    m = O.Decoder(shape, weights, cache_f64=False)
    total = args.warmup + args.steps
    cache = m.new_cache(total + 1)
    tok = int(S.make_prompt(shape, 0)[0])
    for _ in range(args.warmup):
        tok = O.argmax_lowest(m.step(tok, cache))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        tok = O.argmax_lowest(m.step(tok, cache))
    dt = time.perf_counter() - t0
    v = args.steps / dt
    sample = (f"{args.steps} timed decode steps (after {args.warmup} warm-up) of the {shape.name} "
              f"workload from an empty context; one step = one token")
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": shape.name, "prompt": shape.prompt_len, "decode": shape.decode_len,
                       "batch": 1},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


PHASE_KINDS = ("qkv", "attention", "o_proj", "gate_up", "down", "lm_head")


def summarize_phase_trace(t: np.ndarray, n_layers: int) -> dict:
    """Per-token phase times from a trace-build record array t [grid, steps *
    (5 L + 2), 4] (start, input ready, tiles done, epilogue done; the step
    barrier last in each step as arrival, release, release, release).

    Per CTA and step, each phase kind's input wait (start -> input ready),
    tile time and epilogue time are summed over the layers (attention: the
    wait for q and this token's k/v, the CTA's own units, the cross-CTA chunk
    merge); the figures are
    medians over CTAs of the per-step mean. The step time is the interval
    between consecutive barrier releases (median over CTAs); the wait share is
    the phases' input waits plus the barrier wait over the step time."""
    G, R, _ = t.shape
    rps = 5 * n_layers + 2
    steps = R // rps
    t = t[:, :steps * rps].reshape(G, steps, rps, 4).astype(np.float64)
    bar = t[:, :, rps - 1, :]
    rel = np.median(bar[:, :, 1], axis=0)
    step_us = float(np.diff(rel).mean() / 1000.0) if steps > 1 else float("nan")
    out = {"steps": int(steps), "step_us": step_us, "per_token_us": {}}
    total_wait = np.zeros((G, steps))
    for k, name in enumerate(PHASE_KINDS):
        idx = [n_layers * 5] if name == "lm_head" else [l * 5 + k for l in range(n_layers)]
        rec = t[:, :, idx, :]
        if not np.any(rec[..., 3] > 0):
            continue
        wait = (rec[..., 1] - rec[..., 0]).sum(axis=2)
        tiles = (rec[..., 2] - rec[..., 1]).sum(axis=2)
        epi = (rec[..., 3] - rec[..., 2]).sum(axis=2)
        total_wait += wait
        med = lambda a: float(np.median(a.mean(axis=1)) / 1000.0)
        out["per_token_us"][name] = {"input_wait": med(wait), "tiles": med(tiles), "epilogue": med(epi)}
    bw = bar[:, :, 1] - bar[:, :, 0]
    out["per_token_us"]["step_barrier"] = {"wait": float(np.median(bw.mean(axis=1)) / 1000.0)}
    if steps > 1:
        span = float(np.median(np.diff(bar[:, :, 1], axis=1).sum(axis=1)))
        out["flag_wait_share"] = float(np.median(total_wait[:, 1:].sum(axis=1)) / span)
        out["barrier_wait_share"] = float(np.median(bw[:, 1:].sum(axis=1)) / span)
    return out


def phase_trace(shape, weights, prompt, device: int, m: int) -> dict:
    """Run the trace build (libkie_trace.so) over the first and the last m
    steps of the workload's decode and summarize both (see
    summarize_phase_trace)."""
    import torch
    from transformer_decode_persistent_b200 import Engine
    P, n = len(prompt), shape.decode_len
    eng = Engine(shape, device=device, max_ctx=P + n, trace_build=True)
    eng.load_weights(weights)
    grid = eng.info()["grid"]
    cap = m * (5 * shape.n_layers + 2)
    res = {}
    eng.prefill(prompt)
    if n > m:
        eng.decode(n - m)
        tr = torch.zeros((grid, cap, 4), dtype=torch.int64, device=f"cuda:{device}")
        eng.decode(m, trace=tr)
        res["last"] = summarize_phase_trace(tr.cpu().numpy(), shape.n_layers)
        res["last"]["positions"] = [P - 1 + n - m, P - 2 + n]
        eng.reset()
        eng.prefill(prompt)
    tr = torch.zeros((grid, cap, 4), dtype=torch.int64, device=f"cuda:{device}")
    eng.decode(m, trace=tr)
    res["first"] = summarize_phase_trace(tr.cpu().numpy(), shape.n_layers)
    res["first"]["positions"] = [P - 1, P - 2 + m]
    eng.close()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kie", choices=["kie", "reference"])
    ap.add_argument("--workload", default="dense2b", choices=["tiny", "small", "dense2b", "moe", "long2b"])
    ap.add_argument("--decode", type=int, default=None, help="override decode length (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--trace", action="store_true",
                    help="also run the trace build over the first and last 64 steps: per-phase input wait, "
                         "tile and epilogue time per token, flag-wait share")
    args = ap.parse_args()

    import synthetic as S
    shape = {"tiny": S.TINY, "small": S.SMALL, "dense2b": S.DENSE_2B, "moe": S.MOE,
             "long2b": S.LONG_2B}[args.workload]
    if args.decode:
        shape = shape.with_(decode_len=args.decode)

    if args.impl == "reference":
        run_reference(args, shape)
        return

    import numpy as np
    import torch
    import torch.distributed as dist

    from transformer_decode_persistent_b200 import Engine

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=torch.device("cuda", local))

    P, n = shape.prompt_len, shape.decode_len
    weights = S.make_weights(shape, seed=0)
    prompt = S.make_prompt(shape, seed=0)
    eng = Engine(shape, device=local, max_ctx=P + n)
    eng.load_weights(weights)
    info = eng.info()
    eng.prefill(prompt)
    out = torch.empty(n, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        eng.rewind(P - 1, int(prompt[-1]))
        eng.decode(n, out=out)

    for _ in range(args.warmup):
        step()
    props = torch.cuda.get_device_properties(local)
    uuid = getattr(props, "uuid", None)
    uuid = f"GPU-{uuid}" if uuid is not None and not str(uuid).startswith("GPU-") else (str(uuid) if uuid else None)
    clk = Clocks(uuid)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    l0 = eng.info()["launches"]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clocks = clk.stop()
    launches = eng.info()["launches"] - l0
    elapsed_ms = t_all0.elapsed_time(t_all1)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    elapsed_ms = max_over_ranks([elapsed_ms])[0]
    tokens_total = n * args.steps * ws
    value = job_value(n * args.steps, ws, elapsed_ms)

    # roofline of the decode kernel (the only kernel in the timed region)
    kvp = info["kv_bytes_per_pos"]
    positions = np.arange(P - 1, P - 1 + n)
    alg_bytes = n * info["stream_bytes"] + kvp * int((positions + 1).sum()) + kvp * n
    avg_launch_s = statistics.mean(launch_ms) / 1000.0
    achieved = alg_bytes / avg_launch_s / 1e9
    peak, peak_kind = _peaks()
    tpt = _traffic_per_token(args.workload)

    # end to end through the C ABI with host buffers
    e2e = None
    prefill = None
    if not args.no_e2e:
        host_out = torch.empty(n, dtype=torch.int32).pin_memory()
        host_prompt = np.ascontiguousarray(prompt.astype(np.int32))
        eng.reset()
        eng.prefill(host_prompt)
        eng.decode(n, out=host_out)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.perf_counter()
        a.record(stream)
        for _ in range(args.steps):
            eng.reset()
            eng.prefill(host_prompt)
            eng.decode(n, out=host_out)
        b.record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - w0
        e_ms = max_over_ranks([max(a.elapsed_time(b), wall * 1000.0)])[0]
        e2e = {"value": job_value(n * args.steps, ws, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(host_prompt.nbytes), "d2h_bytes_per_step": int(n * 4),
               "includes": f"reset + prefill of the {P}-token prompt from host memory + decode into pinned host memory"}
        # the prompt path alone (the tensor-core prefill)
        pms = []
        for _ in range(max(1, args.steps)):
            eng.reset()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            eng.prefill(host_prompt)
            b.record(stream)
            torch.cuda.synchronize()
            pms.append(a.elapsed_time(b))
        prefill = {"prompt_tokens": P, "ms": min(pms), "tokens_per_s": (P - 1) / (min(pms) / 1000.0),
                   "path": "tensor cores"}

    stall = None
    if args.trace and rank == 0:
        stall = phase_trace(shape, weights, prompt, local, min(n, 64))

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, steps, dt, threads = cpu_oracle_sample(shape, weights, budget_s=20.0, max_steps=6)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{steps} oracle decode steps (positions 0-{steps - 1}) of the {shape.name} workload "
                         f"from an empty context on {threads} BLAS threads ({dt:.1f} s; the per-token cost is "
                         f"the weight GEMVs, attention over <= {P + n} positions adds < 1%)"}

    eng.close()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": shape.name, "prompt": P, "decode": n, "batch": 1,
                       "parallelism": f"replicas{ws}" if ws > 1 else "single-gpu",
                       "l2": "no flush: 4.3 GB of weights (> 126 MB L2) stream from HBM every token",
                       "weights": "fp16 N(0,0.02) seeded synthetic; fp32 activations and accumulation",
                       "us_per_token": 1e6 * (elapsed_ms / 1000.0) / (n * args.steps)},
            "gpu_launches": int(launches),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": f"{peak_kind} copy bandwidth (hbm_gbs)",
                         "traffic": (tpt * n) if tpt else None,
                         "algorithmic_bytes_per_launch": int(alg_bytes),
                         "kernel": "kie::decode_kernel", "avg_launch_ms": 1000 * avg_launch_s,
                         "frac_of_8TBps_spec": achieved / 8000.0},
            "clocks": clocks,
            "e2e": e2e,
            "prefill": prefill,
            "cpu_baseline": cpu,
        }
        if stall is not None:
            line["trace"] = stall
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
