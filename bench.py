#!/usr/bin/env python
"""Benchmark of the MoBA causal prefill forward on B200.

Workload (one step = one whole forward: pooling, gating + top-k, selection
inversion, block-sparse attention, log-sum-exp merge): the Llama-3.1-8B
attention shape at one million tokens, B=1, Hq=32, Hkv=8, d=128,
N=1048576, block_size=4096, topk=12, bf16, seeded synthetic inputs with the
pages' distribution (Q, V ~ N(0,1); K = N(0,1) + a per key-block offset
N(0, 0.5^2)), seed 3.

Metric: useful TFLOP/s (4 d FLOPs per attended query/key pair) and ms per
forward; the JSON line also carries the fraction of the bf16 tensor-core peak,
the speedup over dense causal attention on the same GPU, the end-to-end number
through host buffers, the attention kernel's roofline and the CPU oracle
baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl moba|reference]

With N > 1 (one process per GPU under torch.distributed.run) every rank runs
its own independent forward of the same shape (weak scaling; the method has no
exchange step between sequences). `--impl reference` times the fp64 CPU oracle
on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = {"B": 1, "Hq": 32, "Hkv": 8, "d": 128, "N": 1 << 20, "block_size": 4096, "topk": 12, "seed": 3}
WORKLOAD_NAME = ("Llama-3.1-8B attention shape at 1M tokens: B=1, Hq=32, Hkv=8, d=128, N=1048576, "
                 "block_size=4096, topk=12, causal, bf16, seed 3")
METRIC = "MoBA prefill fwd useful TFLOP/s @1M tokens"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SRC = [os.path.join(ROOT, "block_sparse_long_gate_b200", "csrc", f)
            for f in ("k_attn_tc.cuh", "k_attn_common.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.json")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=("moba", "reference"), default="moba")
    p.add_argument("--seq-len", type=int, default=WORKLOAD["N"], help="override N (diagnostic runs only)")
    p.add_argument("--hq", type=int, default=None, help="override Hq (diagnostic runs only)")
    p.add_argument("--hkv", type=int, default=None, help="override Hkv (diagnostic runs only)")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--sample-rows", type=int, default=1024, help="oracle rows per CPU sample")
    return p.parse_args(argv)


# ---------------------------------------------------------------- helpers shared with the tests
def workload(seq_len: int | None = None, hq: int | None = None, hkv: int | None = None) -> dict:
    w = dict(WORKLOAD)
    if seq_len:
        w["N"] = int(seq_len)
    if hq:
        w["Hq"] = int(hq)
    if hkv:
        w["Hkv"] = int(hkv)
    return w


def workload_name(w: dict) -> str:
    if all(w[k] == WORKLOAD[k] for k in ("N", "Hq", "Hkv")):
        return WORKLOAD_NAME
    return f"{WORKLOAD_NAME} (diagnostic override: N={w['N']}, Hq={w['Hq']}, Hkv={w['Hkv']})"


def useful_flops(w: dict) -> float:
    from block_sparse_long_gate_b200 import flops
    return flops.useful_flops(w["B"], w["Hq"], w["N"], w["d"], w["block_size"], w["topk"])


def aggregate(local_ms: float, local_units: float, world: int) -> tuple[float, float]:
    """(max elapsed ms over ranks, total units over ranks) through torch.distributed when world > 1."""
    if world <= 1:
        return local_ms, local_units
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    u = torch.tensor([local_units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def sample_rows(w: dict, n_rows: int, seed: int):
    """Seeded rows (b, hq, t) spread over every head and the whole sequence."""
    import numpy as np
    rng = np.random.default_rng(seed)
    per = max(1, n_rows // (w["B"] * w["Hq"]))
    rows = []
    for b in range(w["B"]):
        for h in range(w["Hq"]):
            ts = np.sort(rng.integers(0, w["N"], size=per))
            rows += [(b, h, int(t)) for t in ts]
    return np.array(rows, dtype=np.int64)


def rows_useful_flops(w: dict, rows) -> float:
    """4 d times the number of keys the sampled rows attend."""
    bs, kp = w["block_size"], w["topk"] - 1
    n = 0
    for _, _, t in rows:
        c = int(t) // bs
        n += min(c, kp) * bs + (int(t) - c * bs + 1)
    return 4.0 * w["d"] * n


def read_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def attention_traffic() -> float | None:
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, or None when
    the kernel source changed since those counters were taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for path in ATTN_SRC:
            with open(path, "rb") as f:
                h.update(f.read())
        digest = h.hexdigest()
        if rec.get("source_sha256") != digest:
            return None
        return float(rec["bytes_per_full_launch"])
    except (OSError, ValueError, KeyError):
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self) -> dict:
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        sm, mx, reasons = [], [], set()
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                s, m, pw = float(parts[0]), float(parts[1]), float(parts[2])
            except ValueError:
                continue
            if pw < 200.0:  # idle sample (before the first or after the last launch)
                continue
            sm.append(s)
            mx.append(m)
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle baseline
def oracle_sample(q, k, v, w: dict, n_rows: int, seed: int) -> tuple[float, float, int]:
    """Time the oracle on a row sample: (seconds, useful FLOPs of the sample, rows)."""
    import oracle
    rows = sample_rows(w, n_rows, seed)
    t0 = time.perf_counter()
    oracle.forward(q, k, v, w["block_size"], w["topk"], rows)
    dt = time.perf_counter() - t0
    return dt, rows_useful_flops(w, rows), len(rows)


def host_inputs(w: dict, seed: int, pin: bool):
    import synth
    return synth.inputs(w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], w["block_size"], seed, pin=pin)


def cpu_cores() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


# ---------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(args.seq_len, args.hq, args.hkv)
    q, k, v = host_inputs(w, w["seed"], pin=False)
    for i in range(args.warmup):
        oracle_sample(q, k, v, w, args.sample_rows, 1000 + i)
    secs, fl = 0.0, 0.0
    for i in range(args.steps):
        dt, f, nrows = oracle_sample(q, k, v, w, args.sample_rows, 2000 + i)
        secs += dt
        fl += f
    value = fl / secs / 1e12
    sample = (f"{nrows} seeded rows per step spread over all {w['B'] * w['Hq']} heads and the whole sequence; "
              f"each step pools all of K, then gates and attends the sampled rows in fp64")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(w),
                   "global_batch": w["B"], "seq_len": w["N"], "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def run_moba(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)

    from block_sparse_long_gate_b200.build import build_library
    if rank == 0:
        build_library()
    if dist:
        dist.barrier()
    import block_sparse_long_gate_b200 as moba

    moba.lib()
    w = workload(args.seq_len, args.hq, args.hkv)
    B, N, Hq, Hkv, d, bs, topk = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], w["block_size"], w["topk"]
    seed = w["seed"] + rank

    q_h, k_h, v_h = host_inputs(w, seed, pin=True)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    ws = torch.empty(moba.workspace_size(B, Hq, Hkv, N, d, bs, topk), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        moba.forward(q, k, v, bs, topk, out=out, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if moba.sync_status() != 0:
        raise SystemExit("device error during warm-up")

    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local_rank)
    moba.stage_timing(True)
    launches0 = moba.launch_count()
    with ClockSampler(gpu_id) as clk:
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
    launches = moba.launch_count() - launches0
    stages, calls = moba.stage_times()
    moba.stage_timing(False)
    status = moba.sync_status()
    local_ms = e0.elapsed_time(e1)
    fl = useful_flops(w)
    total_ms, total_flops = aggregate(local_ms, fl * args.steps, world)
    value = total_flops / (total_ms * 1e-3) / 1e12
    ms_per_step = total_ms / args.steps

    # end to end through host buffers: H2D of q, k, v and D2H of out, lse inside the timed region
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

    def e2e_step():
        q.copy_(q_h, non_blocking=True)
        k.copy_(k_h, non_blocking=True)
        v.copy_(v_h, non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    h2d = (q.numel() + k.numel() + v.numel()) * 2
    d2h = out.numel() * 2 + lse.numel() * 4
    e2e = None
    if args.e2e_steps > 0:
        e2e_step()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms, e2e_flops = aggregate(e0.elapsed_time(e1), fl * args.e2e_steps, world)
        e2e = {"value": e2e_flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}

    # dense causal attention of the same shape on the same GPU (our tcgen05 kernel), once
    dense = None
    if not args.no_dense and rank == 0:
        del ws
        torch.cuda.empty_cache()
        dout, dlse = torch.empty_like(q), torch.empty_like(lse)
        moba.dense_causal(q[:, :4096].contiguous(), k[:, :4096].contiguous(), v[:, :4096].contiguous())
        torch.cuda.synchronize()
        e0.record(stream)
        moba.dense_causal(q, k, v, out=dout, lse=dlse)
        e1.record(stream)
        torch.cuda.synchronize()
        from block_sparse_long_gate_b200 import flops as fx
        dms = e0.elapsed_time(e1)
        dense = {"ms": dms, "tflops": fx.dense_causal_flops(B, Hq, N, d) / dms / 1e9, "kernel": "moba_dense_causal"}
        del dout, dlse
        if moba.sync_status() != 0:
            dense["status"] = "device error"

    peaks, peak_src = read_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    attn_ms = stages["attention"] / max(calls, 1)
    achieved = fl / (attn_ms * 1e-3) / 1e12
    traffic = attention_traffic()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        del q, k, v
        torch.cuda.empty_cache()
        secs, sfl, nrows = oracle_sample(q_h, k_h, v_h, w, args.sample_rows, 77)
        cpu = {"value": sfl / secs / 1e12, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
               "sample": f"{nrows} seeded rows over all heads and the whole sequence (pool of all of K, then "
                         f"gate + attend of the sampled rows, fp64), {secs:.1f} s"}

    if rank == 0:
        clocks = clk.summary()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_name(w),
                       "global_batch": B * world, "seq_len": N,
                       "parallelism": f"{world} independent forward(s), one per GPU, no collective",
                       "l2": "inputs (12 GiB) far exceed the 126 MB L2; no flush between steps"},
            "pct_of_peak": 100.0 * value / world / peak,
            "peak_tflops": peak, "peak_source": f"bf16_tflops_sustained of {peak_src}",
            "stages_ms_per_step": {s: t / max(calls, 1) for s, t in stages.items()},
            "roofline": {"kernel": "moba_attn_tc_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"bf16_tflops_sustained, {peak_src}"},
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
            "device_status": status,
        }
        if dense:
            line["dense"] = dense
            line["speedup_vs_dense"] = dense["ms"] / ms_per_step
        line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_moba(args)


if __name__ == "__main__":
    sys.exit(main())
