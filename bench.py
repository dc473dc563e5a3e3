#!/usr/bin/env python
"""Benchmark of the MoBA causal prefill forward on B200.

Workload (one step = one whole forward: pooling, gating + top-k, selection
inversion, block-sparse attention, log-sum-exp merge), by default the
Llama-3.1-8B attention shape at one million tokens: B=1, Hq=32, Hkv=8, d=128,
N=1048576, block_size=4096, topk=12, bf16, seeded synthetic inputs with the
pages' distribution (Q, V ~ N(0,1); K = N(0,1) + a per key-block offset
N(0, 0.5^2)), seed 3. `--config` selects the other workloads of the same
family (0: tiny single head, 1: single head at 32K, 2: fine-granularity GQA,
3: the Llama shape, with `--seq-len` for 128K / 512K, 4: 10M tokens, one head).

Metric: useful TFLOP/s (4 d FLOPs per attended query/key pair) and ms per
forward; the JSON line also carries the fraction of the bf16 tensor-core peak,
the speedup over dense causal attention on the same GPU (this library's dense
kernel and torch's scaled_dot_product_attention, the faster of the two), the
end-to-end number through host buffers, the attention kernel's roofline and the
CPU oracle baseline.

  python bench.py [--config C] [--gpus N] [--steps K] [--warmup W] [--impl moba|reference]

With N > 1 (one process per GPU under torch.distributed.run) one forward is split
by kv-head groups: rank r owns a contiguous range of kv heads and their query
heads, and runs the single-GPU forward on its slices with no exchange between
ranks (total work fixed: strong scaling). Workloads with fewer kv heads than
ranks run one independent forward per rank instead (weak scaling).
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores.
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

CONFIGS = {
    0: {"B": 1, "Hq": 1, "Hkv": 1, "d": 128, "N": 4096, "block_size": 512, "topk": 3, "seed": 0},
    1: {"B": 1, "Hq": 1, "Hkv": 1, "d": 128, "N": 32768, "block_size": 2048, "topk": 3, "seed": 1},
    2: {"B": 2, "Hq": 32, "Hkv": 8, "d": 128, "N": 32768, "block_size": 256, "topk": 32, "seed": 2},
    3: {"B": 1, "Hq": 32, "Hkv": 8, "d": 128, "N": 1 << 20, "block_size": 4096, "topk": 12, "seed": 3},
    4: {"B": 1, "Hq": 1, "Hkv": 1, "d": 128, "N": 10485760, "block_size": 4096, "topk": 12, "seed": 4},
}
CONFIG_NAMES = {
    0: "Tiny reference",
    1: "Single-head long sequence",
    2: "Fine-granularity GQA",
    3: "Llama-3.1-8B attention shape at long context",
    4: "Extreme length (10M tokens, one head)",
}
DEFAULT_CONFIG = 3
WORKLOAD = CONFIGS[DEFAULT_CONFIG]
WORKLOAD_NAME = ("Llama-3.1-8B attention shape at 1M tokens: B=1, Hq=32, Hkv=8, d=128, N=1048576, "
                 "block_size=4096, topk=12, causal, bf16, seed 3")
METRIC = "MoBA prefill fwd useful TFLOP/s @1M tokens"
UNIT = "TFLOP/s"
SPEC_BF16_TFLOPS = 2250.0  # nominal dense bf16 tensor-core peak of one B200, for context
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SRC = [os.path.join(ROOT, "block_sparse_long_gate_b200", "csrc", f)
            for f in ("k_attn_tc.cuh", "k_attn_common.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.json")
L2_FLUSH_BELOW = 512 << 20  # inputs smaller than this get an L2 flush between timed steps


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--config", type=int, choices=sorted(CONFIGS), default=DEFAULT_CONFIG)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=("moba", "reference"), default="moba")
    p.add_argument("--seq-len", type=int, default=None,
                   help="override N (config 3: 131072 / 524288 / 1048576; other values are diagnostic)")
    p.add_argument("--hq", type=int, default=None, help="override Hq (diagnostic runs only)")
    p.add_argument("--hkv", type=int, default=None, help="override Hkv (diagnostic runs only)")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-sdpa", action="store_true", help="skip torch's dense attention in the dense arm")
    p.add_argument("--mode", choices=("prefill", "decode", "backward"), default="prefill",
                   help="decode: one new query per sequence against a KV cache of the workload's length; "
                        "backward: dq, dk, dv of the workload's forward")
    p.add_argument("--pooling", choices=("mean", "max", "weighted"), default="mean",
                   help="the gate's block summary (weighted: weights rising linearly from 0.5 to 1.5 across a block)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--sample-rows", type=int, default=1024, help="oracle rows per CPU sample")
    return p.parse_args(argv)


# ---------------------------------------------------------------- helpers shared with the tests
def workload(seq_len: int | None = None, hq: int | None = None, hkv: int | None = None,
             config: int = DEFAULT_CONFIG) -> dict:
    w = dict(CONFIGS[config])
    w["config"] = config
    if seq_len:
        w["N"] = int(seq_len)
    if hq:
        w["Hq"] = int(hq)
    if hkv:
        w["Hkv"] = int(hkv)
    return w


def workload_name(w: dict) -> str:
    cfg = w.get("config", DEFAULT_CONFIG)
    base = CONFIGS[cfg]
    pooling = w.get("pooling", "mean")
    suffix = "" if pooling == "mean" else f", {pooling} pooling" + (
        " (weights 0.5..1.5 across a block)" if pooling == "weighted" else "")
    if cfg == DEFAULT_CONFIG and all(w[k] == WORKLOAD[k] for k in ("N", "Hq", "Hkv")):
        return WORKLOAD_NAME + suffix
    name = (f"{CONFIG_NAMES[cfg]}: B={w['B']}, Hq={w['Hq']}, Hkv={w['Hkv']}, d={w['d']}, N={w['N']}, "
            f"block_size={w['block_size']}, topk={w['topk']}, causal, bf16, seed {w['seed']}")
    if any(w[k] != base[k] for k in ("Hq", "Hkv")) or (w["N"] != base["N"] and not (
            cfg == 3 and w["N"] in (131072, 524288))):
        name += " (diagnostic override)"
    return name + suffix


def pool_weights_host(w: dict):
    """The weighted-pooling recipe of the bench: one weight per position inside a block, rising
    linearly from 0.5 (first key) to 1.5 (last key), as fp32."""
    import numpy as np
    return np.linspace(0.5, 1.5, w["block_size"]).astype(np.float32)


def metric_name(w: dict) -> str:
    if w.get("config", DEFAULT_CONFIG) == DEFAULT_CONFIG and w["N"] == WORKLOAD["N"]:
        return METRIC
    return f"MoBA prefill fwd useful TFLOP/s @{w['N']} tokens"


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
    """Time the oracle on a row sample (every row when the workload has no more than n_rows):
    (seconds, useful FLOPs of the sample, rows)."""
    import oracle
    total = w["B"] * w["Hq"] * w["N"]
    rows = oracle.all_rows(w["B"], w["Hq"], w["N"]) if total <= n_rows else sample_rows(w, n_rows, seed)
    pooling = w.get("pooling", "mean")
    pw = pool_weights_host(w).astype("float64") if pooling == "weighted" else None
    t0 = time.perf_counter()
    oracle.forward(q, k, v, w["block_size"], w["topk"], rows, pooling=pooling, weights=pw)
    dt = time.perf_counter() - t0
    return dt, rows_useful_flops(w, rows), len(rows)


def sample_text(w: dict, nrows: int) -> str:
    total = w["B"] * w["Hq"] * w["N"]
    if nrows >= total:
        return f"all {total} rows of the workload per step (pool, gate and attention in fp64)"
    return (f"{nrows} seeded rows per step spread over all {w['B'] * w['Hq']} heads and the whole sequence; "
            f"each step pools all of K, then gates and attends the sampled rows in fp64")


def host_inputs(w: dict, seed: int, pin: bool, hkv_range=None):
    import synth
    if hkv_range is None:
        return synth.inputs(w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], w["block_size"], seed, pin=pin)
    return synth.inputs_heads(w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], w["block_size"], seed,
                              hkv_range[0], hkv_range[1], pin=pin)


def cpu_cores() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


def peak_fields(value_per_gpu: float, clocks: dict, peaks: dict, peak_src: str) -> dict:
    """Fractions of the bf16 tensor-core peak: the measured burst cuBLAS figure (headline),
    the measured sustained one, the nominal spec, and the burst fraction at the SM clock
    the run saw scaled to the maximum clock (so the power cap's share is visible)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    out = {
        "pct_of_peak": 100.0 * value_per_gpu / burst,
        "peak_tflops": burst,
        "peak_source": f"bf16_tflops (burst cuBLAS bf16 GEMM) of {peak_src}",
        "pct_of_sustained_peak": 100.0 * value_per_gpu / sust,
        "sustained_peak_tflops": sust,
        "pct_of_spec_peak": 100.0 * value_per_gpu / SPEC_BF16_TFLOPS,
        "spec_peak_tflops": SPEC_BF16_TFLOPS,
    }
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm and mx:
        out["clock_normalised_tflops"] = value_per_gpu * mx / sm
        out["pct_of_peak_at_max_clock"] = 100.0 * value_per_gpu * mx / sm / burst
    return out


# ---------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(args.seq_len, args.hq, args.hkv, args.config)
    w["pooling"] = args.pooling
    q, k, v = host_inputs(w, w["seed"], pin=False)
    for i in range(args.warmup):
        oracle_sample(q, k, v, w, args.sample_rows, 1000 + i)
    secs, fl = 0.0, 0.0
    nrows = 0
    for i in range(args.steps):
        dt, f, nrows = oracle_sample(q, k, v, w, args.sample_rows, 2000 + i)
        secs += dt
        fl += f
    value = fl / secs / 1e12
    line = {
        "impl": "reference", "metric": metric_name(w), "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(w),
                   "global_batch": w["B"], "seq_len": w["N"], "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample_text(w, nrows)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- dense comparison
def time_sdpa(q, k, v, stream) -> dict:
    """torch's scaled_dot_product_attention, causal, with its fused backends only (no math
    fallback, which would materialise N x N): grouped-query heads through enable_gqa, or with
    the kv heads repeated (outside the timed region) when no fused backend takes enable_gqa."""
    import torch
    from torch.nn.attention import SDPBackend, sdpa_kernel
    F = torch.nn.functional
    backends = [SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION]
    G = q.shape[2] // k.shape[2]
    qt, kt, vt = q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    def attempt(kk, vv, gqa):
        with sdpa_kernel(backends):
            # warm up at the timed shape: a backend may build its plan for a new shape on the first call
            F.scaled_dot_product_attention(qt, kk, vv, is_causal=True, enable_gqa=gqa)
            torch.cuda.synchronize()
            e0.record(stream)
            o = F.scaled_dot_product_attention(qt, kk, vv, is_causal=True, enable_gqa=gqa)
            e1.record(stream)
            torch.cuda.synchronize()
        del o
        return e0.elapsed_time(e1)

    try:
        return {"ms": attempt(kt, vt, G > 1), "kernel": "torch sdpa" + (" (enable_gqa)" if G > 1 else "")}
    except RuntimeError as exc:
        if G == 1:
            return {"error": str(exc).splitlines()[0][:200]}
        first = str(exc).splitlines()[0][:120]
    torch.cuda.empty_cache()
    try:
        kr = kt.repeat_interleave(G, dim=1)
        vr = vt.repeat_interleave(G, dim=1)
        ms = attempt(kr, vr, False)
        del kr, vr
        return {"ms": ms, "kernel": "torch sdpa (kv heads repeated)", "enable_gqa_error": first}
    except RuntimeError as exc:
        return {"error": str(exc).splitlines()[0][:200]}


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
    from block_sparse_long_gate_b200 import flops as fx
    from block_sparse_long_gate_b200 import partition

    moba.lib()
    w = workload(args.seq_len, args.hq, args.hkv, args.config)
    w["pooling"] = args.pooling
    B, N, Hq, Hkv, d, bs, topk = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], w["block_size"], w["topk"]
    split = world > 1 and partition.can_split(Hq, Hkv, world)
    if split:  # one forward, split by kv-head groups
        sl = partition.head_slices(Hq, Hkv, world)[rank]
        hq_r, hkv_r, seed = sl.n_q, sl.n_kv, w["seed"]
        q_h, k_h, v_h = host_inputs(w, seed, pin=True, hkv_range=(sl.hkv0, sl.hkv1))
        parallelism = (f"one forward split over {world} GPUs by kv-head groups (rank {rank}: kv heads "
                       f"[{sl.hkv0}, {sl.hkv1}) and their query heads), no collective on the data path")
        scaling = "strong"
    else:  # independent forwards (world 1, or fewer kv heads than ranks)
        hq_r, hkv_r, seed = Hq, Hkv, w["seed"] + rank
        q_h, k_h, v_h = host_inputs(w, seed, pin=True)
        parallelism = ("single GPU" if world == 1 else
                       f"{world} independent forwards, one per GPU (seed + rank), no collective")
        scaling = "weak"
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, hq_r, N), dtype=torch.float32, device=dev)
    ws = torch.empty(moba.workspace_size(B, hq_r, hkv_r, N, d, bs, topk), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    in_bytes = (q.numel() + k.numel() + v.numel()) * 2
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < L2_FLUSH_BELOW else None

    pw = torch.from_numpy(pool_weights_host(w)).to(dev) if args.pooling == "weighted" else None

    def step():
        moba.forward(q, k, v, bs, topk, out=out, lse=lse, workspace=ws, pooling=args.pooling, pool_weights=pw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if moba.sync_status() != 0:
        raise SystemExit("device error during warm-up")

    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local_rank)
    moba.stage_timing(True)
    launches0 = moba.launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(gpu_id) as clk:
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        if flush is None:
            ev[0][0].record(stream)
            for _ in range(args.steps):
                step()
            ev[0][1].record(stream)
        else:  # small inputs: rewrite a 256 MB buffer (twice the L2) between timed steps
            for a, b in ev:
                flush.fill_(1)
                a.record(stream)
                step()
                b.record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
    launches = moba.launch_count() - launches0
    stages, calls = moba.stage_times()
    moba.stage_timing(False)
    status = moba.sync_status()
    local_ms = ev[0][0].elapsed_time(ev[0][1]) if flush is None else sum(a.elapsed_time(b) for a, b in ev)
    fl_local = fx.useful_flops(B, hq_r, N, d, bs, topk)
    total_ms, total_flops = aggregate(local_ms, fl_local * args.steps, world)
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

    h2d = in_bytes
    d2h = out.numel() * 2 + lse.numel() * 4
    e2e = None
    if args.e2e_steps > 0:
        e2e_step()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0, e1 = ev[0]
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms, e2e_flops = aggregate(e0.elapsed_time(e1), fl_local * args.e2e_steps, world)
        e2e = {"value": e2e_flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps, "ms_per_step": e2e_ms / args.e2e_steps}

    # dense causal attention of the same shape on the same GPU: this library's tcgen05 kernel and
    # torch's fused attention, each once (the whole shape, on rank 0 only)
    dense = None
    if not args.no_dense and rank == 0 and not split:
        del ws
        torch.cuda.empty_cache()
        dout, dlse = torch.empty_like(q), torch.empty_like(lse)
        moba.dense_causal(q[:, :4096].contiguous(), k[:, :4096].contiguous(), v[:, :4096].contiguous())
        torch.cuda.synchronize()
        e0, e1 = ev[0]
        if flush is not None:
            flush.fill_(1)
        e0.record(stream)
        moba.dense_causal(q, k, v, out=dout, lse=dlse)
        e1.record(stream)
        torch.cuda.synchronize()
        dms = e0.elapsed_time(e1)
        dflops = fx.dense_causal_flops(B, Hq, N, d)
        dense = {"moba_dense_causal": {"ms": dms, "tflops": dflops / dms / 1e9}}
        if moba.sync_status() != 0:
            dense["moba_dense_causal"]["status"] = "device error"
        del dout, dlse
        torch.cuda.empty_cache()
        if not args.no_sdpa:
            sd = time_sdpa(q, k, v, stream)
            if "ms" in sd:
                sd["tflops"] = dflops / sd["ms"] / 1e9
            dense["torch_sdpa"] = sd
        best = min((x for x in dense.values() if "ms" in x), key=lambda x: x["ms"])
        dense["fastest"] = [n for n, x in dense.items() if x is best][0]
        dense["ms"] = best["ms"]

    peaks, peak_src = read_peaks()
    sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    attn_ms = stages["attention"] / max(calls, 1)
    achieved = fl_local / (attn_ms * 1e-3) / 1e12
    traffic = attention_traffic() if (w["config"] == DEFAULT_CONFIG and N == WORKLOAD["N"]
                                      and Hq == WORKLOAD["Hq"] and not split) else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        del q, k, v
        torch.cuda.empty_cache()
        secs, sfl, nrows = oracle_sample(q_h, k_h, v_h, w, args.sample_rows, 77)
        cpu = {"value": sfl / secs / 1e12, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
               "sample": sample_text(w, nrows) + f", {secs:.1f} s"}

    if rank == 0:
        clocks = clk.summary()
        line = {
            "metric": metric_name(w), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": scaling,
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_name(w),
                       "global_batch": B * (1 if split else world), "seq_len": N, "parallelism": parallelism,
                       "l2": ("inputs far exceed the 126 MB L2; no flush between steps" if flush is None else
                              "a 256 MB buffer is rewritten before every timed step (L2 flush), "
                              "steps timed one by one")},
        }
        line.update(peak_fields(value / world, clocks, peaks, peak_src))
        line.update({
            "stages_ms_per_step": {s: t / max(calls, 1) for s, t in stages.items()},
            "roofline": {"kernel": "moba_attn_tc_kernel", "bound": "tensor", "achieved": achieved, "peak": sust,
                         "unit": "TFLOP/s", "frac": achieved / sust, "traffic": traffic,
                         "peak_source": f"bf16_tflops_sustained (kernel timed inside a long step), {peak_src}"},
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
            "device_status": status,
        })
        if dense:
            line["dense"] = dense
            line["speedup_vs_dense"] = dense["ms"] / ms_per_step
        line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def decode_bytes(B, Hq, Hkv, L, d, bs, topk, idx_host, full: bool) -> tuple[float, int]:
    """Algorithmic HBM bytes of one decode step: K and V of the blocks the step reads (the union of
    the kept blocks of each kv head's query heads, the own block up to L - 1), the block summaries
    the gate reads (fp64, c rows per kv head), q in and out / lse written. Also the number of
    blocks read."""
    c = (L - 1) // bs
    G = Hq // Hkv
    blocks = 0
    keys = 0
    for b in range(B):
        for hk in range(Hkv):
            if full:
                kept = set(range(c + 1))
            else:
                kept = {int(j) for h in range(hk * G, (hk + 1) * G) for j in idx_host[b, h] if j >= 0}
            blocks += len(kept)
            keys += sum((L - j * bs) if j == c else bs for j in kept)
    kv = keys * 2 * d * 2
    gate = 0 if full else B * Hkv * c * d * 8
    return float(kv + gate + B * Hq * d * 2 * 2 + B * Hq * 4), blocks


def run_decode(args):
    """One decode step per sequence: the newest query of each of the workload's sequences against
    a KV cache holding the workload's length (all sequences of the batch the same length)."""
    import torch

    from block_sparse_long_gate_b200.build import build_library
    build_library()
    import block_sparse_long_gate_b200 as moba
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        raise SystemExit("--mode decode runs on one GPU")
    dev = torch.device("cuda", 0)
    w = workload(args.seq_len, args.hq, args.hkv, args.config)
    B, L, Hq, Hkv, d, bs, topk = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], w["block_size"], w["topk"]
    _, k_h, v_h = synth.inputs(B, L, 1, Hkv, d, bs, w["seed"], pin=True)
    q_h = synth.normal(w["seed"] + 1000, synth.Q_ID, (B, Hq, d), pin=True)
    k, v, q = k_h.to(dev), v_h.to(dev), q_h.to(dev)
    del k_h, v_h
    kbar = moba.pool_cache(k, bs, L)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    idx = torch.empty((B, Hq, topk), dtype=torch.int32, device=dev)
    res = {}
    stream = torch.cuda.current_stream()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else "0"
    peaks, peak_src = read_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clocks = None
    for full in (False, True):
        ws = torch.empty(moba.decode_workspace_size(B, Hq, Hkv, L, d, bs, topk, full), dtype=torch.uint8, device=dev)

        def step():
            moba.decode(q, k, v, kbar, bs, topk, L, full_attention=full, out=out, lse=lse,
                        idx=None if full else idx, workspace=ws)

        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize()
        n = max(args.steps, 20)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        l0 = moba.launch_count()
        with ClockSampler(gpu_id) as clk:
            for a, b_ in ev:
                flush.fill_(1)  # the cache is re-read from HBM, not L2, every step
                a.record(stream)
                step()
                b_.record(stream)
            torch.cuda.synchronize()
        launches = (moba.launch_count() - l0) // n
        us = statistics.median(a.elapsed_time(b_) for a, b_ in ev) * 1e3
        status = moba.sync_status()
        nbytes, blocks = decode_bytes(B, Hq, Hkv, L, d, bs, topk, None if full else idx.cpu().numpy(), full)
        res["full" if full else "moba"] = {"us": us, "bytes": nbytes, "blocks_read": blocks,
                                           "achieved_gbs": nbytes / (us * 1e-6) / 1e9, "launches": launches,
                                           "status": status}
        if not full:
            clocks = clk.summary()
        del ws
    sd = None
    if not args.no_sdpa:  # torch's fused attention of the single query over the whole cache
        from torch.nn.attention import SDPBackend, sdpa_kernel
        qt = q.unsqueeze(2)
        kt, vt = k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3)
        try:
            with sdpa_kernel([SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION]):
                for _ in range(3):
                    torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, enable_gqa=Hq != Hkv)
                torch.cuda.synchronize()
                ts = []
                for _ in range(10):
                    flush.fill_(1)
                    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, enable_gqa=Hq != Hkv)
                    b_.record(stream)
                    torch.cuda.synchronize()
                    ts.append(a.elapsed_time(b_) * 1e3)
            sd = {"us": statistics.median(ts), "kernel": "torch sdpa"}
        except RuntimeError as exc:
            sd = {"error": str(exc).splitlines()[0][:200]}
    m = res["moba"]
    line = {
        "metric": "MoBA decode step latency (one new token per sequence)", "value": m["us"], "unit": "us",
        "n_gpus": 1, "steps": max(args.steps, 20), "warmup": max(args.warmup, 3), "ms_per_step": m["us"] / 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "decode step, KV cache of " + workload_name(w), "global_batch": B, "seq_len": L,
                   "parallelism": "single GPU", "l2": "a 256 MB buffer is rewritten before every timed step"},
        "tokens_per_s": B / (m["us"] * 1e-6),
        "roofline": {"kernel": "moba decode (select, union, attend, merge)", "bound": "hbm", "achieved": m["achieved_gbs"],
                     "peak": hbm, "unit": "GB/s", "frac": m["achieved_gbs"] / hbm, "traffic": None,
                     "bytes_per_step": m["bytes"], "peak_source": f"hbm_gbs of {peak_src}"},
        "full_attention_decode": res["full"],
        "speedup_vs_full_attention_decode": res["full"]["us"] / m["us"],
        "torch_sdpa_decode": sd,
        "gpu_launches": m["launches"], "clocks": clocks, "device_status": m["status"],
        "blocks_read": m["blocks_read"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_backward(args):
    """The backward of the workload's forward (dq, dk, dv through its selection), timed on its own:
    useful work = 2.5 x the forward's useful FLOPs (five products per attended pair instead of two)."""
    import torch

    from block_sparse_long_gate_b200.build import build_library
    build_library()
    import block_sparse_long_gate_b200 as moba
    from block_sparse_long_gate_b200 import flops as fx
    import synth

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--mode backward runs on one GPU")
    dev = torch.device("cuda", 0)
    w = workload(args.seq_len, args.hq, args.hkv, args.config)
    B, N, Hq, Hkv, d, bs, topk = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], w["block_size"], w["topk"]
    q_h, k_h, v_h = host_inputs(w, w["seed"], pin=True)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    g = synth.normal(w["seed"] + 7, synth.V_ID, (B, N, Hq, d)).to(dev)
    out, lse = moba.forward(q, k, v, bs, topk)
    idx = moba.gate(q, k, bs, topk)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(moba.backward_workspace_size(B, Hq, Hkv, N, d, bs, topk), dtype=torch.uint8, device=dev)

    def step():
        moba.backward(q, k, v, out, lse, g, bs, topk, idx=idx, dq=dq, dk=dk, dv=dv, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else "0"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0 = moba.launch_count()
    with ClockSampler(gpu_id) as clk:
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    status = moba.sync_status()
    fl = 2.5 * fx.useful_flops(B, Hq, N, d, bs, topk)
    value = fl / (ms * 1e-3) / 1e12
    peaks, peak_src = read_peaks()
    sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    line = {
        "metric": "MoBA backward useful TFLOP/s (dq, dk, dv)", "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "backward of " + workload_name(w), "global_batch": B, "seq_len": N,
                   "parallelism": "single GPU", "l2": "inputs far exceed the 126 MB L2"},
        "roofline": {"kernel": "moba_bwd_kernel and its helpers (whole backward)", "bound": "tensor",
                     "achieved": value, "peak": sust, "unit": "TFLOP/s", "frac": value / sust, "traffic": None,
                     "peak_source": f"bf16_tflops_sustained, {peak_src}"},
        "gpu_launches": (moba.launch_count() - l0) // max(args.steps, 1), "clocks": clk.summary(),
        "device_status": status,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.mode == "decode":
        return run_decode(args)
    if args.mode == "backward":
        return run_backward(args)
    return run_moba(args)


if __name__ == "__main__":
    sys.exit(main())
