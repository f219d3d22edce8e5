#!/usr/bin/env python
"""Throughput of the tensor-parallel MLP sublayer forward on B200.

Workload (default): S=2048, H=4096, F=16384, t=4 logical shards, bf16 storage,
f32 accumulation, tanh-GeLU, fused shard-reduce + residual + LayerNorm; seeded
synthetic inputs.  One step = one full sublayer forward
Y = LN(X + sum_i GeLU(X A_i) B_i) through the C ABI (three kernels: the
column-split GEMM with the GeLU epilogue, the row-split GEMM summing the shards
in TMEM, the reduce + residual + LayerNorm kernel).

Prints one JSON line (rank 0).  `value` is the whole-job TFLOP/s: the FLOPs
all ranks processed divided by the slowest rank's device time for the K timed
steps (CUDA events on the launching stream, barrier + synchronize on both
sides).  Multi-GPU runs are independent replicas of the workload, one per rank
(weak scaling); NCCL is used only for the barrier and the max over ranks.

`--impl reference` times the fp64 CPU oracle on the host cores instead (rows
sampled from the same workload each step); see the JSON's cpu_baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TP MLP block fwd TFLOP/s (bf16, 1 B200) and % of dense bf16 tensor peak"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 2**20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-rows", type=int, default=2048)
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"bf16_tflops": p["bf16_tflops"], "bf16_tflops_sustained": p.get("bf16_tflops_sustained"),
                "hbm_gbs": p["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def source_digest() -> str:
    """Hash of the GEMM kernel sources, to tie stored ncu counters to the code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "megatron_tensor_transformer_gelu_b200", "csrc")
    for name in ("gemm_tcgen05.cuh", "ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("source_digest") != source_digest():
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        import threading
        self.thread = threading.Thread(target=self._read, daemon=True)
        if self.proc:
            self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        win = [p for (ts, p) in self.samples if t0 - 0.15 <= ts <= t1 + 0.15]
        if not win:
            win = [p for (_, p) in self.samples]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in win if num(p[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in win for i, v in enumerate(p[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(win[0][2]),
                "reasons": reasons, "samples": len(win),
                "power_w_max": max((num(p[3]) or 0.0) for p in win)}


def max_over_ranks(values, world, device=None):
    """Element-wise max of per-rank floats across the process group (every rank
    gets the result); world == 1 returns them unchanged."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_tflops(flops_per_step: int, steps: int, world: int, ms_max: float) -> float:
    """Units all ranks processed / the slowest rank's time (weak scaling)."""
    return world * flops_per_step * steps / (ms_max * 1e-3) / 1e12


# ----------------------------------------------------------------- our arm

def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist

    from megatron_tensor_transformer_gelu_b200 import _lib as L
    from megatron_tensor_transformer_gelu_b200 import synth
    from megatron_tensor_transformer_gelu_b200.workloads import HEADLINE, WORKLOADS

    w = WORKLOADS[args.workload or HEADLINE]
    assert w.kind == "mlp" and w.dtype == "bf16"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from megatron_tensor_transformer_gelu_b200 import build as _build
    if rank == 0:
        _build.build()  # no-op when libtpblock.so is newer than its sources
    if world > 1:
        dist.barrier()
    L.lib()  # load the CUDA library (raises if it is not built)
    S, H, F, t = w.S, w.H, w.F, w.t
    inp = synth.gen_mlp(S, H, F, seed=w.seed + rank)
    X = inp.X.to(dev)
    As = [a.to(dev) for a in synth.split_columns(inp.A, t)]
    Bs = [b.to(dev) for b in synth.split_rows(inp.B, t)]
    Y = torch.empty(S, H, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(L.mlp_workspace_bytes(S, H, F, t, torch.bfloat16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    input_bytes = (X.numel() + sum(a.numel() for a in As) + sum(b.numel() for b in Bs)) * 2

    def step():
        L.mlp_forward(X, As, Bs, Y, ws, stream=stream)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    sampler = ClockSampler(local)
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    barrier()
    # ---- timed region: K steps, device time on the launching stream
    L.profile_enable(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    t_wall1 = time.time()
    ms_total = e0.elapsed_time(e1)
    prof = L.profile_collect()
    L.profile_enable(False)
    assert L.device_error() == 0, "a device-side wait timed out"

    # ---- end to end through the public call with host buffers
    Xh = inp.X.pin_memory()
    Yh = torch.empty(S, H, dtype=torch.bfloat16).pin_memory()
    Xd = torch.empty_like(X)

    def e2e_step():
        Xd.copy_(Xh, non_blocking=True)
        L.mlp_forward(Xd, As, Bs, Y, ws, stream=stream)
        Yh.copy_(Y, non_blocking=True)

    e2e_steps = max(1, min(args.steps, 200))
    with torch.cuda.stream(stream):
        for _ in range(max(1, min(args.warmup, 5))):
            e2e_step()
    barrier()
    with torch.cuda.stream(stream):
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        f1.record(stream)
    barrier()
    e2e_ms = f0.elapsed_time(f1)
    sampler.stop()

    ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], world, dev)

    result = None
    if rank == 0:
        peaks = load_peaks()
        ms_step = ms_total / args.steps
        value = whole_job_tflops(w.flops, args.steps, world, ms_total)
        e2e_value = whole_job_tflops(w.flops, e2e_steps, world, e2e_ms)
        _, g_launch, g_ms = prof.get("gemm_tcgen05", (0, 0, 0.0))
        _, ln_launch, ln_ms = prof.get("reduce_residual_layernorm", (0, 0, 0.0))
        launches = sum(v[0] for v in prof.values())
        gemm_flops_per_launch = w.flops / 2  # both GEMMs are 2*S*H*F
        achieved = gemm_flops_per_launch / (g_ms / g_launch * 1e-3) / 1e12 if g_launch else None
        traffic = stored_traffic("gemm_tcgen05", w.name)
        clocks = sampler.summary(t_wall0, t_wall1)
        ln_bytes = S * H * 4 + S * H * 2 * 2 + H * 8  # Zsum f32 read, X read, Y written, gamma/beta
        result = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded torch.randn; X~N(0,1), weights~N(0,1/fan_in))",
            "config": {
                "workload": w.name, "S": S, "H": H, "F": F, "t": t, "act": "gelu_tanh",
                "flops_per_step": w.flops, "parallelism": f"{t} logical TP shards per GPU; {world} independent replicas",
                "l2": f"inputs larger than L2 ({input_bytes / 2**20:.0f} MiB resident vs {L2_BYTES // 2**20} MiB L2)",
            },
            "pct_of_peak": round(100 * value / world / peaks["bf16_tflops"], 2),
            "roofline": {
                "kernel": "gemm_tcgen05",
                "bound": "tensor",
                "achieved": round(achieved, 2) if achieved else None,
                "peak": peaks["bf16_tflops"],
                "peak_source": peaks["source"] + " bf16 burst (MEASURED_PEAKS.json bf16_tflops)",
                "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_tflops"], 4) if achieved else None,
                "frac_of_sustained": (round(achieved / peaks["bf16_tflops_sustained"], 4)
                                      if achieved and peaks.get("bf16_tflops_sustained") else None),
                "traffic": traffic,
                "flops_per_launch": gemm_flops_per_launch,
                "avg_launch_ms": round(g_ms / g_launch, 5) if g_launch else None,
                "launches": g_launch,
                "share_of_step": round(g_ms / (g_ms + ln_ms), 4) if g_launch else None,
            },
            "other_kernels": {
                "reduce_residual_layernorm": {
                    "launches": ln_launch, "avg_launch_ms": round(ln_ms / max(ln_launch, 1), 5),
                    "bound": "hbm", "bytes_per_launch": ln_bytes,
                    "achieved_gbs": round(ln_bytes / (ln_ms / max(ln_launch, 1) * 1e-3) / 1e9, 1) if ln_launch else None,
                    "peak_gbs": peaks["hbm_gbs"],
                },
            },
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT,
                    "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2,
                    "steps": e2e_steps,
                    "note": "pinned host X -> device, tp_mlp_forward, device Y -> pinned host, one stream"},
            "gpu_launches": launches,
            "clocks": clocks,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# -------------------------------------------------- oracle on host cores

def cpu_oracle_timing(w, rows_per_step: int, steps: int, warmup: int):
    """Time the fp64 oracle (as it stands) on a row sample of the workload."""
    import numpy as np
    import torch

    from megatron_tensor_transformer_gelu_b200 import synth
    from oracle import tp_oracle as O

    inp = synth.gen_mlp(w.S, w.H, w.F, seed=w.seed)
    rows = list(range(min(rows_per_step, w.S)))
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    for _ in range(warmup):
        O.mlp_block(inp.X, inp.A, inp.B, rows=rows)
    t0 = time.perf_counter()
    for _ in range(steps):
        O.mlp_block(inp.X, inp.A, inp.B, rows=rows)
    dt = time.perf_counter() - t0
    flops = 4 * w.H * w.F * len(rows) * steps
    del np, torch
    return {"value": round(flops / dt / 1e12, 5), "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"{len(rows)} of {w.S} rows of {w.name} per step, {steps} step(s), fp64 numpy/OpenBLAS",
            "seconds": round(dt, 3)}


def run_reference(args, rank, world):
    from megatron_tensor_transformer_gelu_b200.workloads import HEADLINE, WORKLOADS
    if rank != 0:
        return None
    w = WORKLOADS[args.workload or HEADLINE]
    rows = 64
    cb = cpu_oracle_timing(w, rows, args.steps, args.warmup)
    ms_step = cb["seconds"] / args.steps * 1e3
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": cb["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded torch.randn)",
        "config": {"workload": w.name, "S": w.S, "H": w.H, "F": w.F, "t": w.t,
                   "sample_rows_per_step": rows},
        "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
        "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    res = run_ours(args, rank, world, local)
    if rank == 0 and res is not None:
        from megatron_tensor_transformer_gelu_b200.workloads import HEADLINE, WORKLOADS
        if not args.no_cpu_baseline:
            w = WORKLOADS[args.workload or HEADLINE]
            res["cpu_baseline"] = cpu_oracle_timing(w, args.cpu_sample_rows, 1, 0)
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
