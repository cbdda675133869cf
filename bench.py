#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 + RAC rollout linear on B200.

One step = one pass of the whole path over one batch of the dense rollout
projection (X bf16 4096 x 2048, W bf16 2048 x 2048, RAC k = 50%):
    weight_qdq(W)                 W' , Q(W), colamax_W   (trainer-side QDQ)
    nvfp4_quantize(X)             Q(X), channel scores, residual col-max
    rac_select                    top-k% mask, sel, Q(dX_sel)
    rac_weight_quant              Q(W_sel)
    w4a4_gemm_quantized           Y = s s' A B^T + s_R s_Ws R Ws^T  (bf16)
The metric is the effective throughput of the RAC linear, 2 M N (K + n_sel)
FLOPs per step over the whole step time, in TFLOP/s; the JSON line also
carries the GEMM TFLOP/s, the quantizer GB/s, the RAC overhead over plain
W4A4, per-call times and the roofline of the dominant kernel.

Multi-GPU: every rank runs an independent replica on its own batch (the path
has no exchange step), value = all ranks' FLOPs / max-over-ranks time.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4+RAC GEMM TFLOPS & % FP4 peak; quantizer GB/s & % HBM; RAC overhead %"
WORKLOADS = {
    # name: (M, K, N, k)
    "dense_rollout_projection": (4096, 2048, 2048, 50.0),
    "decode_step_up": (256, 4096, 11008, 50.0),
    "single_linear": (64, 512, 512, 50.0),
    "large_prefill": (32768, 4096, 4096, 50.0),
}
DEFAULT_WORKLOAD = "dense_rollout_projection"
FP4_OVER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ORACLE_SAMPLE_ROWS = 1024
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    p.add_argument("--k", type=float, default=None, help="RAC k percent (default: workload's)")
    p.add_argument("--no-graph", action="store_true", help="issue calls directly, no CUDA graphs")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- algorithmic work
def work(M, K, N, n_sel, width):
    """Algorithmic FLOPs / bytes per call (see the design notes)."""
    return {
        "prepare_weight": dict(bytes=6.5625 * N * K + 4 * K, bound="hbm"),
        "quantize": dict(bytes=4.0 * M * K + 0.5625 * M * K + 12 * K, bound="hbm"),
        "select": dict(bytes=2.5625 * M * n_sel + 0.5625 * M * width + 12 * K + 4 * n_sel, bound="hbm"),
        "weight_select": dict(bytes=2.0 * N * n_sel + 0.5625 * N * width, bound="hbm"),
        "gemm": dict(flops=2.0 * M * N * (K + n_sel), bytes=0.5625 * (M + N) * (K + width) + 2.0 * M * N,
                     bound="tensor"),
    }


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"nvfp4_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        power = [float(r[3]) for r in rows if re.match(r"^[0-9.]+$", r[3])]
        loaded = [float(r[1]) for r in rows if re.match(r"^[0-9.]+$", r[3]) and float(r[3]) > 250.0]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(loaded or sm) if (loaded or sm) else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- profile traffic
def kernel_sources_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "precision_rl_rollout_nvfp4_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """dram bytes per launch recorded in profiles/ for this kernel and
    workload, or None when absent or taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    if not os.path.exists(path):
        return None
    src = kernel_sources_hash()
    with open(path) as f:
        for line in f:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 4 and cells[0] == kernel and cells[1] == workload and cells[3] == src:
                try:
                    return float(cells[2])
                except ValueError:
                    return None
    return None


# ---------------------------------------------------------------- ranks
def max_over_ranks(values, world, device="cpu"):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def replica_seed(rank):
    """Each data-parallel replica quantizes its own batch."""
    return rank


# ---------------------------------------------------------------- ours
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from precision_rl_rollout_nvfp4_b200 import binding as B
    from precision_rl_rollout_nvfp4_b200 import synthetic as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M, K, N, k = WORKLOADS[args.workload]
    k = args.k if args.k is not None else k
    seed = replica_seed(rank)
    x_host = S.activations(M, K, seed=seed).pin_memory()
    w_host = S.weights(N, K, seed=seed).pin_memory()
    x = x_host.to(dev)
    w = w_host.to(dev)
    plan = B.RacLinearPlan(M, K, N, k, out_dtype=torch.bfloat16, device=dev).bind(x, w)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    calls = ["prepare_weight", "quantize", "select", "weight_select", "gemm"]
    fns = {"prepare_weight": plan.prepare_weight, "quantize": plan.quantize, "select": plan.select,
           "weight_select": plan.weight_select, "gemm": plan.gemm}

    def full_step():
        plan.full_step()                      # weight prep overlapped on a side stream

    # warm-up (also sets kernel attributes before any capture)
    for _ in range(max(args.warmup, 1)):
        full_step()
        plan.plain_step()
    torch.cuda.synchronize()
    if B.stream_status() != 0:
        raise RuntimeError("device error word set during warm-up")

    use_graph = not args.no_graph
    graphs = {}
    if use_graph:
        try:
            for name, fn in [("step", full_step), ("plain", plan.plain_step)] + [(c, fns[c]) for c in calls]:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    fn()
                graphs[name] = g
            torch.cuda.synchronize()
        except Exception as exc:  # capture not possible: time direct calls
            print(f"# CUDA graph capture failed ({exc}); timing direct calls", file=sys.stderr)
            use_graph = False
            graphs = {}

    def launch(name):
        if use_graph:
            graphs[name].replay()
        elif name == "step":
            full_step()
        elif name == "plain":
            plan.plain_step()
        else:
            fns[name]()

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        flush.zero_()
        launch("step")
    torch.cuda.synchronize()

    # ---- timed region: K full steps, L2 flushed between steps
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        step_ms = []
        for _ in range(args.steps):
            flush.zero_()
            e0 = ev()
            launch("step")
            e1 = ev()
            step_ms.append((e0, e1))
        torch.cuda.synchronize()
        barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in step_ms)
    clock = clocks.summary()

    # per-call breakdown inside the same sequence (same L2 state as a step)
    per_call = {c: [] for c in calls}
    for _ in range(args.steps):
        flush.zero_()
        evs = [ev()]
        for c in calls:
            launch(c)
            evs.append(ev())
        torch.cuda.synchronize()
        for i, c in enumerate(calls):
            per_call[c].append(evs[i].elapsed_time(evs[i + 1]))
    # plain W4A4 linear (no RAC) and the RAC linear without weight prep, for the overhead
    plain_ms, rac_ms = [], []
    for _ in range(args.steps):
        flush.zero_()
        a = ev(); launch("plain"); b_ = ev()
        flush.zero_()
        c = ev()
        for name in calls[1:]:
            launch(name)
        d = ev()
        torch.cuda.synchronize()
        plain_ms.append(a.elapsed_time(b_))
        rac_ms.append(c.elapsed_time(d))

    # ---- end to end through the API from pinned host buffers
    y_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        e0 = ev()
        x.copy_(x_host, non_blocking=True)
        w.copy_(w_host, non_blocking=True)
        full_step()
        y_host.copy_(plan.y, non_blocking=True)
        e1 = ev()
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    if B.stream_status() != 0:
        raise RuntimeError("device error word set during timing")

    total_ms, e2e_total = max_over_ranks([total_ms, sum(e2e_ms)], world, dev)

    n_sel, width = plan.n_sel, plan.width
    flops_step = 2.0 * M * N * (K + n_sel)
    ms_per_step = total_ms / args.steps
    value = flops_step * world * args.steps / (total_ms * 1e-3) / 1e12
    e2e_value = flops_step * world * args.steps / (e2e_total * 1e-3) / 1e12
    med = {c: statistics.median(v) for c, v in per_call.items()}
    wk = work(M, K, N, n_sel, width)
    peaks, peak_kind = load_peaks()
    hbm_peak = peaks["hbm_gbs"]
    fp4_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * FP4_OVER_BF16
    dominant = max(med, key=med.get)
    d = wk[dominant]
    dur = med[dominant] * 1e-3
    traffic = profiled_traffic(dominant, args.workload)
    if d["bound"] == "tensor":
        achieved = d["flops"] / dur / 1e12
        roof = {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 1),
                "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / fp4_peak, 4),
                "traffic": traffic, "peak_source": f"{peak_kind}: bf16 sustained x {FP4_OVER_BF16:g} (FP4/BF16 nominal)"}
    else:
        achieved = d["bytes"] / dur / 1e9
        roof = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                "peak_source": f"{peak_kind}: hbm_gbs"}
    gemm_tflops = wk["gemm"]["flops"] / (med["gemm"] * 1e-3) / 1e12
    quant_gbs = wk["quantize"]["bytes"] / (med["quantize"] * 1e-3) / 1e9
    rac_over = (statistics.median(rac_ms) - statistics.median(plain_ms)) / statistics.median(plain_ms)
    launches_per_step = sum(B.RacLinearPlan.LAUNCHES[c] for c in calls) - (0 if n_sel else 2)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s (effective 2MN(K+n_sel) per step)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1/ue4m3) x fp32 acc",
        "data": "synthetic (seeded channel-scaled heavy-tailed X, N(0,0.02) W; see DESIGN.md)",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N, "k_percent": k, "n_sel": n_sel,
                   "y_dtype": "bf16", "parallelism": f"replicas x{world}", "l2": "flushed between steps (256 MiB write)",
                   "cuda_graph": use_graph},
        "gemm_tflops": round(gemm_tflops, 1), "gemm_frac_fp4_peak": round(gemm_tflops / fp4_peak, 4),
        "quantizer_gbs": round(quant_gbs, 1), "quantizer_frac_hbm": round(quant_gbs / hbm_peak, 4),
        "rac_overhead_pct": round(100 * rac_over, 1),
        "plain_w4a4_linear_us": round(1e3 * statistics.median(plain_ms), 2),
        "rac_linear_us": round(1e3 * statistics.median(rac_ms), 2),
        "per_call_us": {c: round(1e3 * v, 2) for c, v in med.items()},
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": int(2 * (M * K + N * K)),
                "d2h_bytes_per_step": int(2 * M * N), "ms_per_step": round(e2e_total / args.steps, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clock,
    }
    return line


# ---------------------------------------------------------------- oracle (CPU)
def oracle_step_time(M, K, N, k, rows, seed=0):
    import numpy as np

    import oracle
    from precision_rl_rollout_nvfp4_b200 import synthetic as S
    x = S.bf16_bits(S.activations(M, K, seed=seed))[:rows]
    w = S.bf16_bits(S.weights(N, K, seed=seed))
    t0 = time.perf_counter()
    wq = oracle.weight_qdq(w)
    r = oracle.rac_linear(x, w, k, wq=wq)
    dt = time.perf_counter() - t0
    return dt, 2.0 * rows * N * (K + r["n_sel"]), np.asarray(r["y"]).shape


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(args, budget_s=12.0):
    M, K, N, k = WORKLOADS[args.workload]
    k = args.k if args.k is not None else k
    rows = min(M, ORACLE_SAMPLE_ROWS)
    t, flops, n = 0.0, 0.0, 0
    while t < budget_s or n == 0:
        dt, f, _ = oracle_step_time(M, K, N, k, rows)
        t += dt
        flops += f
        n += 1
        if n >= 8:
            break
    return {"value": round(flops / t / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} oracle step(s) of weight_qdq(W {N}x{K}) + RAC linear on the first {rows} of {M} "
                      f"rows of X (numpy; fp64 product via BLAS)"}


def run_reference(args):
    M, K, N, k = WORKLOADS[args.workload]
    k = args.k if args.k is not None else k
    rows = min(M, ORACLE_SAMPLE_ROWS)
    for _ in range(args.warmup):
        oracle_step_time(M, K, N, k, rows)
    t, flops = 0.0, 0.0
    for _ in range(args.steps):
        dt, f, _ = oracle_step_time(M, K, N, k, rows)
        t += dt
        flops += f
    value = flops / t / 1e12
    cores = blas_threads()
    sample = (f"weight_qdq(W {N}x{K}) + RAC linear on the first {rows} of {M} rows of X per step "
              f"(numpy oracle; fp64 product via BLAS)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s (effective 2MN(K+n_sel) per step)",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantizer steps, f64 product",
            "data": "synthetic", "config": {"workload": args.workload, "M": M, "K": K, "N": N, "k_percent": k},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(args)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
