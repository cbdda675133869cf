#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 + RAC rollout linear on B200.

Default workload: large prefill + trainer QDQ.  One step is one pass of the
whole path over one batch:
    weight_qdq(W)                 W', Q(W), colamax_W   (weight preparation)
    nvfp4_quantize(X)             Q(X), channel scores, residual col-max
    rac_select                    top-k% mask, sel, Q(dX_sel)
    rac_weight_quant              Q(W_sel)
    w4a4_gemm_quantized           Y = s s' A B^T + s_R s_Ws R Ws^T  (bf16)
for X bf16 32768 x 4096, W bf16 4096 x 4096, RAC k = 50%, plus the trainer's
W4A16 fake quantization weight_qdq over 64 experts x (1024 x 2048 and
2048 x 1024) bf16 weights (independent of the linear, on its own stream).
The metric is the effective throughput of the RAC linear, 2 M N (K + n_sel)
FLOPs per step over the whole step time, in TFLOP/s; the JSON line also
carries the GEMM TFLOP/s, the quantizer GB/s, the RAC overhead over plain
W4A4, the expert QDQ time and GB/s, per-call times, a bf16 GEMM of the same
shape for comparison and the roofline of the dominant kernel.

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
    "decode_step_down": (256, 11008, 4096, 50.0),
    "single_linear": (64, 512, 512, 50.0),
    "large_prefill": (32768, 4096, 4096, 50.0),
}
DEFAULT_WORKLOAD = "large_prefill"
# trainer-side W4A16 QDQ of a stacked expert weight set that runs with a
# workload's step: workload -> (experts, [(N, K) of each stacked weight])
QDQ_EXPERTS = {"large_prefill": (64, [(1024, 2048), (2048, 1024)])}
# grouped MoE expert FFN (up 2048 -> 1024, down 1024 -> 2048 over 64 experts,
# 8192 tokens routed top-8): its own step, see run_moe
MOE_WORKLOAD = "moe_expert_ffn"
# trainer-side QAT step of one linear (forward + backward): (M, K, N, act_quant)
QAT_WORKLOADS = {"qat_w4a16_step": (4096, 2048, 2048, False), "qat_w4a4_step": (4096, 2048, 2048, True)}
FP4_OVER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ORACLE_SAMPLE_ROWS = 1024
L2_FLUSH_BYTES = 256 << 20
PER_CALL_REPS = 10
PER_CALL_SAMPLES = 20       # per-call graphs of PER_CALL_REPS launches timed this many times


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=sorted(WORKLOADS) + [MOE_WORKLOAD] + sorted(QAT_WORKLOADS),
                   default=DEFAULT_WORKLOAD)
    p.add_argument("--k", type=float, default=None, help="RAC k percent (default: workload's)")
    p.add_argument("--no-graph", action="store_true", help="issue calls directly, no CUDA graphs")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--wsel", choices=["bf16", "fp4"], default="bf16",
                   help="W_sel source: the bf16 weight (default) or its NVFP4 codes (variant)")
    p.add_argument("--static-amax", action="store_true",
                   help="pass max|X| as a caller-supplied amax (computed once before timing), so the "
                        "quantizer skips its amax pass")
    p.add_argument("--mask", choices=["per_call", "reuse"], default="per_call",
                   help="reuse: keep the channel mask, sel and Q(W_sel) of a first selecting step and time "
                        "the steps that reuse them (variant; weights resident, no weight preparation)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- algorithmic work
def work(M, K, N, n_sel, width, wsel="bf16", static_amax=False):
    """Algorithmic FLOPs / bytes per call.  Bytes count every tensor a call
    must read or write once: X is read twice by the quantizer (its amax is a
    global dependency of every code) unless the caller supplies amax; the
    residual gather reads the selected channels of X plus their codes and
    scales; the GEMM reads the FP4 operands and writes bf16 Y.  With
    wsel="fp4" the weight preparation also reads Q(W) once for the DQ column
    maxima, and W_sel is gathered from the 0.5625 B/element NVFP4 weight."""
    fp4 = wsel == "fp4"
    d = {
        "prepare_weight": dict(bytes=6.5625 * N * K + 4 * K + (0.5625 * N * K + 4 * K if fp4 else 0.0),
                               bound="hbm"),
        "quantize": dict(bytes=(2.0 if static_amax else 4.0) * M * K + 0.5625 * M * K + 12 * K, bound="hbm"),
        "select": dict(bytes=2.5625 * M * n_sel + 0.5625 * M * width + 12 * K + 4 * n_sel, bound="hbm"),
        "weight_select": dict(bytes=(0.5625 if fp4 else 2.0) * N * n_sel + 0.5625 * N * width, bound="hbm"),
        "gemm": dict(flops=2.0 * M * N * (K + n_sel), bytes=0.5625 * (M + N) * (K + width) + 2.0 * M * N,
                     bound="tensor"),
    }
    # the fused calls of the step: quantize + selection, and both second passes
    d["quantize_select"] = dict(bytes=d["quantize"]["bytes"] + 4 * n_sel + K, bound="hbm")
    d["second_pass"] = dict(bytes=d["select"]["bytes"] - 12 * K - 4 * n_sel + 4 * n_sel + d["weight_select"]["bytes"],
                            bound="hbm")
    return d


# ---------------------------------------------------------------- clocks
def gpu_selector(local_rank):
    """The `nvidia-smi -i` argument that names the GPU this process runs on:
    its UUID ("GPU-..."), else its PCI bus id.  nvidia-smi ignores
    CUDA_VISIBLE_DEVICES, so a bare index could name another GPU of the
    machine.  None when neither is known."""
    try:
        import torch
        props = torch.cuda.get_device_properties(local_rank)
    except Exception:
        return None
    u = str(getattr(props, "uuid", "") or "")
    if u:
        return u if u.startswith("GPU-") else "GPU-" + u
    try:
        return f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    except AttributeError:
        return None


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank):
        self.gpu = gpu_selector(local_rank)
        self.proc = None
        self.path = os.path.join("/tmp", f"nvfp4_clocks_{os.getpid()}.csv")

    def __enter__(self):
        if self.gpu is None:              # unknown identity: sample nothing rather than another GPU
            return self
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
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
        return {"gpu": self.gpu, "sm_mhz": statistics.median(loaded or sm) if (loaded or sm) else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- profile traffic
KERNEL_SOURCES = ("common.cuh", "gemm.cu", "kernels.h", "quant.cu", "select.cu", "topk.cuh")
# the files that hold each call's kernels and their launch code (a recorded
# DRAM figure stays valid while these are unchanged)
CALL_SOURCES = {"gemm": ("common.cuh", "gemm.cu", "kernels.h"),
                "gemm_plain": ("common.cuh", "gemm.cu", "kernels.h")}


def kernel_sources_hash(call=None):
    """sha256 (first 16 hex digits) over the files that hold the kernels of
    `call` (all kernel files when None) and their launch code; the host-only
    ABI layer is not part of it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "precision_rl_rollout_nvfp4_b200", "csrc")
    for name in CALL_SOURCES.get(call, KERNEL_SOURCES):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """dram bytes per launch recorded in profiles/ for this kernel and
    workload, or None when absent or taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    if not os.path.exists(path):
        return None
    src = kernel_sources_hash(kernel)
    with open(path) as f:
        for line in f:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 4 and cells[0] == kernel and cells[1] == workload and cells[3] == src:
                try:
                    return float(cells[2])
                except ValueError:
                    return None
    return None


# ---------------------------------------------------------------- end to end
def e2e_pipelined(sets, steps, warmup):
    """End-to-end time of `steps` steps through the public API with host
    buffers: every step copies its inputs from pinned host memory, runs, and
    reads its result back.  Two buffer sets alternate, and the host-to-device
    copies, the compute and the device-to-host copies sit on three streams,
    so step i+1's inputs travel while step i computes.  sets: two dicts with
    "h2d" [(device dst, host src)], "d2h" [(host dst, device src)] and "step"
    (enqueues the step on the current stream).  Returns ms over the steps,
    measured on the device from before the first copy to after the last one."""
    import torch
    H, D = torch.cuda.Stream(), torch.cuda.Stream()
    C = torch.cuda.current_stream()
    ev_comp, ev_d2h = [None, None], [None, None]

    def one(i):
        b = i % 2
        st = sets[b]
        with torch.cuda.stream(H):
            if ev_comp[b] is not None:
                H.wait_event(ev_comp[b])          # step i-2 is done reading these inputs
            for dst, src in st["h2d"]:
                dst.copy_(src, non_blocking=True)
            eh = torch.cuda.Event()
            eh.record(H)
        C.wait_event(eh)
        if ev_d2h[b] is not None:
            C.wait_event(ev_d2h[b])               # step i-2's result has left
        st["step"]()
        ec = torch.cuda.Event()
        ec.record(C)
        ev_comp[b] = ec
        with torch.cuda.stream(D):
            D.wait_event(ec)
            for dst, src in st["d2h"]:
                dst.copy_(src, non_blocking=True)
            ed = torch.cuda.Event()
            ed.record(D)
            ev_d2h[b] = ed

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(H)
    for i in range(warmup, warmup + steps):
        one(i)
    t1.record(D)                                  # after the last step's result left
    torch.cuda.synchronize()
    return t0.elapsed_time(t1)


# ---------------------------------------------------------------- launches
def graph_kernel_count(g):
    """Kernel nodes in a captured torch CUDA graph (None when the graph or
    cuda-python cannot tell)."""
    if g is None:
        return None
    try:
        from cuda.bindings import runtime as rt
        raw = rt.cudaGraph_t(init_value=int(g.raw_cuda_graph()))
        err, nodes, n = rt.cudaGraphGetNodes(raw, 0)
        err, nodes, n = rt.cudaGraphGetNodes(raw, n)
        count = 0
        for nd in nodes[:n]:
            err, ty = rt.cudaGraphNodeGetType(nd)
            if ty == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                count += 1
        return count
    except Exception:
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
class ExpertQDQ:
    """The trainer-side W4A16 fake quantization of a stacked expert weight
    set (one weight_qdq call per stacked weight shape), with preallocated
    outputs and workspaces, so it can be captured in a CUDA graph."""

    def __init__(self, B, experts, shapes, seed, dev, hosts=None):
        import torch

        from precision_rl_rollout_nvfp4_b200 import synthetic as S
        self.B = B
        self.hosts, self.w, self.out, self.ws = [], [], [], []
        for i, (n, kk) in enumerate(shapes):
            h = (S.weights(n, kk, seed, batch=experts, stream=S.STREAM_W + 10 * i).pin_memory()
                 if hosts is None else hosts[i])
            self.hosts.append(h)
            self.w.append(h.to(dev))
            self.out.append(torch.empty(experts, n, kk, dtype=torch.bfloat16, device=dev))
            self.ws.append(torch.empty(B.workspace_size(B.OP_WEIGHT_QDQ, 0, n, kk, experts),
                                       dtype=torch.uint8, device=dev))
        self.shapes, self.experts = shapes, experts
        self.elements = sum(experts * n * kk for n, kk in shapes)

    def run(self, stream=None):
        for w, out, ws in zip(self.w, self.out, self.ws):
            self.B.weight_qdq(w, want_q=False, want_colamax=False, out=out, stream=stream, ws=ws)

    def bytes(self):
        """Algorithmic bytes: W read twice (amax, then the quantization) and
        W' written once, 2 bytes each."""
        return 6.0 * self.elements


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
    # a caller-supplied amax (its own max here, taken once outside every timed region)
    amax = x.detach().abs().max().float().reshape(1) if args.static_amax else None
    plan = B.RacLinearPlan(M, K, N, k, out_dtype=torch.bfloat16, device=dev, wsel=args.wsel).bind(x, w, amax)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    # the calls of one step, each timed alone below: weight preparation, the
    # quantize pass with the fused top-k selection, both second passes, GEMM
    calls = ["prepare_weight", "quantize_select", "second_pass", "gemm"]
    fns = {"prepare_weight": plan.prepare_weight, "quantize_select": plan.quantize_select,
           "second_pass": plan.second_pass, "gemm": plan.gemm}
    reuse = args.mask == "reuse"
    qdq = None
    if args.workload in QDQ_EXPERTS and not reuse:
        E_q, shapes = QDQ_EXPERTS[args.workload]
        qdq = ExpertQDQ(B, E_q, shapes, seed, dev)
        calls.append("qdq_experts")
        fns["qdq_experts"] = qdq.run
    qstream = torch.cuda.Stream(device=dev)
    q_fork, q_join = torch.cuda.Event(), torch.cuda.Event()

    def linear_step(p):
        if reuse:
            p.reuse_step()                    # mask, sel and Q(W_sel) kept from the warm-up
        else:
            p.full_step()                     # weight prep overlapped on a side stream

    def step_with(p, q):
        """The linear on the current stream; the expert QDQ (independent of
        it) on its own stream, forked from and joined back into the current one."""
        main = torch.cuda.current_stream()
        if q is not None:
            q_fork.record(main)
            qstream.wait_event(q_fork)
            q.run(stream=qstream)
            q_join.record(qstream)
        linear_step(p)
        if q is not None:
            main.wait_event(q_join)

    def full_step():
        step_with(plan, qdq)

    # warm-up (also sets kernel attributes before any capture; with --mask
    # reuse the first full step selects the mask the timed steps keep)
    if reuse:
        plan.full_step()
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
                g = torch.cuda.CUDAGraph(keep_graph=(name == "step"))   # kept: its kernel nodes are counted
                with torch.cuda.graph(g):
                    fn()
                if name == "step":
                    g.instantiate()
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

    # per-call breakdown: each call's average launch duration with L2
    # flushed before every launch, from one graph of PER_CALL_REPS (flush,
    # call) pairs minus a graph of the flushes alone (no replay gaps inside),
    # sampled PER_CALL_SAMPLES times
    per_call = {c: [] for c in calls}

    def reps_graph(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(PER_CALL_REPS):
                flush.zero_()
                fn()
        return g

    def time_graph(g):
        g.replay()
        a = ev()
        g.replay()
        b = ev()
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    # comparators timed the same way (not part of the step): the plain W4A4
    # GEMM alone, and the FP8 path on the same shape -- MXFP8 quantization of
    # X and the kind::mxf8f6f4 W8A8 GEMM (W quantized once beforehand)
    cmp_fns = {"gemm_plain": lambda: plan.gemm(plain=True), "quantize": plan.quantize}
    if K % 256 == 0:
        qa8, qb8 = B.mxfp8_quantize(x), B.mxfp8_quantize(w)
        y8 = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        cmp_fns["fp8_quantize"] = lambda: B.mxfp8_quantize(x, out=qa8)
        cmp_fns["fp8_gemm"] = lambda: B.w8a8_gemm(qa8, qb8, out=y8)
        for f in cmp_fns.values():
            f()
        torch.cuda.synchronize()
    cmp_call = {c: [] for c in cmp_fns}
    if use_graph:
        g_flush = reps_graph(lambda: None)
        g_calls = {c: reps_graph(fns[c]) for c in calls}
        g_cmp = {c: reps_graph(f) for c, f in cmp_fns.items()}
        torch.cuda.synchronize()
        for _ in range(PER_CALL_SAMPLES):
            base = time_graph(g_flush)
            for c in calls:
                per_call[c].append(max(time_graph(g_calls[c]) - base, 0.0) / PER_CALL_REPS)
            for c in cmp_fns:
                cmp_call[c].append(max(time_graph(g_cmp[c]) - base, 0.0) / PER_CALL_REPS)
        del g_flush, g_calls, g_cmp
    else:
        for _ in range(max(args.steps, PER_CALL_SAMPLES)):
            flush.zero_()
            evs = [ev()]
            for c in calls:
                launch(c)
                evs.append(ev())
            torch.cuda.synchronize()
            for i, c in enumerate(calls):
                per_call[c].append(evs[i].elapsed_time(evs[i + 1]))
            for c, f in cmp_fns.items():
                flush.zero_()
                a = ev(); f(); b_ = ev()
                torch.cuda.synchronize()
                cmp_call[c].append(a.elapsed_time(b_))
    # the RAC linear without weight preparation as one graph (launch count)
    g_rac = None
    if use_graph and not reuse:
        g_rac = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g_rac):
            plan.quantize_select()
            plan.second_pass()
            plan.gemm()
        g_rac.instantiate()
        torch.cuda.synchronize()
    # plain W4A4 linear (no RAC) and the RAC linear without weight prep, for the overhead
    plain_ms, rac_ms = [], []
    for _ in range(args.steps):
        flush.zero_()
        a = ev(); launch("plain"); b_ = ev()
        flush.zero_()
        c = ev()
        if reuse:
            launch("step")
        else:
            for name in ("quantize_select", "second_pass", "gemm"):
                launch(name)
        d = ev()
        torch.cuda.synchronize()
        plain_ms.append(a.elapsed_time(b_))
        rac_ms.append(c.elapsed_time(d))

    # bf16 comparator: the same product Y = X W^T as one torch (cuBLAS) bf16
    # GEMM, timed the same way (a comparison only; not part of the step)
    y_bf16 = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

    def bf16_gemm():
        torch.matmul(x, w.t(), out=y_bf16)

    bf16_gemm()
    bf16_ms = []
    for _ in range(max(args.steps, 5)):
        flush.zero_()
        a = ev(); bf16_gemm(); b_ = ev()
        torch.cuda.synchronize()
        bf16_ms.append(a.elapsed_time(b_))
    del y_bf16

    # ---- end to end through the API from pinned host buffers (two buffer
    # sets, copies overlapped with the neighbouring steps' compute)
    x1, w1 = torch.empty_like(x), torch.empty_like(w)
    plan1 = B.RacLinearPlan(M, K, N, k, out_dtype=torch.bfloat16, device=dev, wsel=args.wsel).bind(x1, w1, amax)
    qdq1 = ExpertQDQ(B, qdq.experts, qdq.shapes, seed, dev, hosts=qdq.hosts) if qdq is not None else None
    if reuse:                                 # weights resident; both plans select once, then reuse
        x1.copy_(x_host)
        w1.copy_(w_host)
        plan1.full_step()
        torch.cuda.synchronize()

    def h2d(p_x, p_w, q):
        pairs = [(p_x, x_host)] + ([] if reuse else [(p_w, w_host)])
        if q is not None:
            pairs += [(dst, src) for dst, src in zip(q.w, qdq.hosts)]
        return pairs

    sets = [{"h2d": h2d(x, w, qdq), "d2h": [(torch.empty(M, N, dtype=torch.bfloat16).pin_memory(), plan.y)],
             "step": lambda: step_with(plan, qdq)},
            {"h2d": h2d(x1, w1, qdq1), "d2h": [(torch.empty(M, N, dtype=torch.bfloat16).pin_memory(), plan1.y)],
             "step": lambda: step_with(plan1, qdq1)}]
    h2d_bytes = sum(dst.numel() * dst.element_size() for dst, _ in sets[0]["h2d"])
    e2e_ms = e2e_pipelined(sets, args.steps, max(args.warmup, 2))
    if B.stream_status() != 0:
        raise RuntimeError("device error word set during timing")

    total_ms, e2e_total = max_over_ranks([total_ms, e2e_ms], world, dev)

    n_sel, width = plan.n_sel, plan.width
    flops_step = 2.0 * M * N * (K + n_sel)
    ms_per_step = total_ms / args.steps
    value = flops_step * world * args.steps / (total_ms * 1e-3) / 1e12
    e2e_value = flops_step * world * args.steps / (e2e_total * 1e-3) / 1e12
    med = {c: statistics.median(v) for c, v in per_call.items()}
    wk = work(M, K, N, n_sel, width, args.wsel, args.static_amax)
    if qdq is not None:
        wk["qdq_experts"] = dict(bytes=qdq.bytes(), bound="hbm")
    peaks, peak_kind = load_peaks()
    hbm_peak = peaks["hbm_gbs"]
    # per-call kernels are timed alone, in bursts: the burst bf16 peak; the
    # whole step is a long loop: the sustained one
    fp4_burst = peaks["bf16_tflops"] * FP4_OVER_BF16
    fp4_sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * FP4_OVER_BF16
    dominant = max(med, key=med.get)
    d = wk[dominant]
    dur = med[dominant] * 1e-3
    traffic = profiled_traffic(dominant, args.workload)
    traffic_source = (f"profiles/dram_traffic.md, ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, "
                      f"kernel sources sha256 {kernel_sources_hash(dominant)}") if traffic is not None else None
    if d["bound"] == "tensor":
        achieved = d["flops"] / dur / 1e12
        roof = {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 1),
                "peak": round(fp4_burst, 1), "unit": "TFLOP/s", "frac": round(achieved / fp4_burst, 4),
                "traffic": traffic, "traffic_source": traffic_source,
                "peak_source": f"{peak_kind}: bf16 burst x {FP4_OVER_BF16:g} (FP4/BF16 nominal); kernel timed alone"}
    else:
        achieved = d["bytes"] / dur / 1e9
        roof = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                "traffic_source": traffic_source, "peak_source": f"{peak_kind}: hbm_gbs"}
    gemm_tflops = wk["gemm"]["flops"] / (med["gemm"] * 1e-3) / 1e12
    quant_gbs = wk["quantize"]["bytes"] / (statistics.median(cmp_call["quantize"])) / 1e6
    rac_over = (statistics.median(rac_ms) - statistics.median(plain_ms)) / statistics.median(plain_ms)
    bf16_us = 1e3 * statistics.median(bf16_ms)
    launches_per_step = graph_kernel_count(graphs.get("step")) if use_graph else None
    if launches_per_step is None:                 # static count of the step's calls
        launches_per_step = ((plan.launches["reuse_step"] if n_sel else 3) if reuse else
                             sum(plan.launches[c] for c in calls if c in plan.launches) - (0 if n_sel else 1)) \
            - (1 if args.static_amax else 0)      # no amax pass
        if qdq is not None:
            launches_per_step += 2 * len(qdq.shapes)  # amax pass + quantization per stacked weight
    rac_launches = graph_kernel_count(g_rac) if use_graph else None

    cfg = {"workload": args.workload, "M": M, "K": K, "N": N, "k_percent": k, "n_sel": n_sel,
           "y_dtype": "bf16", "wsel": args.wsel, "mask": args.mask,
           "amax": "caller-supplied" if args.static_amax else "computed per call",
           "parallelism": f"replicas x{world}",
           "l2": "flushed between steps and before every per-call launch (256 MiB write)",
           "cuda_graph": use_graph}
    if qdq is not None:
        cfg["qdq_experts"] = {"experts": qdq.experts, "shapes": [list(sh) for sh in qdq.shapes],
                              "stream": "own stream, overlapped with the linear"}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s (effective 2MN(K+n_sel) per step)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1/ue4m3) x fp32 acc",
        "data": "synthetic, seeded: X = N(0,1) x per-channel exp(N(0,1)) scales with 1% outlier channels x20, W = N(0, 0.02^2), bf16",
        "config": cfg,
        "useful_tflops": round(2.0 * M * N * K * world * args.steps / (total_ms * 1e-3) / 1e12, 2),
        "gemm_tflops": round(gemm_tflops, 1), "gemm_frac_fp4_peak": round(gemm_tflops / fp4_burst, 4),
        "quantizer_gbs": round(quant_gbs, 1), "quantizer_frac_hbm": round(quant_gbs / hbm_peak, 4),
        "rac_overhead_pct": round(100 * rac_over, 1),
        "plain_w4a4_linear_us": round(1e3 * statistics.median(plain_ms), 2),
        "rac_linear_us": round(1e3 * statistics.median(rac_ms), 2),
        "bf16_gemm_us": round(bf16_us, 2),
        "bf16_gemm_tflops": round(2.0 * M * N * K / (bf16_us * 1e-6) / 1e12, 1),
        "fp4_gemm_speedup_over_bf16": round(bf16_us / (1e3 * med["gemm"]), 3),
        "per_call_us": {c: round(1e3 * v, 2) for c, v in med.items()},
        "per_call_samples": len(next(iter(per_call.values()))),
        "peaks": {"fp4_burst_tflops": round(fp4_burst, 1), "fp4_sustained_tflops": round(fp4_sustained, 1),
                  "hbm_gbs": hbm_peak, "source": peak_kind},
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(2 * M * N),
                "ms_per_step": round(e2e_total / args.steps, 4),
                "pipelined": "2 buffer sets; H2D, compute and D2H on separate streams"},
        "gpu_launches": launches_per_step * args.steps,
        "launches_per_step": launches_per_step,
        "rac_linear_launches": rac_launches,
        "clocks": clock,
    }
    if "quantize_select" in med:
        line["quantize_select_gbs"] = round(wk["quantize"]["bytes"] / (med["quantize_select"] * 1e-3) / 1e9, 1)
    cmp_us = {c: 1e3 * statistics.median(v) for c, v in cmp_call.items() if v}
    line["comparators_us"] = {c: round(v, 2) for c, v in cmp_us.items()}
    if "fp8_gemm" in cmp_us:
        fl = 2.0 * M * N * K
        line["fp8_gemm_us"] = round(cmp_us["fp8_gemm"], 2)
        line["fp8_gemm_tflops"] = round(fl / (cmp_us["fp8_gemm"] * 1e-6) / 1e12, 1)
        line["fp4_gemm_plain_us"] = round(cmp_us["gemm_plain"], 2)
        # throughput of the NVFP4 W4A4 GEMM over the MXFP8 W8A8 GEMM, same M, N, K
        line["fp4_over_fp8"] = round(cmp_us["fp8_gemm"] / cmp_us["gemm_plain"], 3)
        line["fp4_rac_over_fp8"] = round(cmp_us["fp8_gemm"] / (1e3 * med["gemm"]), 3)
        line["fp8_linear_us"] = round(cmp_us["fp8_gemm"] + cmp_us["fp8_quantize"], 2)
    if qdq is not None:
        q_us = 1e3 * med["qdq_experts"]
        line["qdq_experts_us"] = round(q_us, 2)
        line["qdq_experts_gbs"] = round(qdq.bytes() / (q_us * 1e-6) / 1e9, 1)
        line["qdq_experts_frac_hbm"] = round(qdq.bytes() / (q_us * 1e-6) / 1e9 / hbm_peak, 4)
    return line


# ---------------------------------------------------------------- MoE expert FFN
def moe_flops(offsets, K_up, N_up, K_dn, N_dn, k):
    """Effective FLOPs of the up and down grouped RAC linears (every expert's
    rows times N times K + n_sel)."""
    from precision_rl_rollout_nvfp4_b200 import binding as B
    T = int(offsets[-1])
    return 2.0 * T * (N_up * (K_up + B.rac_nsel(k, K_up)) + N_dn * (K_dn + B.rac_nsel(k, K_dn)))


def run_moe(args, rank, world, local_rank):
    """Grouped MoE expert FFN: one step = the up (K 2048 -> N 1024) and the
    down (K 1024 -> N 2048) grouped W4A4 + RAC linears over 64 experts, rows
    expert-contiguous (8192 tokens routed top-8 with Zipf(1.1) loads).  Each
    call runs, per expert, the quantizer, the channel selection, the W_sel
    quantization and the grouped tensor-core GEMM.  Expert weights are
    prepared once (weight_qdq over all experts, timed separately).  The
    step's inputs (402 MB) exceed L2, so no flush is needed between steps."""
    import torch
    import torch.distributed as dist

    from precision_rl_rollout_nvfp4_b200 import binding as B
    from precision_rl_rollout_nvfp4_b200 import synthetic as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = S.MOE
    k = args.k if args.k is not None else cfg["k"]
    inp = S.moe_inputs(cfg["T"], cfg["hidden"], cfg["inter"], cfg["E"], cfg["topk"], seed=replica_seed(rank))
    xu_host = inp["x_perm"].contiguous().pin_memory()
    xd_host = inp["x_down"].contiguous().pin_memory()
    xu, xd = xu_host.to(dev), xd_host.to(dev)
    wu, wd = inp["w_up"].to(dev), inp["w_down"].to(dev)
    off = torch.from_numpy(inp["offsets"]).to(dev)
    E, N_up, K_up = wu.shape
    _, N_dn, K_dn = wd.shape
    T = xu.shape[0]
    stream = torch.cuda.current_stream()

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    # weight preparation (per weight sync): Q(W) and the column maxima of
    # every expert (of W, or with --wsel fp4 of DQ(Q(W)))
    fp4 = args.wsel == "fp4"
    wu_out, wd_out = torch.empty_like(wu), torch.empty_like(wd)
    prep = {}
    for _ in range(3):              # the last pass reuses cached buffers
        torch.cuda.synchronize()
        a = ev()
        _, qu, cu = B.weight_qdq(wu, want_colamax=not fp4, out=wu_out)
        if fp4:
            cu = B.dq_colamax(qu, E)
        b = ev()
        _, qd, cd = B.weight_qdq(wd, want_colamax=not fp4, out=wd_out)
        if fp4:
            cd = B.dq_colamax(qd, E)
        c = ev()
        torch.cuda.synchronize()
        prep = {"weight_qdq_up": a.elapsed_time(b) * 1e3, "weight_qdq_down": b.elapsed_time(c) * 1e3}
    # W_sel source: the bf16 experts, or (None) their NVFP4 codes
    wu_sel, wd_sel = (None, None) if fp4 else (wu, wd)
    yu = torch.empty(T, N_up, dtype=torch.bfloat16, device=dev)
    yd = torch.empty(T, N_dn, dtype=torch.bfloat16, device=dev)

    def up(kk=k):
        B.moe_rac(xu, off, wu_sel, qu, cu, kk, out_dtype=torch.bfloat16, masks=False, out=yu)

    def down(kk=k):
        B.moe_rac(xd, off, wd_sel, qd, cd, kk, out_dtype=torch.bfloat16, masks=False, out=yd)

    def step():
        up()
        down()

    def plain():
        up(0.0)
        down(0.0)

    for _ in range(max(args.warmup, 1)):
        step()
        plain()
    torch.cuda.synchronize()
    if B.stream_status() != 0:
        raise RuntimeError("device error word set during warm-up")
    graphs = {}
    use_graph = not args.no_graph
    if use_graph:
        for name, fn in [("step", step), ("plain", plain), ("up", up), ("down", down)]:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs[name] = g
        torch.cuda.synchronize()
    fns = {"step": step, "plain": plain, "up": up, "down": down}

    def launch(name):
        if use_graph:
            graphs[name].replay()
        else:
            fns[name]()

    for _ in range(args.warmup):
        launch("step")
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        evs = []
        for _ in range(args.steps):
            a = ev()
            launch("step")
            evs.append((a, ev()))
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in evs)
    clock = clocks.summary()
    per = {n: [] for n in ("up", "down", "plain")}
    for _ in range(args.steps):
        for n in per:
            a = ev()
            launch(n)
            b = ev()
            torch.cuda.synchronize()
            per[n].append(a.elapsed_time(b))
    # end to end: both inputs from pinned host memory, the step's output back
    # (two buffer sets, copies overlapped with the neighbouring steps' compute)
    xu1, xd1 = torch.empty_like(xu), torch.empty_like(xd)
    yu1, yd1 = torch.empty_like(yu), torch.empty_like(yd)

    def step1():
        B.moe_rac(xu1, off, wu_sel, qu, cu, k, out_dtype=torch.bfloat16, masks=False, out=yu1)
        B.moe_rac(xd1, off, wd_sel, qd, cd, k, out_dtype=torch.bfloat16, masks=False, out=yd1)

    sets = [{"h2d": [(xu, xu_host), (xd, xd_host)], "d2h": [(torch.empty(T, N_dn, dtype=torch.bfloat16).pin_memory(), yd)],
             "step": step},
            {"h2d": [(xu1, xu_host), (xd1, xd_host)], "d2h": [(torch.empty(T, N_dn, dtype=torch.bfloat16).pin_memory(), yd1)],
             "step": step1}]
    e2e_ms = e2e_pipelined(sets, args.steps, max(args.warmup, 2))
    if B.stream_status() != 0:
        raise RuntimeError("device error word set during timing")
    total_ms, e2e_total = max_over_ranks([total_ms, e2e_ms], world, dev)

    flops = moe_flops(inp["offsets"], K_up, N_up, K_dn, N_dn, k)
    value = flops * world * args.steps / (total_ms * 1e-3) / 1e12
    med = {n: statistics.median(v) for n, v in per.items()}
    peaks, peak_kind = load_peaks()
    fp4_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * FP4_OVER_BF16
    fl_up = 2.0 * T * N_up * (K_up + B.rac_nsel(k, K_up))
    up_tf = fl_up / (med["up"] * 1e-3) / 1e12
    step_ms = total_ms / args.steps
    loads = [int(inp["offsets"][i + 1] - inp["offsets"][i]) for i in range(E)]
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s (effective 2MN(K+n_sel) per step)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1/ue4m3) x fp32 acc",
        "data": "synthetic, seeded: top-8 routing of 8192 tokens over 64 experts with Zipf(1.1) loads; X as the dense workload's, W = N(0, 0.02^2), bf16",
        "config": {"workload": MOE_WORKLOAD, "tokens": cfg["T"], "topk": cfg["topk"], "routed_rows": T, "experts": E,
                   "up": [K_up, N_up], "down": [K_dn, N_dn], "k_percent": k, "wsel": args.wsel,
                   "expert_rows_max": max(loads),
                   "expert_rows_min": min(loads), "y_dtype": "bf16", "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (402 MB per step)", "cuda_graph": use_graph},
        "per_call_us": {"up": round(1e3 * med["up"], 2), "down": round(1e3 * med["down"], 2),
                        **{n: round(v, 2) for n, v in prep.items()}},
        "plain_w4a4_step_us": round(1e3 * med["plain"], 2),
        "rac_overhead_pct": round(100 * (step_ms - med["plain"]) / med["plain"], 1),
        "roofline": {"kernel": "moe_grouped_w4a4_rac_gemm (up call: quantizer, selection and GEMM)",
                     "bound": "tensor", "achieved": round(up_tf, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(up_tf / fp4_peak, 4), "traffic": None,
                     "peak_source": f"{peak_kind}: bf16 sustained x {FP4_OVER_BF16:g} (FP4/BF16 nominal)"},
        "e2e": {"value": round(flops * world * args.steps / (e2e_total * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(2 * (xu.numel() + xd.numel())), "d2h_bytes_per_step": int(2 * yd.numel()),
                "ms_per_step": round(e2e_total / args.steps, 4),
                "pipelined": "2 buffer sets; H2D, compute and D2H on separate streams"},
        # per grouped call: group tiles, amax, quantize, score reduce, top-k,
        # residual gather, W_sel scale, W_sel gather, GEMM (one memset too)
        "gpu_launches": (9 if B.rac_nsel(k, K_up) else 6) * 2 * args.steps,
        "clocks": clock,
    }


def run_qat(args, rank, world, local_rank):
    """Trainer-side QAT step of one linear, forward and backward: Y = X' W'^T,
    dX = dY W', dW = dY^T X' with W' = bf16(DQ(Q(W))) (the library's
    weight_qdq, straight-through gradient) and, for the symmetric W4A4
    ablation, X' = bf16(DQ(Q(X))); the three bf16 GEMMs are torch's.  Each
    step (forward and backward) is replayed as one CUDA graph, so host-side
    autograd does not enter the device time.  Timed with the same step
    without fake quantization beside it; L2 flushed between steps."""
    import torch
    import torch.distributed as dist

    from precision_rl_rollout_nvfp4_b200 import binding as B
    from precision_rl_rollout_nvfp4_b200 import synthetic as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M, K, N, act = QAT_WORKLOADS[args.workload]
    seed = replica_seed(rank)
    x_host = S.activations(M, K, seed=seed).pin_memory()
    dy_host = (0.01 * torch.randn(M, N, generator=torch.Generator().manual_seed(seed))).to(torch.bfloat16).pin_memory()
    w = S.weights(N, K, seed=seed).to(dev).requires_grad_(True)
    x, dy = x_host.to(dev).requires_grad_(True), dy_host.to(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(qat=True, xs=None, dys=None):
        xs = x if xs is None else xs
        dys = dy if dys is None else dys
        xs.grad = None
        w.grad = None
        y = B.qat_linear(xs, w, act_quant=act) if qat else xs @ w.t()
        y.backward(dys)
        return y

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    def timed(fn, reps):
        ts = []
        for _ in range(reps):
            flush.zero_()
            a = ev()
            fn()
            b = ev()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return ts

    # warm-up on a side stream, then capture each step (autograd included)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(max(args.warmup, 3)):
            step()
            step(qat=False)
            B.fake_quant(w.detach())
    stream.wait_stream(side)
    torch.cuda.synchronize()
    if B.stream_status() != 0:
        raise RuntimeError("device error word set during warm-up")
    graphs = {}
    for name, fn in [("qat", step), ("plain", lambda: step(qat=False)), ("fq", lambda: B.fake_quant(w.detach()))]:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        graphs[name] = gr
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        qat_ms = timed(graphs["qat"].replay, args.steps)
        if world > 1:
            dist.barrier()
    clock = clocks.summary()
    total_ms = sum(qat_ms)
    plain_ms = timed(graphs["plain"].replay, args.steps)
    fq_ms = timed(graphs["fq"].replay, args.steps)
    # end to end: X and dY from pinned host memory, a 4-byte loss-like scalar back
    bufs = [(torch.empty_like(x), torch.empty_like(dy), torch.empty(1, dtype=torch.float32, device=dev))
            for _ in range(2)]

    def step_e2e(xb, dyb, out):
        xs = xb.requires_grad_(True)
        y = step(xs=xs, dys=dyb)
        out.copy_(y.detach().float().sum().reshape(1))

    sets = [{"h2d": [(xb.detach(), x_host), (dyb, dy_host)], "d2h": [(torch.empty(1).pin_memory(), out)],
             "step": (lambda xb=xb, dyb=dyb, out=out: step_e2e(xb, dyb, out))} for xb, dyb, out in bufs]
    e2e_ms = e2e_pipelined(sets, args.steps, max(args.warmup, 2))
    if B.stream_status() != 0:
        raise RuntimeError("device error word set during timing")
    total_ms, e2e_total = max_over_ranks([total_ms, e2e_ms], world, dev)
    flops = 6.0 * M * N * K
    value = flops * world * args.steps / (total_ms * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    med = {"qat_step": statistics.median(qat_ms), "plain_bf16_step": statistics.median(plain_ms),
           "fake_quant_w": statistics.median(fq_ms)}
    fq_bytes = 4.0 * N * K            # read W once, write W' once (algorithmic)
    fq_gbs = fq_bytes / (med["fake_quant_w"] * 1e-3) / 1e9
    return {
        "metric": "QAT linear step TFLOP/s (6MNK per forward + backward)", "value": round(value, 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 GEMMs (torch) + nvfp4 fake quantization (library)",
        "data": "synthetic (seeded channel-scaled heavy-tailed X, N(0,0.02) W, N(0,0.01) dY)",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N, "act_quant": act,
                   "parallelism": f"replicas x{world}", "l2": "flushed before every timed step (256 MiB write)",
                   "cuda_graph": True},
        "per_call_us": {k: round(1e3 * v, 2) for k, v in med.items()},
        "qdq_overhead_pct": round(100 * (med["qat_step"] - med["plain_bf16_step"]) / med["plain_bf16_step"], 1),
        "roofline": {"kernel": "fake_quant(W): amax pass + weight_qdq", "bound": "hbm", "achieved": round(fq_gbs, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(fq_gbs / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_source": f"{peak_kind}: hbm_gbs"},
        "e2e": {"value": round(flops * world * args.steps / (e2e_total * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(2 * (x.numel() + dy.numel())), "d2h_bytes_per_step": 4,
                "ms_per_step": round(e2e_total / args.steps, 4),
                "pipelined": "2 buffer sets; H2D, compute and D2H on separate streams"},
        # per step: fake quantization of W (2 launches) and, for W4A4, of X (2)
        "gpu_launches": (4 if act else 2) * args.steps,
        "clocks": clock,
    }


# ---------------------------------------------------------------- oracle (CPU)
_ORACLE_INPUTS = {}


def oracle_step_time(M, K, N, k, rows, seed=0, wsel="bf16", qdq_shapes=()):
    """One oracle step on a bounded sample of the workload: weight_qdq(W),
    then the RAC linear of the first `rows` rows of X taken as a batch of
    their own (their own amax, scores and mask), and weight_qdq of one expert
    of every stacked shape in `qdq_shapes`."""
    import numpy as np

    import oracle
    from precision_rl_rollout_nvfp4_b200 import synthetic as S
    key = (M, K, N, rows, seed, tuple(qdq_shapes))
    if key not in _ORACLE_INPUTS:
        x = S.bf16_bits(S.activations(rows, K, seed=seed))     # the first `rows` rows of X
        w = S.bf16_bits(S.weights(N, K, seed=seed))
        experts = [S.bf16_bits(S.weights(n, kk, seed, batch=1, stream=S.STREAM_W + 10 * i))[0]
                   for i, (n, kk) in enumerate(qdq_shapes)]
        _ORACLE_INPUTS[key] = (x, w, experts)
    x, w, experts = _ORACLE_INPUTS[key]
    t0 = time.perf_counter()
    wq = oracle.weight_qdq(w)
    r = oracle.rac_linear(x, w, k, wq=wq, wsel_source=wsel)
    for we in experts:
        oracle.weight_qdq(we)
    dt = time.perf_counter() - t0
    return dt, 2.0 * rows * N * (K + r["n_sel"]), np.asarray(r["y"]).shape


def oracle_sample_text(M, K, N, rows, qdq_shapes):
    t = (f"weight_qdq(W {N}x{K}) + the RAC linear of the first {rows} of {M} rows of X as a batch of "
         f"their own (own amax, scores and mask)")
    if qdq_shapes:
        t += " + weight_qdq of one expert of each stacked shape " + ", ".join(f"{n}x{kk}" for n, kk in qdq_shapes)
    return t + " (numpy oracle; fp64 product via BLAS)"


def oracle_qat_time(M, K, N, act, rows, seed=0):
    """Oracle QAT step (fake quantization of the whole W, and of X for the
    W4A4 ablation, then the fp64 forward and backward products) on the first
    `rows` rows of X and dY."""
    import torch

    from oracle import qat
    from precision_rl_rollout_nvfp4_b200 import synthetic as S
    x = S.bf16_bits(S.activations(M, K, seed=seed))[:rows]
    w = S.bf16_bits(S.weights(N, K, seed=seed))
    dy = (0.01 * torch.randn(M, N, generator=torch.Generator().manual_seed(seed))).to(torch.bfloat16)
    dy = dy.float().numpy()[:rows]
    t0 = time.perf_counter()
    qat.qat_linear(x, w, dy, act_quant=act)
    return time.perf_counter() - t0, 6.0 * rows * N * K


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


_MOE_SAMPLE = {}


def oracle_moe_time(k, n_experts=8, seed=0, wsel="bf16"):
    """Oracle up projection of the last n_experts experts (the smallest row
    groups) of the MoE workload: every step of the grouped RAC linear on those
    groups.  Returns (seconds, effective FLOPs, description)."""
    import oracle
    from precision_rl_rollout_nvfp4_b200 import synthetic as S
    cfg = S.MOE
    E = cfg["E"]
    e0 = E - n_experts
    if (n_experts, seed) not in _MOE_SAMPLE:
        inp = S.moe_inputs(cfg["T"], cfg["hidden"], cfg["inter"], cfg["E"], cfg["topk"], seed=seed)
        off = inp["offsets"]
        r0, r1 = int(off[e0]), int(off[E])
        _MOE_SAMPLE[(n_experts, seed)] = (S.bf16_bits(inp["x_perm"][r0:r1]), S.bf16_bits(inp["w_up"][e0:E]),
                                          off[e0:] - r0, r0, r1)
    x, w, sub_off, r0, r1 = _MOE_SAMPLE[(n_experts, seed)]
    t0 = time.perf_counter()
    oracle.moe_rac(x, sub_off, w, k, wsel_source=wsel)
    dt = time.perf_counter() - t0
    K, N = cfg["hidden"], cfg["inter"]
    n_sel = oracle.n_selected(k, K)
    return dt, 2.0 * (r1 - r0) * N * (K + n_sel), f"up projection of experts {e0}..{E - 1} ({r1 - r0} rows)"


def cpu_baseline(args, budget_s=12.0):
    if args.workload in QAT_WORKLOADS:
        M, K, N, act = QAT_WORKLOADS[args.workload]
        rows = min(M, ORACLE_SAMPLE_ROWS)
        t, flops, n = 0.0, 0.0, 0
        while (t < budget_s and n < 8) or n == 0:
            dt, f = oracle_qat_time(M, K, N, act, rows)
            t, flops, n = t + dt, flops + f, n + 1
        return {"value": round(flops / t / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                "sample": f"{n} oracle QAT step(s): fake quantization of W {N}x{K} and the fp64 forward and "
                          f"backward on the first {rows} of {M} rows (numpy; products via BLAS)"}
    if args.workload == MOE_WORKLOAD:
        k = args.k if args.k is not None else 50.0
        t, flops, n, desc = 0.0, 0.0, 0, ""
        while (t < budget_s and n < 4) or n == 0:
            dt, f, desc = oracle_moe_time(k, wsel=args.wsel)
            t, flops, n = t + dt, flops + f, n + 1
        return {"value": round(flops / t / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                "sample": f"{n} oracle run(s) of the grouped RAC linear: {desc} (numpy; fp64 product via BLAS)"}
    M, K, N, k = WORKLOADS[args.workload]
    k = args.k if args.k is not None else k
    rows = min(M, ORACLE_SAMPLE_ROWS)
    shapes = QDQ_EXPERTS[args.workload][1] if args.workload in QDQ_EXPERTS else ()
    t, flops, n = 0.0, 0.0, 0
    while t < budget_s or n == 0:
        dt, f, _ = oracle_step_time(M, K, N, k, rows, wsel=args.wsel, qdq_shapes=shapes)
        t += dt
        flops += f
        n += 1
        if n >= 8:
            break
    return {"value": round(flops / t / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} oracle step(s) of " + oracle_sample_text(M, K, N, rows, shapes)}


def run_reference(args):
    if args.workload in QAT_WORKLOADS:
        M, K, N, act = QAT_WORKLOADS[args.workload]
        rows = min(M, ORACLE_SAMPLE_ROWS)
        for _ in range(args.warmup):
            oracle_qat_time(M, K, N, act, rows)
        t, flops = 0.0, 0.0
        for _ in range(args.steps):
            dt, f = oracle_qat_time(M, K, N, act, rows)
            t, flops = t + dt, flops + f
        value = flops / t / 1e12
        return {"impl": "reference", "metric": "QAT linear step TFLOP/s (6MNK per forward + backward)",
                "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantizer steps, f64 products",
                "data": "synthetic", "config": {"workload": args.workload, "M": M, "K": K, "N": N, "act_quant": act},
                "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                                 "sample": f"the first {rows} of {M} rows per step (numpy oracle)"},
                "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if args.workload == MOE_WORKLOAD:
        k = args.k if args.k is not None else 50.0
        for _ in range(args.warmup):
            oracle_moe_time(k, wsel=args.wsel)
        t, flops, desc = 0.0, 0.0, ""
        for _ in range(args.steps):
            dt, f, desc = oracle_moe_time(k, wsel=args.wsel)
            t, flops = t + dt, flops + f
        value = flops / t / 1e12
        return {"impl": "reference", "metric": METRIC, "value": round(value, 6),
                "unit": "TFLOP/s (effective 2MN(K+n_sel) per step)", "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantizer steps, f64 product",
                "data": "synthetic", "config": {"workload": MOE_WORKLOAD, "k_percent": k},
                "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                                 "sample": f"{desc} per step (numpy oracle; fp64 product via BLAS)"},
                "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    M, K, N, k = WORKLOADS[args.workload]
    k = args.k if args.k is not None else k
    rows = min(M, ORACLE_SAMPLE_ROWS)
    shapes = QDQ_EXPERTS[args.workload][1] if args.workload in QDQ_EXPERTS else ()
    for _ in range(args.warmup):
        oracle_step_time(M, K, N, k, rows, wsel=args.wsel, qdq_shapes=shapes)
    t, flops = 0.0, 0.0
    for _ in range(args.steps):
        dt, f, _ = oracle_step_time(M, K, N, k, rows, wsel=args.wsel, qdq_shapes=shapes)
        t += dt
        flops += f
    value = flops / t / 1e12
    cores = blas_threads()
    sample = oracle_sample_text(M, K, N, rows, shapes) + " per step"
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
        runner = run_moe if args.workload == MOE_WORKLOAD else run_qat if args.workload in QAT_WORKLOADS else run_ours
        line = runner(args, rank, world, local_rank)
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
