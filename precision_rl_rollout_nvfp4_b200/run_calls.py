"""Run chosen library calls of one rollout workload a few times, untimed.

For profilers (ncu with -k / -s / -c): the calls are the steps of
RacLinearPlan on synthetic inputs of the workload's shape, issued directly
(no CUDA graph), so each launch appears on its own.

    python -m precision_rl_rollout_nvfp4_b200.run_calls --M 32768 --K 4096 --N 4096 \
        --calls prepare_weight,quantize,select,weight_select,gemm --reps 2
"""
from __future__ import annotations

import argparse


def main(argv=None):
    import torch

    from . import binding as B
    from . import synthetic as S

    p = argparse.ArgumentParser()
    p.add_argument("--M", type=int, default=32768)
    p.add_argument("--K", type=int, default=4096)
    p.add_argument("--N", type=int, default=4096)
    p.add_argument("--k", type=float, default=50.0)
    p.add_argument("--calls", default="prepare_weight,quantize,select,weight_select,gemm")
    p.add_argument("--reps", type=int, default=2)
    p.add_argument("--y-dtype", choices=["bf16", "fp32"], default="bf16")
    a = p.parse_args(argv)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    x = S.activations(a.M, a.K).to(dev)
    w = S.weights(a.N, a.K).to(dev)
    plan = B.RacLinearPlan(a.M, a.K, a.N, a.k, out_dtype=torch.bfloat16 if a.y_dtype == "bf16" else torch.float32,
                           device=dev).bind(x, w)
    fns = {"prepare_weight": plan.prepare_weight, "quantize": plan.quantize, "select": plan.select,
           "weight_select": plan.weight_select, "gemm": plan.gemm, "gemm_plain": lambda: plan.gemm(plain=True),
           "quantize_plain": lambda: plan.quantize(scores=False), "quantize_select": plan.quantize_select,
           "second_pass": plan.second_pass, "select_channels": plan.select_channels}
    calls = [c for c in a.calls.split(",") if c]
    # the steps depend on each other: one full pass first
    plan.prepare_weight()
    plan.quantize()
    plan.select()
    plan.weight_select()
    plan.gemm()
    for _ in range(a.reps):
        for c in calls:
            fns[c]()
    torch.cuda.synchronize()
    st = B.stream_status()
    if st != 0:
        raise SystemExit(f"device error word set: {st}")
    print(f"ok: {a.M}x{a.K}x{a.N} k={a.k} calls={calls} reps={a.reps}")


if __name__ == "__main__":
    main()
