"""Seeded synthetic inputs shaped like the QUADS rollout workloads.

This module only draws random numbers; it holds none of the method's
arithmetic, and both the CUDA library's tests and the CPU oracle take their
inputs from it.  The pages' workloads (a 25B-parameter MoE with 2.8B active
parameters, GRPO rollouts on math and code tasks; QUADS technical summary,
section 4 "Experimentele Resultaten") are not available, so these generators
stand in for them:

* activations X = N(0, 1) * s_c with a per-channel scale s_c = exp(N(0, 1))
  and round(0.01 K) outlier channels scaled by 20 (heavy-tailed channels are
  what makes some channels "high-residual");
* weights W ~ N(0, 0.02^2);
* MoE routing: each token picks 8 of 64 experts without replacement with
  probabilities proportional to (e + 1)^-1.1 (Gumbel top-k), and rows are
  permuted so that each expert's rows are contiguous.

Everything is rounded to bf16 (nearest even) by torch.  Random streams:
numpy ``default_rng([seed, stream])`` with stream 0 = channel scales and
outliers, 1 = X, 2 = W, 3 = routing, 4 = the down-projection input X'.
"""
from __future__ import annotations

import numpy as np
import torch

STREAM_CHANNELS, STREAM_X, STREAM_W, STREAM_ROUTING, STREAM_X_DOWN = range(5)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, stream])


def to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (a view when possible)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def channel_scales(K: int, seed: int = 0, outlier_frac: float = 0.01,
                   outlier_gain: float = 20.0) -> np.ndarray:
    rng = _rng(seed, STREAM_CHANNELS)
    s = np.exp(rng.standard_normal(K))
    n_out = int(round(outlier_frac * K))
    if n_out:
        s[rng.choice(K, size=n_out, replace=False)] *= outlier_gain
    return s


def activations(M: int, K: int, seed: int = 0, stream: int = STREAM_X) -> torch.Tensor:
    """bf16 [M, K] channel-scaled heavy-tailed activations."""
    s = channel_scales(K, seed).astype(np.float32)
    x = _rng(seed, stream).standard_normal((M, K), dtype=np.float32)
    x *= s[None, :]
    return to_bf16(x)


def weights(N: int, K: int, seed: int = 0, std: float = 0.02, batch: int | None = None,
            stream: int = STREAM_W) -> torch.Tensor:
    """bf16 [N, K] (or [batch, N, K]) weights ~ N(0, std^2)."""
    shape = (N, K) if batch is None else (batch, N, K)
    w = _rng(seed, stream).standard_normal(shape, dtype=np.float32) * np.float32(std)
    return to_bf16(w)


def moe_routing(T: int, E: int = 64, topk: int = 8, zipf: float = 1.1, seed: int = 0):
    """Expert-contiguous routing of T tokens to topk of E experts.

    Returns (token_of_row int64 [T*topk], offsets int64 [E+1]): row r of the
    permuted activations is token token_of_row[r]; expert e owns rows
    offsets[e]:offsets[e+1].
    """
    rng = _rng(seed, STREAM_ROUTING)
    logp = -zipf * np.log(np.arange(1, E + 1, dtype=np.float64))
    g = logp[None, :] + rng.gumbel(size=(T, E))
    chosen = np.argsort(-g, axis=1, kind="stable")[:, :topk]          # [T, topk]
    tok = np.repeat(np.arange(T), topk)
    exp = chosen.reshape(-1)
    order = np.lexsort((tok, exp))                                     # by expert, then token
    counts = np.bincount(exp, minlength=E)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    return tok[order].astype(np.int64), offsets


def moe_inputs(T: int = 8192, hidden: int = 2048, inter: int = 1024, E: int = 64,
               topk: int = 8, seed: int = 0):
    """The MoE expert-FFN workload: permuted activations for the up
    projection [T*topk, hidden], a synthetic down-projection input
    [T*topk, inter] of the same distribution, expert weights and offsets."""
    tok, offsets = moe_routing(T, E, topk, seed=seed)
    x = activations(T, hidden, seed)
    x_perm = x[torch.from_numpy(tok)]
    x_down = activations(T * topk, inter, seed, stream=STREAM_X_DOWN)
    w_up = weights(inter, hidden, seed, batch=E)
    w_down = weights(hidden, inter, seed, batch=E, stream=STREAM_W + 10)
    return dict(x_perm=x_perm, x_down=x_down, w_up=w_up, w_down=w_down,
                offsets=offsets, token_of_row=tok)


# Workload shapes (M tokens, K in-features, N out-features).
SINGLE = dict(M=64, K=512, N=512, k=50.0)
DENSE = dict(M=4096, K=2048, N=2048, k_sweep=(0.0, 25.0, 50.0, 100.0))
MOE = dict(T=8192, hidden=2048, inter=1024, E=64, topk=8, k=50.0)
DECODE = dict(M=256, K=4096, N=11008, k=50.0)
PREFILL = dict(M=32768, K=4096, N=4096, k=50.0, qdq_experts=64)
