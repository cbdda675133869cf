"""Trainer-side quantization-aware training (QAT) of one linear layer.

Test infrastructure: see the package header in ``oracle/__init__.py``.

What the pages fix (QUADS technical summary, gist.science):
  * section 2.2 A "Asymmetrische Quantization-Aware Training": the trainer
    fake-quantizes the weights to NVFP4 (W4) and keeps the activations in
    BF16 (A16), so that its weight path matches the rollout engine's;
  * section 2.1, bullet on activations, and section 4 (ablation): symmetric
    W4A4 QAT, which fake-quantizes the activations on the trainer as well, is
    the comparison that mismatches more.
The pages do not say how the gradient crosses the fake quantizer.  The
reading adopted here is the straight-through estimator: the backward pass
treats bf16(DQ(Q(t))) as the identity, so with Y = X' W'^T

    dX = dY W'          (through X' = X, or X' = QDQ(X) for W4A4)
    dW = dY^T X'        (through W' = QDQ(W))

The fake quantizer is ``weight_qdq`` (one tensor scale per matrix); the
symmetric ablation applies the same function to the activations.  Products
are fp64 sums of the exact bf16 operand values.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_to_f32
from .rac import weight_qdq


def fake_quant(t_bf16):
    """bf16(DQ(Q(t))) of a bf16 [R, K] tensor with its own tensor scale, as bf16 bits."""
    return weight_qdq(t_bf16)["w_out"]


def qat_linear(x_bf16, w_bf16, dy=None, act_quant=False):
    """Forward (and, when ``dy`` [M, N] is given, backward) of the QAT linear
    Y = X' W'^T.  W' = fake_quant(W) always (W4A16); X' = fake_quant(X) only
    for the symmetric W4A4 ablation (``act_quant``).  Returns dict(w_q, x_q,
    y, and dx, dw when dy is given); w_q and x_q are bf16 bits, the rest fp64."""
    w_q = fake_quant(w_bf16)
    x_q = fake_quant(x_bf16) if act_quant else np.asarray(x_bf16, np.uint16)
    xf = bf16_to_f32(x_q).astype(np.float64)
    wf = bf16_to_f32(w_q).astype(np.float64)
    out = dict(w_q=w_q, x_q=x_q, y=xf @ wf.T)
    if dy is not None:
        g = np.asarray(dy, np.float64)
        out["dx"] = g @ wf
        out["dw"] = g.T @ xf
    return out
