"""Residual Activation Compensation (RAC) and the W4A4 / W4A16 products.

Test infrastructure: see the package header in ``oracle/__init__.py``.

What the pages fix (QUADS technical summary, gist.science, section 2.2 B
"Residual Activation Compensatie (Rollout-zijde)"):
  * the rollout engine finds the "high-residual" channels, where the FP4
    quantization error is largest;
  * a second-pass quantization is applied to those channels and the residual
    correction term (Delta X_q) is added to the quantized output;
  * a binary channel mask selects the top k% of channels (50% is the example)
    by residual magnitude;
  * the aim is a rollout output closer to the BF16 reference.
The AI-Wiki QUADS summary ("Methodology") words it as adding the quantized
activation errors back before the native W4A4 GEMMs.  Both readings are the
same product:

    Y = DQ(Q(X)) DQ(Q(W))^T + DQ(Q(dX_sel)) DQ(Q(W_sel))^T

which is what this module computes.  Readings adopted where the pages are
silent (each is listed because the pages leave it open):
  * dX = RN(X - DQ(Q(X))) in fp32, never rounded to bf16;
  * score_j = sum over tokens of |dX_ij| in fp64, in a fixed order: rows in
    consecutive chunks of 128 (from row 0), each chunk summed from 0.0 in row
    order, then the chunk sums added from 0.0 in chunk order (one fixed
    order, so that the ranking and the mask are reproducible bit for bit);
  * n_sel = floor(k * K / 100) with k taken exactly;
  * the n_sel largest scores win, ties to the lower channel index, and sel is
    listed in ascending channel order;
  * dX_sel = dX[:, sel] gets its own tensor scale from its own amax; W_sel =
    W[:, sel] is re-quantized from bf16 W with its own tensor scale; blocks of
    16 run over the gathered positions and the last block is zero-padded.
"""
from __future__ import annotations

from fractions import Fraction
import math

import numpy as np

from .formats import bf16_to_f32, f32_to_bf16
from .nvfp4 import (BLOCK, F32, amax, block_values, dequantize, quantize,
                    tensor_scale)

SCORE_CHUNK = 128


def n_selected(k_percent, K: int) -> int:
    """n_sel = floor(k * K / 100), with the float k taken as its exact value."""
    k = Fraction(float(np.float32(k_percent)))
    if k < 0 or k > 100:
        raise ValueError("k must be in [0, 100]")
    return math.floor(k * K / 100)


def residual(x, codes, scales, s_t):
    """dX = RN(x - DQ(Q(x))) in fp32."""
    x = np.asarray(x, F32)
    return (x - dequantize(codes, scales, s_t)).astype(F32)


def channel_score(dx):
    """score_j (fp64, fixed order) and colamax_j = max_i |dX_ij| (fp32).
    Order: rows in chunks of 128 from row 0; a chunk is summed from 0.0 row
    by row in row order; the chunk sums are added from 0.0 in chunk order.
    Every addition is one fp64 operation rounded to nearest even."""
    a = np.abs(np.asarray(dx, F32))
    M, K = a.shape
    score = np.zeros(K, np.float64)
    for c0 in range(0, M, SCORE_CHUNK):
        part = np.zeros(K, np.float64)
        for r in range(c0, min(c0 + SCORE_CHUNK, M)):
            part = part + a[r].astype(np.float64)
        score = score + part
    colamax = a.max(axis=0) if M else np.zeros(K, F32)
    return score, colamax.astype(F32)


def select_channels(score, n_sel: int):
    """Top-n_sel channels by score, ties to the lower index.
    Returns (sel int32 ascending, mask uint8 [K])."""
    score = np.asarray(score, np.float64)
    K = score.shape[0]
    idx = np.arange(K)
    order = np.lexsort((idx, -score))        # score descending, then index
    sel = np.sort(order[:n_sel]).astype(np.int32)
    mask = np.zeros(K, np.uint8)
    mask[sel] = 1
    return sel, mask


def padded_width(n_sel: int, multiple: int = 64) -> int:
    """Gathered operand width: n_sel rounded up to a whole number of 64-wide
    K steps (the zero padding contributes exactly 0 to the product)."""
    return -(-n_sel // multiple) * multiple


def gather_quantize(src, sel, width: int, amax_value):
    """Second-pass quantization of src[:, sel] zero-padded to ``width``
    columns, with tensor scale RN(amax_value / 2688)."""
    src = np.asarray(src, F32)
    g = np.zeros((src.shape[0], width), F32)
    g[:, : len(sel)] = src[:, sel]
    s_t = tensor_scale(amax_value)
    codes, scales = quantize(g, s_t)
    return codes, scales, s_t


def column_amax(w):
    """colamax_j = max_n |W_nj| (fp32, exact)."""
    w = np.abs(np.asarray(w, F32))
    return w.max(axis=0) if w.shape[0] else np.zeros(w.shape[1], F32)


def weight_sel_from_fp4(w_codes, w_scales, w_st, sel, width: int):
    """Variant of the weight-side second pass (not the pages' reading; an
    option for rollouts that keep only Q(W)): W_sel is re-quantized from the
    trainer's NVFP4 weights, DQ(Q(W))[:, sel] in fp32, zero-padded to
    ``width``, with tensor scale RN(max over the selected columns of
    max_n |DQ(Q(W))_nj| / 2688).  Returns (codes, scales, s_t)."""
    dq = dequantize(w_codes, w_scales, w_st)
    a = column_amax(dq)[np.asarray(sel, np.int64)].max() if len(sel) else F32(0.0)
    return gather_quantize(dq, sel, width, a)


def gemm_fp64(a_codes, a_scales, a_st, b_codes, b_scales, b_st, rows=None):
    """Y = s_ta * s_tb * sum_k a_ik b_jk in fp64, a and b the exact block
    values E2M1dec * E4M3dec.  ``rows`` restricts Y to those rows of A."""
    if rows is not None:
        a_codes, a_scales = a_codes[rows], a_scales[rows]
    A = block_values(a_codes, a_scales)
    B = block_values(b_codes, b_scales)
    return (float(a_st) * float(b_st)) * (A @ B.T)


def quantize_activations(x_bf16):
    """Q(X) of bf16 activations with their own tensor scale, plus dX, the
    channel scores and the per-channel residual maxima."""
    x = bf16_to_f32(x_bf16)
    a = amax(x)
    s_t = tensor_scale(a)
    codes, scales = quantize(x, s_t)
    dx = residual(x, codes, scales, s_t)
    score, colamax = channel_score(dx)
    return dict(amax=a, s_t=s_t, codes=codes, scales=scales, dx=dx,
                score=score, res_colamax=colamax)


def weight_qdq(w_bf16):
    """Trainer-side W4A16 fake quantization of one bf16 weight [N, K]:
    W' = bf16_RNE(DQ(Q(W))) with the matrix's own tensor scale.  Also returns
    Q(W) and colamax_W, which the rollout side reuses.  (QUADS technical
    summary, section 2.2 A "Asymmetrische Quantization-Aware Training":
    weights are fake-quantized to NVFP4, activations stay BF16.)"""
    w = bf16_to_f32(w_bf16)
    a = amax(w)
    s_t = tensor_scale(a)
    codes, scales = quantize(w, s_t)
    w_out = f32_to_bf16(dequantize(codes, scales, s_t))
    return dict(w_out=w_out, codes=codes, scales=scales, s_t=s_t, amax=a,
                colamax=column_amax(w))


def rac_linear(x_bf16, w_bf16, k_percent, rows=None, wq=None, wsel_source="bf16", sel=None):
    """One rollout linear Y = X W^T in NVFP4 W4A4 with RAC.

    ``rows`` restricts the fp64 products to a subset of output rows (all
    quantities that depend on every token, such as the scores and the mask,
    are still computed from all rows).  ``wq`` may pass a precomputed
    ``weight_qdq(w_bf16)``.  ``wsel_source="fp4"`` takes W_sel from Q(W)
    (``weight_sel_from_fp4``) instead of bf16 W.  ``sel`` (ascending channel
    indices) replaces the top-k% selection of this X by a mask kept from an
    earlier call (the mask-reuse variant); everything else (Q(X), dX, the
    residual tensor scale over sel, both second passes) is this call's.
    Returns every intermediate."""
    qa = quantize_activations(x_bf16)
    M, K = qa["codes"].shape
    wq = weight_qdq(w_bf16) if wq is None else wq
    if sel is None:
        n_sel = n_selected(k_percent, K)
        sel, mask = select_channels(qa["score"], n_sel)
    else:
        sel = np.asarray(sel, np.int32)
        n_sel = len(sel)
        mask = np.zeros(K, np.uint8)
        mask[sel] = 1
    width = padded_width(n_sel)
    out = dict(qa)
    out.update(n_sel=n_sel, sel=sel, mask=mask, width=width, wq=wq)
    y_plain = gemm_fp64(qa["codes"], qa["scales"], qa["s_t"],
                        wq["codes"], wq["scales"], wq["s_t"], rows)
    out["y_plain"] = y_plain
    if n_sel == 0:
        out.update(r_codes=np.zeros((M, 0), np.uint8), r_scales=np.zeros((M, 0), np.uint8),
                   r_st=F32(0.0), ws_codes=None, ws_scales=None, ws_st=F32(0.0),
                   y=y_plain.copy())
        return out
    r_amax = qa["res_colamax"][sel].max()
    r_codes, r_scales, r_st = gather_quantize(qa["dx"], sel, width, r_amax)
    if wsel_source == "fp4":
        ws_codes, ws_scales, ws_st = weight_sel_from_fp4(wq["codes"], wq["scales"], wq["s_t"], sel, width)
        ws_amax = column_amax(dequantize(wq["codes"], wq["scales"], wq["s_t"]))[sel].max()
    else:
        w = bf16_to_f32(w_bf16)
        ws_amax = wq["colamax"][sel].max()
        ws_codes, ws_scales, ws_st = gather_quantize(w, sel, width, ws_amax)
    y_corr = gemm_fp64(r_codes, r_scales, r_st, ws_codes, ws_scales, ws_st, rows)
    out.update(r_codes=r_codes, r_scales=r_scales, r_st=r_st, r_amax=r_amax,
               ws_codes=ws_codes, ws_scales=ws_scales, ws_st=ws_st,
               ws_amax=ws_amax, y=y_plain + y_corr)
    return out


def moe_rac(x_perm_bf16, offsets, w_bf16, k_percent, wq=None, wsel_source="bf16"):
    """Grouped expert linears: rows offsets[e]:offsets[e+1] of the
    expert-contiguous activations go through expert e's own RAC linear (own
    amax, scores, mask and residual scale).  An empty group produces no rows;
    its mask is that of an all-zero score (the first n_sel channels).
    ``wsel_source`` is passed to ``rac_linear``.  Returns (y [T, N] fp64, masks [E, K], per-expert results)."""
    E, N, K = w_bf16.shape
    T = x_perm_bf16.shape[0]
    y = np.zeros((T, N), np.float64)
    masks = np.zeros((E, K), np.uint8)
    per = []
    n_sel = n_selected(k_percent, K)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        wqe = weight_qdq(w_bf16[e]) if wq is None else wq[e]
        if r1 == r0:
            sel, mask = select_channels(np.zeros(K), n_sel)
            masks[e] = mask
            per.append(None)
            continue
        res = rac_linear(x_perm_bf16[r0:r1], w_bf16[e], k_percent, wq=wqe, wsel_source=wsel_source)
        y[r0:r1] = res["y"]
        masks[e] = res["mask"]
        per.append(res)
    return y, masks, per
