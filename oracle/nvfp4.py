"""NVFP4 quantization (Q) and dequantization (DQ) of a 2-D tensor.

Test infrastructure: see the package header in ``oracle/__init__.py``.

The quantize-dequantize (QDQ) path is the one the QUADS technical summary
(gist.science, section 2.1 "Foutanalyse en Diagnose", bullet on weights) says
trainer and rollout share.  The pages give no formula; the steps below are the
reading this project adopts (plain NVFP4: the tensor's largest magnitude maps
to 6 x 448), with every step an fp32 operation rounded to nearest even:

    s_t   = RN(amax / 2688)                       tensor decode scale (fp32)
    d     = RN(6 * s_t)
    sb    = E4M3(RN(amax_b / d))                  per 16-element block b
    s_dec = RN(E4M3dec(sb) * s_t)
    code  = E2M1(RN(x / s_dec))                   signed zero of x if s_dec == 0
    DQ    = RN(RN(E2M1dec(code) * E4M3dec(sb)) * s_t)

If s_t == 0 (all-zero tensor) every scale is 0 and every code is the signed
zero of its element.  Blocks run along the last axis (K); a row whose length
is not a multiple of 16 is not accepted here (callers zero-pad).
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode

BLOCK = 16
TENSOR_SCALE_DIVISOR = np.float32(6.0 * 448.0)   # 2688: E2M1 max x E4M3 max
F32 = np.float32


def amax(x) -> np.float32:
    """Largest magnitude of ``x`` (exact); 0 for an empty tensor."""
    x = np.asarray(x, dtype=F32)
    return F32(np.max(np.abs(x))) if x.size else F32(0.0)


def tensor_scale(a) -> np.float32:
    """s_t = RN(amax / 2688) in fp32."""
    return F32(F32(a) / TENSOR_SCALE_DIVISOR)


def quantize(x, s_t):
    """Quantize fp32 ``x`` [R, C] (C % 16 == 0) with tensor decode scale
    ``s_t``.  Returns (codes uint8 [R, C], one E2M1 code per element;
    scales uint8 [R, C/16], one E4M3 code per block)."""
    x = np.asarray(x, dtype=F32)
    R, C = x.shape
    if C % BLOCK:
        raise ValueError("row length must be a multiple of 16")
    s_t = F32(s_t)
    xb = x.reshape(R, C // BLOCK, BLOCK)
    if s_t == 0:
        scales = np.zeros((R, C // BLOCK), np.uint8)
        codes = np.where(np.signbit(x), np.uint8(8), np.uint8(0)).astype(np.uint8)
        return codes, scales
    d = F32(F32(6.0) * s_t)
    amax_b = np.max(np.abs(xb), axis=2)                          # exact
    ratio = (amax_b / d).astype(F32)                             # RN fp32
    scales = e4m3_encode(ratio)
    s_dec = (e4m3_decode(scales).astype(F32) * s_t).astype(F32)  # RN fp32
    s_dec_b = np.broadcast_to(s_dec[:, :, None], xb.shape)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        q = np.where(s_dec_b > 0, xb / s_dec_b, np.copysign(F32(0.0), xb)).astype(F32)
    codes = e2m1_encode(q).reshape(R, C)
    return codes, scales


def dequantize(codes, scales, s_t):
    """DQ = RN(RN(E2M1dec(code) * E4M3dec(scale)) * s_t), fp32 [R, C]."""
    codes = np.asarray(codes, np.uint8)
    R, C = codes.shape
    sv = np.repeat(e4m3_decode(scales), BLOCK, axis=1)
    prod = (e2m1_decode(codes) * sv).astype(F32)    # exact: <= 6 significant bits
    return (prod * F32(s_t)).astype(F32)


def block_values(codes, scales):
    """E2M1dec(code) * E4M3dec(scale) per element, float64 (exact).  These are
    the operand values a block-scaled FP4 tensor-core product multiplies."""
    return e2m1_decode(codes) * np.repeat(e4m3_decode(scales), BLOCK, axis=1)


def quantize_tensor(x, amax_value=None):
    """Q of a whole tensor with its own s_t (from ``amax_value`` if given).
    Returns (codes, scales, s_t)."""
    x = np.asarray(x, dtype=F32)
    a = amax(x) if amax_value is None else F32(amax_value)
    s_t = tensor_scale(a)
    codes, scales = quantize(x, s_t)
    return codes, scales, s_t
