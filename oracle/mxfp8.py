"""MXFP8: E4M3 elements with one power-of-two (UE8M0) scale per 32 elements.

Test infrastructure: see the package header in ``oracle/__init__.py``.

The pages compare NVFP4 rollout against FP8 rollout (QUADS technical summary,
gist.science, section 1 "Probleemstelling": NVFP4 offers about twice the GEMM
throughput of FP8; section 4: about 16 % rollout speed-up over FP8) but do
not say which FP8 scheme.  The reading adopted for the FP8 comparator is the
block-scaled FP8 that Blackwell's tensor cores run natively: the OCP
microscaling format MXFP8 with E4M3 elements and blocks of 32 consecutive
elements along K sharing one UE8M0 scale.  Per block b (the OCP MX
definition, with the element conversion saturating like the NVFP4 side):

    E      = floor(log2(amax_b)) - 8            (8 = exponent of E4M3's 448),
             clamped to [-127, 127]; E = -127 for an all-zero block
    scale  = UE8M0 code E + 127, value 2^E
    code   = E4M3 of x / 2^E, nearest, ties to the even code, saturating at
             448, the sign bit from x (so -0 and values that round to 0 from
             below keep the sign)
    DQ     = E4M3dec(code) * 2^E                (exact)

A product of two MXFP8 operands is the fp64 sum of exact block values.
"""
from __future__ import annotations

import numpy as np

from .formats import e4m3_decode, e4m3_encode

MX_BLOCK = 32
E4M3_EMAX = 8            # 448 = 1.75 * 2^8
UE8M0_BIAS = 127


def _floor_log2(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for finite a > 0, exact (frexp: a = m 2^e, m in [0.5, 1))."""
    _, e = np.frexp(np.asarray(a, np.float64))
    return e.astype(np.int64) - 1


def block_exponents(x) -> np.ndarray:
    """E per 32-element block of fp32 x [R, C] (C % 32 == 0), int64 [R, C/32]."""
    x = np.asarray(x, np.float32)
    R, C = x.shape
    if C % MX_BLOCK:
        raise ValueError("row length must be a multiple of 32")
    amax_b = np.max(np.abs(x).reshape(R, C // MX_BLOCK, MX_BLOCK), axis=2).astype(np.float64)
    e = np.full(amax_b.shape, -UE8M0_BIAS, np.int64)
    nz = amax_b > 0
    e[nz] = _floor_log2(amax_b[nz]) - E4M3_EMAX
    return np.clip(e, -UE8M0_BIAS, UE8M0_BIAS)


def e4m3_encode_signed(v) -> np.ndarray:
    """fp32 v -> signed E4M3 code (bit 7 = sign of v), nearest magnitude,
    ties to the even code, saturating at 448."""
    v = np.asarray(v, np.float32)
    mag = e4m3_encode(np.abs(v))
    return np.where(np.signbit(v), mag | np.uint8(0x80), mag).astype(np.uint8)


def quantize(x):
    """MXFP8 of fp32 x [R, C]: (codes uint8 [R, C], scales uint8 [R, C/32])."""
    x = np.asarray(x, np.float32)
    R, C = x.shape
    e = block_exponents(x)
    # x / 2^E: division by a power of two, exact in float64 and then exactly
    # the value the E4M3 rounding sees
    q = x.astype(np.float64) / np.repeat(np.exp2(e.astype(np.float64)), MX_BLOCK, axis=1)
    codes = e4m3_encode_signed_f64(q)
    return codes, (e + UE8M0_BIAS).astype(np.uint8)


def e4m3_encode_signed_f64(q) -> np.ndarray:
    """Signed E4M3 code of float64 values that are fp32 values scaled by a
    power of two (so nearest-even rounding on them is exact)."""
    q = np.asarray(q, np.float64)
    a = np.minimum(np.abs(q), 1e30)
    # e4m3_encode expects fp32; magnitudes below 2^-149 round to code 0 anyway
    a32 = np.where(a < 2.0 ** -126, 0.0, a).astype(np.float32)
    tiny = (a < 2.0 ** -126) & (a > 0)
    mag = e4m3_encode(a32)
    mag = np.where(tiny, np.uint8(0), mag)
    return np.where(np.signbit(q), mag | np.uint8(0x80), mag).astype(np.uint8)


def block_values(codes, scales):
    """E4M3dec(code) * 2^(scale - 127) per element, float64 (exact)."""
    codes = np.asarray(codes, np.uint8)
    e = np.asarray(scales, np.int64) - UE8M0_BIAS
    return e4m3_decode(codes) * np.repeat(np.exp2(e.astype(np.float64)), MX_BLOCK, axis=1)


def dequantize(codes, scales):
    return block_values(codes, scales)


def gemm_fp64(a_codes, a_scales, b_codes, b_scales, rows=None):
    """Y = A B^T in fp64 with A, B the exact MXFP8 block values."""
    if rows is not None:
        a_codes, a_scales = a_codes[rows], a_scales[rows]
    return block_values(a_codes, a_scales) @ block_values(b_codes, b_scales).T
