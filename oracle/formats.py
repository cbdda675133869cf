"""Element and scale formats of NVFP4, written out from their definitions.

Test infrastructure: see the package header in ``oracle/__init__.py``.

* E2M1 is the FP4 element format: 1 sign bit (bit 3), 2 exponent bits with
  bias 1 and 1 mantissa bit.  Its magnitudes are {0, 0.5, 1, 1.5, 2, 3, 4, 6}:
  the coarse grid with "8 positive levels per sign" that the QUADS technical
  summary (gist.science, "Technische Samenvatting: QUADS", section 1
  "Probleemstelling") blames for the activation error; the AI-Wiki QUADS
  summary ("Key Contributions", Finding 2) calls it the E2M1 grid.
* E4M3 is the block-scale format of NVFP4 (1 sign, 4 exponent bits with
  bias 7, 3 mantissa bits, finite maximum 448, no infinities, 0x7F/0xFF are
  NaN).  The pages only say that NVFP4 "adjusts precision in small steps"
  (QUADS explained, arxivlens, "Detailed Explanation"); the block size 16, the
  E4M3 scale and the FP32 tensor scale come from the public NVFP4 definition.

Rounding: every encoder takes the nearest representable value; an exact
midpoint goes to the code whose lowest mantissa bit is 0 ("even code"), and
values beyond the largest finite magnitude saturate to it.
"""
from __future__ import annotations

import numpy as np

# E2M1 magnitude of magnitude-codes 0..7 (exponent field = code >> 1,
# mantissa bit = code & 1; exponent 0 is subnormal: value = mantissa * 0.5).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E4M3_MAX = 448.0
E4M3_MAX_CODE = 0x7E


def e2m1_decode(codes) -> np.ndarray:
    """E2M1 code (0..15) -> value as float64 (code 8 is -0.0)."""
    c = np.asarray(codes).astype(np.uint8)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def _nearest_even(table: np.ndarray, a: np.ndarray) -> np.ndarray:
    """Index of the entry of the ascending ``table`` nearest to ``a`` (>= 0).

    Exact midpoints go to the even index; beyond the last entry the last
    index is returned (saturation).  ``a`` is float64 holding fp32 values, so
    every distance below is computed exactly.
    """
    n = table.shape[0]
    hi = np.searchsorted(table, a, side="left")          # first entry >= a
    hi = np.minimum(hi, n - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = np.abs(a - table[lo])
    d_hi = np.abs(table[hi] - a)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    # at or beyond the largest entry the result saturates to it (distances
    # to far-away values are no longer exact in float64)
    return np.where(a >= table[-1], n - 1, np.where(pick_hi, hi, lo))


def e2m1_encode(v) -> np.ndarray:
    """fp32 value -> E2M1 code: nearest magnitude, midpoint to even code,
    saturating at 6; the sign bit is the sign bit of ``v`` (so a negative value
    that rounds to zero gives code 0x8, i.e. -0)."""
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v).astype(np.float64)
    mag = _nearest_even(E2M1_MAGNITUDES, a).astype(np.uint8)
    return np.where(np.signbit(v), mag | np.uint8(8), mag).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 code (0..255) -> value as float64, from the bit fields.
    Codes 0x7F and 0xFF decode to NaN."""
    c = np.asarray(codes).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return np.where(s == 1, -mag, mag)


# the 127 finite non-negative E4M3 values, ascending with the code
E4M3_POSITIVE = e4m3_decode(np.arange(E4M3_MAX_CODE + 1))


def e4m3_encode(s) -> np.ndarray:
    """fp32 value >= 0 -> E4M3 code: nearest finite value, midpoint to even
    code, saturating at 448 (code 0x7E).  Never produces a NaN code."""
    s = np.asarray(s, dtype=np.float32)
    if np.any(s < 0) or np.any(np.isnan(s)):
        raise ValueError("e4m3_encode expects non-negative non-NaN input")
    return _nearest_even(E4M3_POSITIVE, s.astype(np.float64)).astype(np.uint8)


def bf16_to_f32(u16) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 (exact)."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def f32_to_bf16(f) -> np.ndarray:
    """float32 -> bf16 bit pattern, nearest, ties to even mantissa.

    The two candidates are the fp32 value with its low 16 bits cleared (toward
    zero) and the next bf16 away from zero; the nearer one wins and a tie goes
    to the one whose lowest bf16 mantissa bit is 0.  Finite inputs whose
    magnitude is below the largest bf16 are assumed (true for every use here).
    """
    f = np.asarray(f, dtype=np.float32)
    bits = f.view(np.uint32)
    toward0 = bits & np.uint32(0xFFFF0000)
    away = toward0 + np.uint32(0x10000)
    a = np.abs(f.astype(np.float64))
    d0 = a - np.abs(toward0.view(np.float32).astype(np.float64))
    d1 = np.abs(away.view(np.float32).astype(np.float64)) - a
    even0 = ((toward0 >> np.uint32(16)) & np.uint32(1)) == 0
    pick_away = (d1 < d0) | ((d1 == d0) & ~even0)
    return (np.where(pick_away, away, toward0) >> np.uint32(16)).astype(np.uint16)
