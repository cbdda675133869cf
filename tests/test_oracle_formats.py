"""Pins of the oracle's element formats against their definitions."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import formats as F


def closed_form_e2m1(code):
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def test_e2m1_table_matches_golden_and_bitfields(golden):
    rows = golden("e2m1_grid.txt")
    assert len(rows) == 16
    for code_s, val_s in rows:
        code, val = int(code_s), float(val_s)
        got = float(oracle.e2m1_decode(code))
        assert got == val and math.copysign(1, got) == math.copysign(1, val)
        assert closed_form_e2m1(code) == val


def test_e2m1_eight_levels_per_sign():
    # "only 8 positive representable levels per sign": 8 magnitudes incl. 0
    vals = oracle.e2m1_decode(np.arange(16))
    assert len(set(np.abs(vals).tolist())) == 8
    assert len(set(vals[:8].tolist())) == 8


def _exhaustive_nearest(table_vals, a):
    """Nearest entry by exhaustive search; ties to the even index."""
    a = np.minimum(a, table_vals[-1] + 1.0)   # beyond the top entry: saturate
    d = np.abs(a[:, None] - table_vals[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    even = cand & (np.arange(table_vals.size)[None, :] % 2 == 0)
    return np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))


def _probe_values(points, span=300, n_random=200000, seed=0):
    rng = np.random.default_rng(seed)
    pts = []
    for p in points:
        b = np.float32(p).view(np.uint32).astype(np.int64)
        pts.append((np.arange(b - span, b + span + 1) & 0xFFFFFFFF).astype(np.uint32).view(np.float32))
    rnd = rng.integers(0, 2**32, n_random, dtype=np.uint64).astype(np.uint32).view(np.float32)
    allv = np.concatenate(pts + [rnd])
    allv = allv[np.isfinite(allv)]
    return np.concatenate([allv, -allv, np.float32([0.0, -0.0, np.inf, -np.inf, 3e38])])


def test_e2m1_encode_exhaustive_nearest():
    grid = np.array([closed_form_e2m1(c) for c in range(8)])
    mids = (grid[1:] + grid[:-1]) / 2
    v = _probe_values(list(grid) + list(mids), span=400)
    got = oracle.e2m1_encode(v)
    a = np.abs(v.astype(np.float64))
    want_mag = _exhaustive_nearest(grid, np.where(np.isinf(a), 1e300, a))
    want = want_mag | np.where(np.signbit(v), 8, 0)
    assert np.array_equal(got, want.astype(np.uint8))


@pytest.mark.parametrize("x,code", [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4),
                                    (3.5, 6), (5.0, 6), (6.0, 7), (7.0, 7), (1e30, 7),
                                    (-0.1, 8), (-0.0, 8), (0.0, 0), (-5.0, 14), (-0.26, 9)])
def test_e2m1_ties_and_saturation(x, code):
    assert int(oracle.e2m1_encode(np.float32(x))) == code


def test_e4m3_anchors(golden):
    for code_s, val_s in golden("e4m3_anchors.txt"):
        assert float(oracle.e4m3_decode(int(code_s, 16))) == float(val_s)
    assert np.isnan(oracle.e4m3_decode(0x7F)) and np.isnan(oracle.e4m3_decode(0xFF))


def test_e4m3_positive_table_properties():
    v = F.E4M3_POSITIVE
    assert v.size == 127 and np.all(np.diff(v) > 0)
    assert v[0] == 0 and v[1] == 2.0 ** -9 and v[-1] == 448.0
    # subnormals are evenly spaced by 2^-9 and continue into the first binade
    assert np.allclose(np.diff(v[:9]), 2.0 ** -9)
    # within a binade the spacing is 1/8 of the binade's base
    for e in range(1, 16):
        b = v[8 * e: 8 * e + 8]
        if b.size == 8:
            assert np.allclose(np.diff(b), b[0] / 8)


def test_e4m3_encode_exhaustive_nearest():
    table = F.E4M3_POSITIVE
    mids = (table[1:] + table[:-1]) / 2
    v = _probe_values(list(table) + list(mids), span=64, n_random=100000)
    v = np.abs(v)
    v = v[np.isfinite(v)]
    got = oracle.e4m3_encode(v)
    want = _exhaustive_nearest(table, v.astype(np.float64))
    assert np.array_equal(got, want.astype(np.uint8))


@pytest.mark.parametrize("x,code", [(2.0 ** -10, 0x00), (3 * 2.0 ** -11, 0x01),
                                    (1.0625, 0x38), (1.1875, 0x3A), (448.0, 0x7E),
                                    (464.0, 0x7E), (1e30, 0x7E), (np.inf, 0x7E), (0.0, 0x00)])
def test_e4m3_ties_and_saturation(x, code):
    assert int(oracle.e4m3_encode(np.float32(x))) == code


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, 400000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f) & (np.abs(f) < 3.3e38)]
    # add exact ties
    tie = (rng.integers(0, 2**16, 1000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32).view(np.float32)
    f = np.concatenate([f, tie[np.isfinite(tie) & (np.abs(tie) < 3.3e38)]])
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(f), want)
    assert np.array_equal(oracle.bf16_to_f32(want), torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())
