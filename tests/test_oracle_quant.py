"""Pins of the oracle's tensor Q / DQ against worked examples and invariants."""
import numpy as np
import pytest

import oracle
from oracle import formats as F
from oracle.nvfp4 import F32


def test_hand_worked_block(golden):
    rows = golden("quant_block_example.txt")
    x = np.zeros(32, F32)
    x[:16] = [float(r[0]) for r in rows]
    x[16] = 2688.0
    codes, scales, s_t = oracle.quantize_tensor(x[None, :])
    assert s_t == 1.0
    assert scales[0].tolist() == [0x30, 0x7E]
    assert codes[0, :16].tolist() == [int(r[2]) for r in rows]
    # x / s_dec column of the fixture
    assert np.array_equal(np.float32([float(r[1]) for r in rows]), x[:16] / F32(0.5))
    assert codes[0, 16] == 7 and codes[0, 17:].tolist() == [0] * 15


def test_round_trip_every_code_every_scale():
    """x built as E2M1(c) x E4M3(sb) with a block maximum 6 x E4M3(sb) and
    s_t = 1 recovers c and sb for all 16 codes and all 126 positive scales."""
    blocks = []
    expect_codes, expect_scales = [], []
    for sb in range(1, 0x7F):
        sbv = F.E4M3_POSITIVE[sb]
        blk = np.zeros(16)
        blk[0] = 6 * sbv
        blk[1:] = [oracle.e2m1_decode(c) * sbv for c in range(15)] + []
        cs = [7] + list(range(15))
        blocks.append(blk)
        expect_codes.append(cs)
        expect_scales.append(sb)
        blk2 = np.zeros(16)
        blk2[0] = -6 * sbv
        blk2[1] = oracle.e2m1_decode(15) * sbv
        blocks.append(blk2)
        expect_codes.append([15, 15] + [0] * 14)
        expect_scales.append(sb)
    x = np.concatenate(blocks + [np.array([2688.0] + [0.0] * 15)]).astype(F32)[None, :]
    codes, scales, s_t = oracle.quantize_tensor(x)
    assert s_t == 1.0
    n = len(expect_scales)
    assert np.array_equal(scales[0, :n], np.array(expect_scales, np.uint8))
    assert np.array_equal(codes[0, : 16 * n].reshape(n, 16), np.array(expect_codes, np.uint8))
    dq = oracle.dequantize(codes, scales, s_t)
    assert np.array_equal(dq, x)      # every value was on the grid


def _heavy(M, K, seed):
    rng = np.random.default_rng(seed)
    s = np.exp(rng.standard_normal(K)) * np.where(rng.random(K) < 0.02, 20, 1)
    return (rng.standard_normal((M, K)) * s).astype(F32)


def test_idempotent_with_fixed_tensor_scale():
    x = _heavy(64, 256, 3)
    codes, scales, s_t = oracle.quantize_tensor(x)
    dq = oracle.dequantize(codes, scales, s_t)
    c2, s2 = oracle.quantize(dq, s_t)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    assert np.array_equal(oracle.dequantize(c2, s2, s_t), dq)


def test_idempotent_with_recomputed_tensor_scale():
    x = _heavy(64, 256, 4)
    codes, scales, s_t = oracle.quantize_tensor(x)
    dq = oracle.dequantize(codes, scales, s_t)
    c2, s2, st2 = oracle.quantize_tensor(dq)
    assert abs(float(st2) - float(s_t)) <= 2 * np.spacing(np.float32(s_t))
    assert np.array_equal(s2, scales)
    assert np.mean(c2 == codes) > 0.999


def test_error_bound_half_largest_gap():
    """|x - DQ| <= 1 x s_dec: the largest gap of the E2M1 grid is 2 (4 -> 6)
    and an element above 6 s_dec exceeds it by at most 6 / 16 of s_dec."""
    x = _heavy(128, 512, 5)
    codes, scales, s_t = oracle.quantize_tensor(x)
    dq = oracle.dequantize(codes, scales, s_t)
    s_dec = np.repeat((F.e4m3_decode(scales) * float(s_t)), 16, axis=1)
    err = np.abs(x.astype(np.float64) - dq)
    assert np.all(err <= s_dec * (1 + 1e-6) + 1e-45)
    # and the block maximum always maps to the top code (x / s_dec in [5.6, 6.4])
    blk_max_code = (codes.reshape(128, 32, 16) & 7).max(axis=2)
    nz = scales > 0
    assert np.all(blk_max_code[nz] == 7)


def test_zero_tensor_and_zero_blocks():
    x = np.zeros((3, 32), F32)
    x[1, 5] = -0.0
    x[2] = -0.0
    codes, scales, s_t = oracle.quantize_tensor(x)
    assert s_t == 0 and not scales.any()
    assert codes[0].tolist() == [0] * 32 and codes[2].tolist() == [8] * 32 and codes[1, 5] == 8
    y = np.zeros((1, 32), F32)
    y[0, 20] = 1.0
    y[0, 3] = -0.0
    c, s, st = oracle.quantize_tensor(y)
    assert s[0, 0] == 0 and c[0, 3] == 8 and s[0, 1] == 0x7E and c[0, 20] == 7


def test_signed_zero_round_trip():
    x = np.float32([[-1e-30] + [0.0] * 14 + [1.0]])
    c, s, st = oracle.quantize_tensor(x)
    assert c[0, 0] == 8
    dq = oracle.dequantize(c, s, st)
    assert np.signbit(dq[0, 0]) and dq[0, 0] == 0
