"""Pins of the MXFP8 oracle (the FP8 comparator's operand format): closed
forms of the OCP microscaling definition, round trips, saturation, ties,
signed zeros, and an independent scalar restatement."""
import numpy as np
import pytest

from oracle import mxfp8 as mx
from oracle import scalar
from oracle.formats import e4m3_decode

F32 = np.float32


@pytest.mark.parametrize("k", [0, 5, -20, -100, 100])
def test_block_of_448_times_2k_has_scale_k(k):
    x = np.zeros((1, 32), F32)
    x[0, 0] = 448.0 * 2.0 ** k
    x[0, 1] = -1.0 * 2.0 ** k
    codes, scales = mx.quantize(x)
    assert scales[0, 0] == k + 127
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xB8      # 448, -1.0
    assert mx.dequantize(codes, scales)[0, 0] == 448.0 * 2.0 ** k


@pytest.mark.parametrize("k", [0, 7, -30])
def test_every_e4m3_code_round_trips(k):
    """x = E4M3dec(c) 2^k for all 127 finite magnitudes, in blocks whose
    maximum is 448 2^k, comes back as c."""
    mags = e4m3_decode(np.arange(0x7F)).astype(np.float64)
    vals = np.concatenate([mags, np.zeros(128 - 127)]) * 2.0 ** k
    x = vals.reshape(4, 32).astype(F32)
    x[:, 31] = 448.0 * 2.0 ** k
    codes, scales = mx.quantize(x)
    assert np.all(scales == k + 127)
    want = np.concatenate([np.arange(0x7F), [0]]).reshape(4, 32).astype(np.uint8)
    want[:, 31] = 0x7E
    assert np.array_equal(codes, want)


def test_saturation_and_ties():
    x = np.zeros((1, 32), F32)
    x[0, 0] = 500.0            # floor(log2 500) = 8: scale 2^0; 500 > 448 saturates
    x[0, 1] = 1.0625           # midpoint of 1.0 (0x38) and 1.125 (0x39): even code
    x[0, 2] = 1.1875           # midpoint of 1.125 (0x39) and 1.25 (0x3A): even code
    x[0, 3] = 2.0 ** -10       # midpoint of 0 and the smallest subnormal 2^-9: 0
    x[0, 4] = -(2.0 ** -11)    # rounds to zero from below: -0
    x[0, 5] = -0.0
    codes, scales = mx.quantize(x)
    assert scales[0, 0] == 127
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0x38 and codes[0, 2] == 0x3A
    assert codes[0, 3] == 0x00 and codes[0, 4] == 0x80 and codes[0, 5] == 0x80


def test_zero_block():
    x = np.zeros((2, 64), F32)
    x[1, 32:] = 3.0
    x[0, 7] = -0.0
    codes, scales = mx.quantize(x)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0
    assert codes[0, 7] == 0x80 and not codes[0, :7].any()
    assert scales[1, 1] == 1 - 8 + 127        # floor(log2 3) = 1


def test_scalar_restatement_agrees():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((6, 96)) * np.exp(3 * rng.standard_normal((6, 96)))).astype(F32)
    x[2, :32] *= 1e-30
    x[3, 40] = 0.0
    codes, scales = mx.quantize(x)
    sc, ss = scalar.mxfp8_quantize_rows(x.astype(np.float64).tolist())
    assert np.array_equal(codes, np.array(sc, np.uint8))
    assert np.array_equal(scales, np.array(ss, np.uint8))


def test_error_bound():
    """|x - DQ| <= half the element spacing at x: at most 2^(E - 4) for
    normal E4M3 values (3 mantissa bits) and 2^(E - 10) in the subnormal
    range, so always <= 2^-4 2^floor(log2 |x|) + 2^(E - 10); saturated
    elements (x above 448 2^E) move by less than 64 2^E."""
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((8, 128)) * 10.0).astype(F32)
    codes, scales = mx.quantize(x)
    dq = mx.dequantize(codes, scales)
    e = np.repeat(scales.astype(np.float64) - 127, 32, axis=1)
    a = np.abs(x.astype(np.float64))
    bound = np.where(a > 0, 2.0 ** (np.floor(np.log2(np.where(a > 0, a, 1))) - 4), 0) + 2.0 ** (e - 10)
    bound = np.where(a > 448 * 2.0 ** e, 64 * 2.0 ** e, bound)
    assert np.all(np.abs(dq - x) <= bound)


def test_gemm_matches_plain_loop():
    rng = np.random.default_rng(8)
    a = rng.standard_normal((3, 64)).astype(F32)
    b = rng.standard_normal((4, 64)).astype(F32)
    ac, asc = mx.quantize(a)
    bc, bsc = mx.quantize(b)
    y = mx.gemm_fp64(ac, asc, bc, bsc)
    for i in range(3):
        for j in range(4):
            acc = 0.0
            for k in range(64):
                acc += (e4m3_decode(ac[i, k]) * 2.0 ** (int(asc[i, k // 32]) - 127)
                        * e4m3_decode(bc[j, k]) * 2.0 ** (int(bsc[j, k // 32]) - 127))
            assert y[i, j] == pytest.approx(acc, rel=1e-12, abs=1e-300)
