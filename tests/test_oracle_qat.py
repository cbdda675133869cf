"""Pins of the oracle's trainer-side QAT linear (W4A16, and the symmetric
W4A4 ablation) with the straight-through gradient."""
import numpy as np
import pytest

import oracle
from oracle import qat
from oracle.formats import e2m1_decode, e4m3_decode, f32_to_bf16


def grid_tensor(rows, cols, rng):
    """A bf16 tensor that NVFP4 represents exactly with tensor scale 1: every
    16-block is E2M1 codes times one E4M3 value sbv, each block holds a
    magnitude-6 element (so its block scale comes back as sbv), and one block
    uses sbv = 448 (so amax = 2688 and s_t = 1).  Returns bf16 bits."""
    codes = rng.integers(0, 16, (rows, cols)).astype(np.uint8)
    codes[:, ::16] = np.where(rng.integers(0, 2, (rows, cols // 16)) == 1, 15, 7)   # +-6 in every block
    sb = rng.integers(0x18, 0x7F, (rows, cols // 16)).astype(np.uint8)              # 2^-6 .. 448
    sb[0, 0] = 0x7E                                                                  # 448
    vals = e2m1_decode(codes) * np.repeat(e4m3_decode(sb), 16, axis=1)              # exact
    bits = f32_to_bf16(vals.astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f32(bits).astype(np.float64), vals)      # bf16 holds them
    return bits


def test_grid_tensor_is_a_fixed_point_of_the_fake_quantizer():
    rng = np.random.default_rng(1)
    w = grid_tensor(48, 128, rng)
    assert np.array_equal(qat.fake_quant(w), w)


@pytest.mark.parametrize("act_quant", [False, True])
def test_qat_linear_on_grid_operands_is_the_plain_linear(act_quant):
    """With operands NVFP4 represents exactly, fake quantization is the
    identity, so the QAT forward is Y = X W^T and the straight-through
    backward is the textbook dX = dY W, dW = dY^T X."""
    rng = np.random.default_rng(2)
    M, K, N = 40, 64, 24
    x, w = grid_tensor(M, K, rng), grid_tensor(N, K, rng)
    dy = rng.standard_normal((M, N))
    r = qat.qat_linear(x, w, dy, act_quant=act_quant)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    wf = oracle.bf16_to_f32(w).astype(np.float64)
    # plain loops, not the oracle's matrix products
    y = np.array([[sum(xf[i, k] * wf[j, k] for k in range(K)) for j in range(N)] for i in range(M)])
    dx = np.array([[sum(dy[i, j] * wf[j, k] for j in range(N)) for k in range(K)] for i in range(M)])
    dw = np.array([[sum(dy[i, j] * xf[i, k] for i in range(M)) for k in range(K)] for j in range(N)])
    assert np.allclose(r["y"], y, rtol=1e-12, atol=0)
    assert np.allclose(r["dx"], dx, rtol=1e-12, atol=1e-300)
    assert np.allclose(r["dw"], dw, rtol=1e-12, atol=1e-300)


def test_w4a16_keeps_activations_and_quantizes_weights():
    rng = np.random.default_rng(3)
    x = f32_to_bf16(rng.standard_normal((16, 64)).astype(np.float32))
    w = f32_to_bf16((0.02 * rng.standard_normal((32, 64))).astype(np.float32))
    r = qat.qat_linear(x, w)
    assert np.array_equal(r["x_q"], x)                        # A16: activations untouched
    assert not np.array_equal(r["w_q"], w)                    # W4: weights moved to the grid


def test_symmetric_ablation_quantizes_activations_too():
    rng = np.random.default_rng(4)
    x = f32_to_bf16(rng.standard_normal((16, 64)).astype(np.float32))
    w = f32_to_bf16((0.02 * rng.standard_normal((32, 64))).astype(np.float32))
    a = qat.qat_linear(x, w)
    s = qat.qat_linear(x, w, act_quant=True)
    assert np.array_equal(s["w_q"], a["w_q"])
    assert not np.array_equal(s["x_q"], x)
    assert np.array_equal(s["x_q"], qat.fake_quant(x))
    # the gradient into the weights sees the fake-quantized activations
    dy = rng.standard_normal((16, 32))
    g = qat.qat_linear(x, w, dy, act_quant=True)
    assert not np.allclose(g["dw"], qat.qat_linear(x, w, dy)["dw"])
