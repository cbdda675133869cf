"""The tcgen05 block-scaled FP4 GEMM and the whole RAC linear through the C
ABI against the oracle's fp64 product of the same dequantized operands."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import REL_TOL, bits, need_gpu, rel_err
from tests.layout import tiled_scale_index

pytestmark = pytest.mark.gpu


def _random_operand(b, rows, cols, rng, st):
    """Random codes / scales (scales in [2^-3, 2^3] so products stay normal)."""
    codes = rng.integers(0, 16, (rows, cols)).astype(np.uint8)
    scales = rng.integers(0x20, 0x51, (rows, cols // 16)).astype(np.uint8)
    t = b.NvFP4Tensor.empty(rows, cols, 1)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    t.codes.copy_(torch.from_numpy(packed))
    buf = np.zeros(b.scale_bytes(rows, cols, 1), np.uint8)
    buf[tiled_scale_index(rows, cols)] = scales
    t.scales.copy_(torch.from_numpy(buf))
    t.tensor_scale.fill_(st)
    return t, codes, scales


@pytest.mark.parametrize("M,N,K,W", [(128, 128, 256, 0), (128, 128, 64, 0), (256, 256, 512, 256),
                                     (300, 144, 320, 64), (1, 16, 64, 0), (130, 384, 1024, 192),
                                     (512, 512, 2048, 1024),
                                     (600, 400, 320, 64), (1024, 2048, 4096, 0), (777, 272, 576, 448),
                                     (512, 16, 64, 64),
                                     # CTA-pair kernel (256 x 256 tiles: enough tiles for its waves
                                     # to pay), ragged edges
                                     (4000, 2000, 320, 64), (2560, 1040, 576, 448), (4096, 2048, 256, 0),
                                     # split over K (few tiles, long K): 2 CTAs per tile; 4 per tile
                                     # with ragged rows / columns and short last K steps; splits
                                     # holding residual steps only
                                     (256, 4096, 4096, 0), (200, 272, 4096, 448), (130, 400, 3904, 576),
                                     (128, 128, 2048, 4096)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_gemm_on_random_operands(M, N, K, W, out):
    b = need_gpu()
    rng = np.random.default_rng(M * 7 + N)
    a, ac, asc = _random_operand(b, M, K, rng, 0.5)
    w, wc, wsc = _random_operand(b, N, K, rng, 0.25)
    ref = oracle.gemm_fp64(ac, asc, np.float32(0.5), wc, wsc, np.float32(0.25))
    r = s = None
    if W:
        r, rc, rsc = _random_operand(b, M, W, rng, 0.125)
        s, sc, ssc = _random_operand(b, N, W, rng, 2.0)
        ref = ref + oracle.gemm_fp64(rc, rsc, np.float32(0.125), sc, ssc, np.float32(2.0))
    dt = torch.float32 if out == "f32" else torch.bfloat16
    y = b.gemm_quantized(a, w, r, s, out_dtype=dt) if W else b.gemm_quantized(a, w, out_dtype=dt)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    tol = REL_TOL if out == "f32" else REL_TOL + 2.0 ** -8
    assert rel_err(y.float().cpu().numpy(), ref) < tol


def _check_linear(b, M, K, N, k, seed=0, rows=None, out_dtype=torch.float32):
    x = S.activations(M, K, seed=seed)
    w = S.weights(N, K, seed=seed)
    y, st = b.rac_linear(x.cuda(), w.cuda(), k, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    ref = oracle.rac_linear(bits(x), bits(w), k, rows=rows)
    yg = y.float().cpu().numpy()
    if rows is not None:
        yg = yg[rows]
    assert np.array_equal(st["mask"].cpu().numpy(), ref["mask"])
    if out_dtype == torch.float32:
        assert rel_err(yg, ref["y"]) < REL_TOL
    else:
        # bf16 output is RN(fp32 Y): within the fp32 bar plus one bf16 rounding
        assert rel_err(yg, ref["y"]) < REL_TOL + 2.0 ** -8
    return ref


@pytest.mark.parametrize("k", [0.0, 25.0, 50.0, 100.0])
def test_rac_linear_single(k):
    b = need_gpu()
    _check_linear(b, 64, 512, 512, k)


@pytest.mark.parametrize("M,K,N,k", [(300, 192, 144, 50.0), (1, 64, 16, 50.0), (130, 1024, 384, 12.5)])
def test_rac_linear_ragged(M, K, N, k):
    b = need_gpu()
    _check_linear(b, M, K, N, k, seed=M)


@pytest.mark.parametrize("k", [0.0, 25.0, 50.0, 100.0])
def test_rac_linear_dense_full_size(k):
    b = need_gpu()
    rows = np.sort(np.random.default_rng(1).choice(4096, 192, replace=False))
    rows = np.concatenate([[0, 127, 128, 4095], rows])
    _check_linear(b, 4096, 2048, 2048, k, rows=rows)


def test_rac_linear_decode_full_size():
    b = need_gpu()
    rows = np.arange(0, 256, 3)
    _check_linear(b, 256, 4096, 11008, 50.0, rows=rows, out_dtype=torch.bfloat16)


def test_bf16_output_is_rounded_fp32():
    b = need_gpu()
    x = S.activations(200, 256, seed=2).cuda()
    w = S.weights(256, 256, seed=2).cuda()
    y32, _ = b.rac_linear(x, w, 50.0, out_dtype=torch.float32)
    y16, _ = b.rac_linear(x, w, 50.0, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(y32.to(torch.bfloat16), y16)


@pytest.mark.parametrize("M,K,N", [(4096, 1024, 2048),   # CTA-pair kernel
                                   (128, 512, 256)])      # single-CTA kernel
@pytest.mark.parametrize("k", [0.0, 50.0])
def test_rac_linear_tiny_tensor_scales(M, K, N, k):
    """X and W scaled by 2^-60 each (exact in bf16): the product of their
    tensor scales, about 2^-140, is below fp32's normal range while Y (about
    2^-120) is representable, so the output scale must not be formed as one
    fp32 product."""
    b = need_gpu()
    x = (S.activations(M, K, seed=11).float() * 2.0 ** -60).to(torch.bfloat16)
    w = (S.weights(N, K, seed=11).float() * 2.0 ** -60).to(torch.bfloat16)
    y, st = b.rac_linear(x.cuda(), w.cuda(), k)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(3).integers(0, M, 96)]))
    ref = oracle.rac_linear(bits(x), bits(w), k, rows=rows)
    assert np.array_equal(st["mask"].cpu().numpy(), ref["mask"])
    assert float(st["qw"].tensor_scale.cpu()[0]) * float(st["qx"].tensor_scale.cpu()[0]) < 2.0 ** -126
    assert rel_err(y.cpu().numpy()[rows], ref["y"]) < REL_TOL
