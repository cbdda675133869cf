"""nvfp4_quantize through the C ABI against the oracle: codes, block scales,
tensor scale, channel scores and residual column maxima, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import bits, need_gpu
from tests.layout import tiled_padding_mask, unpack_codes, untile_scales

pytestmark = pytest.mark.gpu


def _check_quant(b, x, layout, with_amax=False):
    M, K = x.shape
    xd = x.cuda()
    ref = oracle.quantize_activations(bits(x))
    amax = torch.tensor([float(ref["amax"])], dtype=torch.float32, device="cuda") if with_amax else None
    qx, score, cm = b.quantize(xd, amax=amax, layout=layout)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    codes = unpack_codes(qx.codes.cpu().numpy())
    sc = qx.scales.cpu().numpy()
    scales = untile_scales(sc, M, K) if layout == 1 else sc[: M * K // 16].reshape(M, K // 16)
    assert np.float32(qx.tensor_scale.cpu().numpy()[0]) == ref["s_t"]
    assert np.array_equal(scales, ref["scales"])
    assert np.array_equal(codes, ref["codes"])
    assert np.array_equal(score.cpu().numpy(), ref["score"])
    assert np.array_equal(cm.cpu().numpy(), ref["res_colamax"])
    if layout == 1:
        assert not sc[tiled_padding_mask(M, K)].any()


@pytest.mark.parametrize("M,K", [(64, 512), (1, 64), (300, 192), (130, 2048), (257, 4096)])
@pytest.mark.parametrize("layout", [0, 1])
def test_quantize_matches_oracle(M, K, layout):
    b = need_gpu()
    _check_quant(b, S.activations(M, K, seed=M + K), layout)


def test_quantize_caller_amax():
    b = need_gpu()
    _check_quant(b, S.activations(200, 256, seed=5), 1, with_amax=True)


def test_quantize_dense_full_size():
    b = need_gpu()
    _check_quant(b, S.activations(4096, 2048, seed=0), 1)


def test_quantize_edge_values():
    b = need_gpu()
    rng = np.random.default_rng(3)
    x = rng.standard_normal((160, 128)).astype(np.float32)
    x[:, 16:32] = 0.0                          # zero blocks
    x[5, 40:56] = -0.0                         # negative zeros
    x[7, :] = 3e38 * np.sign(x[7, :])          # near-max magnitudes
    x[9, 64:80] = 1e-38                        # tiny block next to huge tensor amax
    x[11, 80:96] = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 2)   # ties once scaled
    t = S.to_bf16(x)
    _check_quant(b, t, 1)
    _check_quant(b, S.to_bf16(np.zeros((70, 64), np.float32)), 1)
    _check_quant(b, S.to_bf16(-np.zeros((3, 64), np.float32)), 0)
