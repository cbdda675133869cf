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


def _boundary_tensor(s_t_target, seed):
    """Blocks whose elements sit within a few bf16 ulps of every E2M1 rounding
    midpoint (times the block's decode scale), for all 126 positive E4M3
    block scales; the first block carries the tensor amax 2688 * s_t."""
    import torch as _t
    from oracle import formats as F
    rng = np.random.default_rng(seed)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    blocks = [np.r_[2688.0 * s_t_target, np.zeros(15)]]
    for sb in range(1, 0x7F):
        sdec = F.E4M3_POSITIVE[sb] * s_t_target
        bmax = 6.0 * sdec
        cands = []
        for m in mids:
            c = np.float32(m * sdec)
            b = _t.tensor([c]).to(_t.bfloat16).view(_t.int16).item() & 0xFFFF
            cands += [np.uint16(b + d).view(np.int16) for d in range(-3, 4)]
        vals = S.bf16_bits(_t.tensor(np.array(cands, np.int16)).view(_t.bfloat16)).astype(np.uint32)
        vals = (vals << 16).view(np.float32)
        vals = vals[np.abs(vals) <= bmax]
        vals = vals * rng.choice([-1.0, 1.0], vals.size)
        for i in range(0, len(vals), 15):
            chunk = vals[i:i + 15]
            blocks.append(np.r_[bmax, chunk, np.zeros(15 - len(chunk))])
    x = np.concatenate(blocks)
    pad = (-len(x)) % 256
    return S.to_bf16(np.r_[x, np.zeros(pad)].astype(np.float32).reshape(-1, 256))


@pytest.mark.parametrize("s_t,seed", [(1.0, 0), (2.0 ** -7, 1), (0.0123456, 2), (3.7e-5, 3)])
def test_quantize_rounding_boundaries(s_t, seed):
    b = need_gpu()
    _check_quant(b, _boundary_tensor(s_t, seed), 1)


def test_score_row_order_on_wide_columns():
    """Columns whose |dX| span far more than 22 binades take the kernel's
    row-order path; their scores must still equal the oracle's (and the
    values that IEEE rounding fixes for the plain order).  Column 0 holds 448
    in every row, so every block's scale makes 1.0 and 2^-53 quantize to 0
    and dX equals x there."""
    b = need_gpu()
    u = 2.0 ** -53
    x = np.zeros((384, 64), np.float32)
    x[:, 0] = 448.0
    x[0, 1] = 1.0
    x[1:128, 1] = u                      # 1 then 127 x u: every addition ties to 1.0
    x[0:127, 2] = u
    x[127, 2] = 1.0                      # 127 u then 1: 1 + 2^-46
    x[0, 3] = 1.0
    x[128, 3] = u
    x[129, 3] = u                        # chunk sums 1 and 2u: 1 + 2^-52
    x[0, 4] = 1.0
    x[128, 4] = u
    x[256, 4] = u                        # chunks 1, u, u in order: 1.0
    xt = torch.from_numpy(x).to(torch.bfloat16)
    _, score, _ = b.quantize(xt.cuda(), layout=1)
    torch.cuda.synchronize()
    got = score.cpu().numpy()
    ref = oracle.quantize_activations(bits(xt))["score"]
    assert np.array_equal(got, ref)
    assert got[1] == 1.0 and got[2] == 1.0 + 2.0 ** -46 and got[3] == 1.0 + 2.0 ** -52 and got[4] == 1.0
