"""rac_select through the C ABI against the oracle: mask, sel, n_sel and the
second-pass quantization of the gathered residual, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import bits, need_gpu
from tests.layout import unpack_codes, untile_scales

pytestmark = pytest.mark.gpu


def _check_select(b, x, k):
    M, K = x.shape
    xd = x.cuda()
    qx, score, cm = b.quantize(xd, layout=1)
    mask, sel, n_sel, q_res = b.rac_select(xd, qx, score, cm, k)
    torch.cuda.synchronize()
    ref = oracle.quantize_activations(bits(x))
    n_ref = oracle.n_selected(k, K)
    sel_ref, mask_ref = oracle.select_channels(ref["score"], n_ref)
    assert n_sel == n_ref
    assert np.array_equal(mask.cpu().numpy(), mask_ref)
    assert np.array_equal(sel.cpu().numpy(), sel_ref)
    if n_sel == 0:
        assert q_res is None
        return
    width = oracle.padded_width(n_sel)
    rc, rs, rst = oracle.gather_quantize(ref["dx"], sel_ref, width, ref["res_colamax"][sel_ref].max())
    assert np.float32(q_res.tensor_scale.cpu().numpy()[0]) == rst
    assert np.array_equal(untile_scales(q_res.scales.cpu().numpy(), M, width), rs)
    assert np.array_equal(unpack_codes(q_res.codes.cpu().numpy()), rc)


@pytest.mark.parametrize("M,K,k", [(64, 512, 50.0), (300, 192, 25.0), (1, 64, 50.0), (130, 1024, 100.0),
                                   (257, 2048, 0.0), (200, 11008 // 2, 50.0), (77, 448, 12.5),
                                   (40, 16384, 50.0), (9, 65536, 3.0)])
def test_select_matches_oracle(M, K, k):
    b = need_gpu()
    _check_select(b, S.activations(M, K, seed=M), k)


@pytest.mark.parametrize("k", [0.0, 25.0, 50.0, 100.0])
def test_select_dense_full_size(k):
    b = need_gpu()
    _check_select(b, S.activations(4096, 2048, seed=0), k)


def test_select_ties_lower_index():
    b = need_gpu()
    x = S.bf16_bits(S.activations(96, 256, seed=9)).copy()
    x[:, 128:256] = x[:, 0:128]          # every channel has an identical twin 128 later
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    for k in (10.0, 50.0, 75.0):
        _check_select(b, t, k)
    z = S.to_bf16(np.zeros((40, 128), np.float32))   # all scores equal: first n_sel channels
    _check_select(b, z, 50.0)
