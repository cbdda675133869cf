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


@pytest.mark.parametrize("M,K,k", [(300, 192, 25.0), (4096, 2048, 50.0), (64, 512, 0.0)])
def test_split_select_equals_rac_select(M, K, k):
    """rac_select_channels followed by rac_residual_quant gives rac_select's
    mask, sel, residual tensor scale, codes and scales byte for byte."""
    b = need_gpu()
    xd = S.activations(M, K, seed=M + 1).cuda()
    qx, score, cm = b.quantize(xd, layout=1)
    mask, sel, n_sel, q_res = b.rac_select(xd, qx, score, cm, k)
    mask2, sel2, n2, st = b.rac_select_channels(score, cm, k)
    torch.cuda.synchronize()
    assert n2 == n_sel
    assert torch.equal(mask, mask2) and torch.equal(sel, sel2)
    if n_sel == 0:
        assert float(st.cpu()[0]) == 0.0
        return
    q2 = b.rac_residual_quant(xd, qx, sel2, n2, st)
    torch.cuda.synchronize()
    assert torch.equal(q_res.tensor_scale, q2.tensor_scale)
    assert torch.equal(q_res.codes, q2.codes)
    assert torch.equal(q_res.scales, q2.scales)


def test_plan_step_with_overlapped_gathers_matches_oracle():
    """The plan's rollout step (W_sel gather on the side stream beside the
    residual gather) against the oracle, dense shape, sampled rows."""
    b = need_gpu()
    M, K, N = 4096, 2048, 2048
    x, w = S.activations(M, K, seed=3), S.weights(N, K, seed=3)
    plan = b.RacLinearPlan(M, K, N, 50.0, out_dtype=torch.float32).bind(x.cuda(), w.cuda())
    plan.prepare_weight()
    for _ in range(2):
        plan.rollout_step()
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    rows = np.arange(0, M, 37)
    ref = oracle.rac_linear(bits(x), bits(w), 50.0, rows=rows)
    assert np.array_equal(plan.mask.cpu().numpy(), ref["mask"])
    from tests.gpu_common import REL_TOL, rel_err
    assert rel_err(plan.y.cpu().numpy()[rows], ref["y"]) < REL_TOL
