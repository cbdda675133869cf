"""The fused calls against the separate ones they replace, bit for bit:
rac_quantize_select (quantize pass with the top-k% selection in its tail)
against nvfp4_quantize + rac_select_channels, rac_second_pass (both second
passes in one call) against rac_residual_quant + rac_weight_quant(_fp4), and
RacLinearPlan.full_step against split_step; plus the selection against the
oracle."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import bits, need_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,k", [(300, 192, 50.0), (1, 64, 100.0), (4096, 2048, 50.0), (257, 11008, 50.0),
                                   (130, 1024, 0.0), (64, 512, 12.5)])
@pytest.mark.parametrize("caller_amax", [False, True])
def test_quantize_select_matches_separate_calls(M, K, k, caller_amax):
    b = need_gpu()
    x = S.activations(M, K, seed=M + K).cuda()
    amax = x.float().abs().max().reshape(1) if caller_amax else None
    qx, score, cm, mask, sel, n_sel, st = b.quantize_select(x, k, amax=amax)
    rq, rscore, rcm = b.quantize(x, amax=amax)
    rmask, rsel, rn, rst = b.rac_select_channels(rscore, rcm, k)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    assert n_sel == rn
    for a_, b_ in [(qx.codes, rq.codes), (qx.scales, rq.scales), (qx.tensor_scale, rq.tensor_scale), (score, rscore),
                   (cm, rcm), (mask, rmask), (sel, rsel), (st, rst)]:
        assert torch.equal(a_, b_)
    if M * K <= 4096 * 2048:
        ref = oracle.quantize_activations(bits(x.cpu()))
        sel_ref, mask_ref = oracle.select_channels(ref["score"], oracle.n_selected(k, K))
        assert np.array_equal(mask.cpu().numpy(), mask_ref)
        assert np.array_equal(sel.cpu().numpy(), sel_ref)


@pytest.mark.parametrize("M,K,N,k", [(300, 192, 144, 50.0), (4096, 2048, 2048, 50.0), (256, 4096, 11008, 50.0),
                                     (64, 512, 512, 25.0),
                                     # row-staged residual with the weight in the same launch
                                     (8192, 1024, 640, 25.0), (16384, 4096, 4096, 50.0)])
@pytest.mark.parametrize("wsel", ["bf16", "fp4"])
def test_second_pass_matches_separate_calls(M, K, N, k, wsel):
    b = need_gpu()
    x, w = S.activations(M, K, seed=M).cuda(), S.weights(N, K, seed=N).cuda()
    _, qw, cmw = b.weight_qdq(w)
    cm = cmw[0] if wsel == "bf16" else b.dq_colamax(qw)[0]
    qx, score, rcm = b.quantize(x)
    mask, sel, n_sel, st = b.rac_select_channels(score, rcm, k)
    q_res, q_ws = b.second_pass(x, qx, sel, n_sel, st, w if wsel == "bf16" else None, qw, cm)
    r_res = b.rac_residual_quant(x, qx, sel, n_sel, st)
    r_ws = b.rac_weight_quant(w, sel, n_sel, cm) if wsel == "bf16" else b.rac_weight_quant_fp4(qw, sel, n_sel, cm)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    for t1, t2 in [(q_res, r_res), (q_ws, r_ws)]:
        assert torch.equal(t1.codes, t2.codes)
        assert torch.equal(t1.scales, t2.scales)
        assert torch.equal(t1.tensor_scale, t2.tensor_scale)


@pytest.mark.parametrize("M,K,N", [(4096, 2048, 2048), (300, 192, 144), (256, 4096, 11008)])
def test_plan_full_step_equals_split_step(M, K, N):
    b = need_gpu()
    x, w = S.activations(M, K, seed=1).cuda(), S.weights(N, K, seed=1).cuda()
    p1 = b.RacLinearPlan(M, K, N, 50.0, out_dtype=torch.float32).bind(x, w)
    p2 = b.RacLinearPlan(M, K, N, 50.0, out_dtype=torch.float32).bind(x, w)
    p1.full_step()
    p2.split_step()
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    assert torch.equal(p1.mask, p2.mask) and torch.equal(p1.sel, p2.sel)
    assert torch.equal(p1.q_res.codes, p2.q_res.codes) and torch.equal(p1.q_wsel.codes, p2.q_wsel.codes)
    assert torch.equal(p1.y, p2.y)
