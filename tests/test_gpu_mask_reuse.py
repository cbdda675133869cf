"""The mask-reuse variant: the quantizer's column-maxima-only mode, the
tensor scale over a given selection, and RacLinearPlan.reuse_step (channel
mask, sel and Q(W_sel) kept from an earlier step) against the oracle's RAC
linear with a given selection."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import REL_TOL, bits, need_gpu, rel_err
from tests.layout import unpack_codes, untile_scales

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [(300, 192), (4096, 2048), (256, 4096), (1, 64)])
def test_colamax_only_quantize_matches_full_mode(M, K):
    b = need_gpu()
    xd = S.activations(M, K, seed=M + 7).cuda()
    qa, score, cm = b.quantize(xd)
    qb, none, cm2 = b.quantize(xd, scores="colamax")
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(qa.codes, qb.codes) and torch.equal(qa.scales, qb.scales)
    assert torch.equal(qa.tensor_scale, qb.tensor_scale)
    assert torch.equal(cm, cm2)
    assert np.array_equal(cm2.cpu().numpy(), oracle.quantize_activations(bits(xd))["res_colamax"])


def test_sel_tensor_scale_matches_oracle():
    b = need_gpu()
    rng = np.random.default_rng(5)
    cm = rng.random(2048).astype(np.float32) * 3.0
    for n in (1, 7, 1024, 2048):
        sel = np.sort(rng.choice(2048, n, replace=False)).astype(np.int32)
        st = b.rac_sel_tensor_scale(torch.from_numpy(cm).cuda(), torch.from_numpy(sel).cuda(), n)
        torch.cuda.synchronize()
        assert np.float32(st.cpu().numpy()[0]) == oracle.tensor_scale(cm[sel].max())


@pytest.mark.parametrize("M,K,N,k", [(300, 192, 144, 50.0), (4096, 2048, 2048, 50.0), (256, 4096, 11008, 50.0)])
def test_reuse_step_matches_oracle_with_kept_mask(M, K, N, k):
    """Select on batch A, then run batch B with A's mask: B's residual
    quantization (its own tensor scale over A's channels) and Y equal the
    oracle's RAC linear with sel = A's selection."""
    b = need_gpu()
    xa, xb = S.activations(M, K, seed=M), S.activations(M, K, seed=M + 1)
    w = S.weights(N, K, seed=M)
    wd = w.cuda()
    plan = b.RacLinearPlan(M, K, N, k, out_dtype=torch.float32).bind(xa.cuda(), wd)
    plan.full_step()
    torch.cuda.synchronize()
    sel_a = plan.sel[:plan.n_sel].cpu().numpy().copy()
    plan.bind(xb.cuda(), wd)
    plan.reuse_step()
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    rows = np.arange(0, M, max(1, M // 97))
    ref = oracle.rac_linear(bits(xb), bits(w), k, rows=rows, sel=sel_a)
    assert np.float32(plan.q_res.tensor_scale.cpu().numpy()[0]) == ref["r_st"]
    assert np.array_equal(unpack_codes(plan.q_res.codes.cpu().numpy()), ref["r_codes"])
    assert np.array_equal(untile_scales(plan.q_res.scales.cpu().numpy(), M, ref["width"]), ref["r_scales"])
    assert rel_err(plan.y.cpu().numpy()[rows], ref["y"]) < REL_TOL


def test_reuse_step_on_the_selecting_batch_equals_the_full_step():
    b = need_gpu()
    M, K, N = 512, 1024, 768
    x, w = S.activations(M, K, seed=11).cuda(), S.weights(N, K, seed=11).cuda()
    plan = b.RacLinearPlan(M, K, N, 25.0, out_dtype=torch.float32).bind(x, w)
    plan.full_step()
    y1 = plan.y.clone()
    plan.reuse_step()
    torch.cuda.synchronize()
    assert torch.equal(plan.y, y1)
