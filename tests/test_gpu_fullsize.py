"""Parity at the full sizes of the rollout workloads, in the launch
configuration the benchmark times.

* large prefill (X 32768 x 4096, W 4096 x 4096, k = 50 %) through
  RacLinearPlan.full_step, the step bench.py times: Q(X) codes, block scales,
  channel scores and residual column maxima in full, the mask and sel, the
  second-pass operands Q(dX_sel) and Q(W_sel) in full, and Y on 520 sampled
  rows against the oracle's fp64 product;
* the decode-shaped down projection (X' 256 x 11008 -> 4096) through
  rac_linear: quantizer at K = 11008, the single-CTA GEMM, all of Y;
* the MoE expert FFN down projection (1024 -> 2048, 65536 routed rows over
  64 experts) and the masks of all 64 experts of both projections.
Every oracle call here quantizes and scores all rows; only the fp64 products
are restricted to sampled rows where noted.
"""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import REL_TOL, bits, need_gpu, rel_err
from tests.layout import unpack_codes, untile_scales

pytestmark = pytest.mark.gpu


def _same_q(t, codes, scales, st, rows, cols):
    assert np.float32(t.tensor_scale.cpu().numpy()[0]) == st
    assert np.array_equal(untile_scales(t.scales.cpu().numpy(), rows, cols), scales)
    assert np.array_equal(unpack_codes(t.codes.cpu().numpy()), codes)


def test_large_prefill_plan_step_matches_oracle():
    b = need_gpu()
    M, K, N, k = 32768, 4096, 4096, 50.0
    x, w = S.activations(M, K, seed=0), S.weights(N, K, seed=0)
    plan = b.RacLinearPlan(M, K, N, k, out_dtype=torch.float32).bind(x.cuda(), w.cuda())
    plan.full_step()
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], rng.integers(0, M, 516)]))
    ref = oracle.rac_linear(bits(x), bits(w), k, rows=rows)
    _same_q(plan.qx, ref["codes"], ref["scales"], ref["s_t"], M, K)
    assert np.array_equal(plan.score.cpu().numpy(), ref["score"])
    assert np.array_equal(plan.res_colamax.cpu().numpy(), ref["res_colamax"])
    assert np.array_equal(plan.mask.cpu().numpy(), ref["mask"])
    assert np.array_equal(plan.sel[: plan.n_sel].cpu().numpy(), ref["sel"])
    _same_q(plan.q_res, ref["r_codes"], ref["r_scales"], ref["r_st"], M, ref["width"])
    _same_q(plan.q_wsel, ref["ws_codes"], ref["ws_scales"], ref["ws_st"], N, ref["width"])
    assert len(rows) >= 512
    assert rel_err(plan.y.cpu().numpy()[rows], ref["y"]) < REL_TOL


def test_decode_down_projection_full():
    b = need_gpu()
    M, K, N, k = 256, 11008, 4096, 50.0
    x = S.activations(M, K, seed=0, stream=S.STREAM_X_DOWN)
    w = S.weights(N, K, seed=0, stream=S.STREAM_W + 10)
    y, st = b.rac_linear(x.cuda(), w.cuda(), k)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    ref = oracle.rac_linear(bits(x), bits(w), k)
    _same_q(st["qx"], ref["codes"], ref["scales"], ref["s_t"], M, K)
    assert np.array_equal(st["score"].cpu().numpy(), ref["score"])
    assert np.array_equal(st["mask"].cpu().numpy(), ref["mask"])
    _same_q(st["q_res"], ref["r_codes"], ref["r_scales"], ref["r_st"], M, ref["width"])
    assert rel_err(y.cpu().numpy(), ref["y"]) < REL_TOL


def _moe_check(b, x, off, w, k, sample_rows):
    E, N, K = w.shape
    xd, wd = x.cuda(), w.cuda()
    _, qw, colamax = b.weight_qdq(wd)
    offd = torch.from_numpy(np.asarray(off, np.int64)).cuda()
    y, masks = b.moe_rac(xd, offd, wd, qw, colamax, k)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    y, masks = y.cpu().numpy(), masks.cpu().numpy()
    xb, wb = bits(x), bits(w).reshape(E, N, K)
    rng = np.random.default_rng(E + N)
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            sel, mask = oracle.select_channels(np.zeros(K), oracle.n_selected(k, K))
            assert np.array_equal(masks[e], mask)
            continue
        rows = np.unique(np.concatenate([[0, r1 - r0 - 1], rng.integers(0, r1 - r0, sample_rows)]))
        ref = oracle.rac_linear(xb[r0:r1], wb[e], k, rows=rows)
        assert np.array_equal(masks[e], ref["mask"]), f"expert {e}"
        assert rel_err(y[r0:r1][rows], ref["y"]) < REL_TOL, f"expert {e}"


def test_moe_down_projection_full_size_all_masks():
    """8192 tokens routed top-8 over 64 Zipf(1.1) experts; down projection
    1024 -> 2048 on the synthetic down-projection input."""
    b = need_gpu()
    cfg = S.MOE
    inp = S.moe_inputs(cfg["T"], cfg["hidden"], cfg["inter"], cfg["E"], cfg["topk"], seed=0)
    _moe_check(b, inp["x_down"], inp["offsets"], inp["w_down"], cfg["k"], sample_rows=6)


def test_moe_up_projection_all_masks():
    b = need_gpu()
    cfg = S.MOE
    inp = S.moe_inputs(cfg["T"], cfg["hidden"], cfg["inter"], cfg["E"], cfg["topk"], seed=0)
    _moe_check(b, inp["x_perm"], inp["offsets"], inp["w_up"], cfg["k"], sample_rows=6)
