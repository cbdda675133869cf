"""The NVFP4-sourced W_sel variant (W_sel re-quantized from DQ(Q(W)), for a
rollout that keeps only the NVFP4 weights): nvfp4_dq_colamax,
rac_weight_quant_fp4 and the w == NULL forms of the RAC linear and of the
grouped MoE call, against the oracle's weight_sel_from_fp4 path."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import REL_TOL, bits, need_gpu, rel_err
from tests.layout import tiled_scale_index, unpack_codes, untile_scales

pytestmark = pytest.mark.gpu


def _upload(b, codes, scales, st, layout):
    """NVFP4 tensor on the device from host codes [rows, cols], scale bytes
    [rows, cols/16] and tensor scales st [batch]."""
    rows, cols = codes.shape
    t = b.NvFP4Tensor.empty(rows, cols, layout, n_scales=len(st))
    t.codes.copy_(torch.from_numpy((codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)))
    buf = np.zeros(b.scale_bytes(rows, cols, layout), np.uint8)
    if layout == 1:
        buf[tiled_scale_index(rows, cols)] = scales
    else:
        buf[:] = scales.reshape(-1)
    t.scales.copy_(torch.from_numpy(buf))
    t.tensor_scale.copy_(torch.from_numpy(np.asarray(st, np.float32)))
    return t


def _random_nvfp4(rows, cols, rng, zero_cols=()):
    """Every E2M1 code (both signed zeros included) and every finite E4M3
    scale byte (0 .. 126, zero scales included); columns in zero_cols hold
    only signed-zero codes."""
    codes = rng.integers(0, 16, (rows, cols)).astype(np.uint8)
    for j in zero_cols:
        codes[:, j] = rng.integers(0, 2, rows).astype(np.uint8) * 8
    scales = rng.integers(0, 127, (rows, cols // 16)).astype(np.uint8)
    return codes, scales


@pytest.mark.parametrize("N,K,batch,layout", [(512, 512, 1, 1), (144, 320, 1, 1), (1, 64, 1, 0),
                                              (100, 192, 3, 0), (256, 128, 5, 1), (2048, 2048, 1, 1),
                                              (11008, 4096, 1, 1)])
def test_dq_colamax_matches_oracle(N, K, batch, layout):
    b = need_gpu()
    rng = np.random.default_rng(N + K + batch)
    codes, scales = _random_nvfp4(batch * N, K, rng, zero_cols=(0, K - 1))
    st = (2.0 ** rng.uniform(-12, 0, batch)).astype(np.float32)
    q = _upload(b, codes, scales, st, layout)
    got = b.dq_colamax(q, batch).cpu().numpy()
    torch.cuda.synchronize()
    for e in range(batch):
        r = slice(e * N, (e + 1) * N)
        ref = oracle.column_amax(oracle.dequantize(codes[r], scales[r], st[e]))
        assert np.array_equal(got[e], ref)


@pytest.mark.parametrize("N,K,k", [(512, 512, 50.0), (144, 1024, 25.0), (2048, 2048, 100.0),
                                   (300, 448, 12.5), (16, 64, 1.5625), (11008, 4096, 50.0),
                                   # 4 rows per pass (shared-memory bound) and the generic
                                   # gather (K beyond 16-bit channel indices)
                                   (48, 16384, 0.5), (16, 65600, 0.1)])
def test_weight_select_fp4_matches_oracle(N, K, k):
    b = need_gpu()
    rng = np.random.default_rng(N * 3 + K)
    codes, scales = _random_nvfp4(N, K, rng, zero_cols=(1, 5))
    st = np.float32(2.0 ** -9)
    q = _upload(b, codes, scales, [st], 1)
    n_sel = oracle.n_selected(k, K)
    sel = np.sort(rng.choice(K, n_sel, replace=False)).astype(np.int32)
    dq_cm = b.dq_colamax(q)[0]
    qs = b.rac_weight_quant_fp4(q, torch.from_numpy(sel).cuda(), n_sel, dq_cm)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    width = oracle.padded_width(n_sel)
    c, s, st_ref = oracle.weight_sel_from_fp4(codes, scales, st, sel, width)
    assert np.float32(qs.tensor_scale.cpu().numpy()[0]) == st_ref
    assert np.array_equal(untile_scales(qs.scales.cpu().numpy(), N, width), s)
    assert np.array_equal(unpack_codes(qs.codes.cpu().numpy()), c)


def test_weight_select_fp4_all_zero_selection():
    """Selected columns that dequantize to signed zeros only: tensor scale 0,
    zero block scales and the signed-zero codes of the values."""
    b = need_gpu()
    rng = np.random.default_rng(11)
    N, K = 256, 256
    sel = np.array([3, 17, 64, 200], np.int32)
    codes, scales = _random_nvfp4(N, K, rng, zero_cols=sel)
    q = _upload(b, codes, scales, [np.float32(0.01)], 1)
    qs = b.rac_weight_quant_fp4(q, torch.from_numpy(sel).cuda(), len(sel), b.dq_colamax(q)[0])
    torch.cuda.synchronize()
    width = oracle.padded_width(len(sel))
    c, s, st_ref = oracle.weight_sel_from_fp4(codes, scales, np.float32(0.01), sel, width)
    assert st_ref == 0.0 and np.float32(qs.tensor_scale.cpu().numpy()[0]) == 0.0
    assert np.array_equal(untile_scales(qs.scales.cpu().numpy(), N, width), s)
    assert np.array_equal(unpack_codes(qs.codes.cpu().numpy()), c)


def _check_linear_fp4(b, M, K, N, k, seed=0, rows=None, out_dtype=torch.float32):
    x = S.activations(M, K, seed=seed)
    w = S.weights(N, K, seed=seed)
    y, st = b.rac_linear(x.cuda(), w.cuda(), k, out_dtype=out_dtype, wsel="fp4")
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    ref = oracle.rac_linear(bits(x), bits(w), k, rows=rows, wsel_source="fp4")
    yg = y.float().cpu().numpy()
    if rows is not None:
        yg = yg[rows]
    assert np.array_equal(st["mask"].cpu().numpy(), ref["mask"])
    tol = REL_TOL if out_dtype == torch.float32 else REL_TOL + 2.0 ** -8
    assert rel_err(yg, ref["y"]) < tol


@pytest.mark.parametrize("M,K,N,k", [(64, 512, 512, 50.0), (64, 512, 512, 100.0), (300, 192, 144, 50.0),
                                     (1, 64, 16, 50.0), (130, 1024, 384, 12.5), (64, 512, 512, 0.0)])
def test_rac_linear_fp4_matches_oracle(M, K, N, k):
    b = need_gpu()
    _check_linear_fp4(b, M, K, N, k, seed=M + K)


def test_rac_linear_fp4_decode_full_size_plan():
    """The decode up projection (256 x 4096 -> 11008) as the bench runs it:
    RacLinearPlan with the weight preparation on a side stream."""
    b = need_gpu()
    M, K, N = 256, 4096, 11008
    x = S.activations(M, K, seed=5)
    w = S.weights(N, K, seed=5)
    plan = b.RacLinearPlan(M, K, N, 50.0, out_dtype=torch.bfloat16, wsel="fp4").bind(x.cuda(), w.cuda())
    plan.full_step()
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    rows = np.arange(0, M, 5)
    ref = oracle.rac_linear(bits(x), bits(w), 50.0, rows=rows, wsel_source="fp4")
    assert np.array_equal(plan.mask.cpu().numpy(), ref["mask"])
    assert rel_err(plan.y.float().cpu().numpy()[rows], ref["y"]) < REL_TOL + 2.0 ** -8
    # the plan's W_sel is the oracle's, byte for byte
    assert np.array_equal(unpack_codes(plan.q_wsel.codes.cpu().numpy()), ref["ws_codes"])
    assert np.array_equal(untile_scales(plan.q_wsel.scales.cpu().numpy(), N, ref["width"]), ref["ws_scales"])
    assert np.float32(plan.q_wsel.tensor_scale.cpu().numpy()[0]) == ref["ws_st"]


@pytest.mark.parametrize("counts,N,K,k", [([70, 0, 130, 5], 128, 256, 50.0),
                                          ([0, 300, 128, 129, 0], 256, 192, 25.0),
                                          ([1], 128, 64, 100.0)])
def test_moe_fp4_wsel_matches_oracle(counts, N, K, k):
    b = need_gpu()
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    E = len(counts)
    x = S.activations(int(off[-1]), K, seed=E + 1)
    w = S.weights(N, K, seed=E + 1, batch=E)
    xd, wd = x.cuda(), w.cuda()
    _, qw, _ = b.weight_qdq(wd, want_colamax=False)
    dq_cm = b.dq_colamax(qw, E)
    offd = torch.from_numpy(off).cuda()
    y, masks = b.moe_rac(xd, offd, None, qw, dq_cm, k)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    y_ref, masks_ref, _ = oracle.moe_rac(bits(x), off, bits(w).reshape(E, N, K), k, wsel_source="fp4")
    assert np.array_equal(masks.cpu().numpy(), masks_ref)
    assert rel_err(y.cpu().numpy(), y_ref) < REL_TOL
