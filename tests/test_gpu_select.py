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


def _check_channels(b, score, k):
    """rac_select_channels on given fp64 scores against oracle.select_channels
    (mask, ascending sel, and s_tR = RN(max colamax over sel / 2688))."""
    K = score.shape[0]
    cm = np.random.default_rng(K).random(K).astype(np.float32)
    mask, sel, n_sel, st = b.rac_select_channels(torch.from_numpy(score).cuda(), torch.from_numpy(cm).cuda(), k)
    torch.cuda.synchronize()
    n_ref = oracle.n_selected(k, K)
    sel_ref, mask_ref = oracle.select_channels(score, n_ref)
    assert n_sel == n_ref
    assert np.array_equal(mask.cpu().numpy(), mask_ref)
    assert np.array_equal(sel.cpu().numpy(), sel_ref)
    want = np.float32(cm[sel_ref].max()) / np.float32(2688.0) if n_ref else np.float32(0.0)
    assert np.float32(st.cpu().numpy()[0]) == want


def _constructed_scores():
    """Score vectors that steer the selection through each of its branches:
    boundary bins taken whole, boundary bins ranked by bits below the 12-bit
    digit (with exact ties), boundary bins of more than 1024 keys (equal or
    merely close), many zero scores, and the two sides of the 16384-channel
    digit limit."""
    rng = np.random.default_rng(2024)
    out = {}
    # every key in its own 12-bit bin: 1 + j / 4096
    out["whole_bins"] = 1.0 + rng.permutation(2048).astype(np.float64) / 4096.0
    # four groups far apart, keys within a group differing only in the lowest
    # 20 mantissa bits, some of them equal
    g = rng.integers(0, 4, 2048).astype(np.float64)
    lo = rng.integers(0, 1 << 20, 2048)
    lo[rng.integers(0, 2048, 300)] = lo[0]
    out["low_bits"] = 1.0 + g * 2.0 ** -8 + lo.astype(np.float64) * 2.0 ** -52
    # 3000 equal keys straddling the boundary, distinct keys around them
    v = np.concatenate([2.0 + rng.random(2500), np.full(3000, 1.5), 1.0 + 0.4 * rng.random(2692)])
    out["big_equal_bin"] = v[rng.permutation(v.size)]
    # 2000 distinct keys that share their leading 12 varying bits
    c = np.concatenate([1.0 + rng.integers(0, 1 << 30, 2000).astype(np.float64) * 2.0 ** -52,
                        8.0 + rng.random(1500), 0.25 * rng.random(596)])
    out["big_close_bin"] = c[rng.permutation(c.size)]
    # mostly zero scores
    z = np.zeros(4096)
    z[rng.choice(4096, 596, replace=False)] = rng.random(596) * 100.0
    out["zeros"] = z
    out["k16384"] = rng.random(16384) * rng.choice([1.0, 1e-3, 1e5], 16384)
    out["k16448"] = rng.random(16448) * rng.choice([1.0, 1e-3, 1e5], 16448)
    return out


@pytest.mark.parametrize("name", ["whole_bins", "low_bits", "big_equal_bin", "big_close_bin", "zeros",
                                  "k16384", "k16448"])
def test_select_channels_constructed_scores(name):
    b = need_gpu()
    score = _constructed_scores()[name]
    for k in (0.05, 12.5, 50.0, 99.96, 100.0, 0.0):
        _check_channels(b, score, k)


def test_select_channels_unaligned_buffers():
    """Scores, colamax and mask at odd offsets (scores 8 bytes past a
    16-byte boundary, colamax 4 bytes, the mask 1 byte) give the same
    selection as the oracle."""
    import ctypes
    b = need_gpu()
    K = 4096
    rng = np.random.default_rng(7)
    score = rng.random(K) * rng.choice([1.0, 1e-3, 1e5], K)
    cm = rng.random(K).astype(np.float32)
    sbuf = torch.zeros(K + 1, dtype=torch.float64, device="cuda")
    cbuf = torch.zeros(K + 1, dtype=torch.float32, device="cuda")
    mbuf = torch.zeros(K + 8, dtype=torch.uint8, device="cuda")
    sbuf[1:] = torch.from_numpy(score).cuda()
    cbuf[1:] = torch.from_numpy(cm).cuda()
    for k in (12.5, 50.0, 99.96):
        n_ref = oracle.n_selected(k, K)
        sel = torch.zeros(max(n_ref, 1), dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.float32, device="cuda")
        n_out = ctypes.c_int64(-1)
        status = b._lib.rac_select_channels(ctypes.c_void_p(sbuf.data_ptr() + 8), ctypes.c_void_p(cbuf.data_ptr() + 4),
                                            K, ctypes.c_float(k), ctypes.c_void_p(mbuf.data_ptr() + 1),
                                            ctypes.c_void_p(sel.data_ptr()), ctypes.byref(n_out),
                                            ctypes.c_void_p(st.data_ptr()), None)
        torch.cuda.synchronize()
        assert status == 0 and n_out.value == n_ref
        sel_ref, mask_ref = oracle.select_channels(score, n_ref)
        assert np.array_equal(mbuf[1:K + 1].cpu().numpy(), mask_ref)
        assert np.array_equal(sel[:n_ref].cpu().numpy(), sel_ref)
        assert np.float32(st.cpu().numpy()[0]) == np.float32(cm[sel_ref].max()) / np.float32(2688.0)
