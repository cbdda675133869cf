"""weight_qdq (trainer-side W4A16 fake quantization, plus Q(W) and colamax
for the rollout side) and rac_weight_quant (Q(W_sel)) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import bits, need_gpu
from tests.layout import unpack_codes, untile_scales

pytestmark = pytest.mark.gpu


def _check_qdq(b, w, layout=1, experts=None):
    wd = w.cuda()
    batch, N, K = (1, *w.shape) if w.dim() == 2 else w.shape
    w_out, qw, colamax = b.weight_qdq(wd, layout=layout)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    wb = bits(w).reshape(batch, N, K)
    got_out = bits(w_out).reshape(batch, N, K)
    codes = unpack_codes(qw.codes.cpu().numpy())
    sc = qw.scales.cpu().numpy()
    scales = untile_scales(sc, batch * N, K) if layout == 1 else sc[: batch * N * K // 16].reshape(batch * N, K // 16)
    for e in (range(batch) if experts is None else experts):
        ref = oracle.weight_qdq(wb[e])
        assert np.array_equal(got_out[e], ref["w_out"])
        assert np.array_equal(codes[e * N:(e + 1) * N], ref["codes"])
        assert np.array_equal(scales[e * N:(e + 1) * N], ref["scales"])
        assert np.float32(qw.tensor_scale.cpu().numpy()[e]) == ref["s_t"]
        assert np.array_equal(colamax.cpu().numpy()[e], ref["colamax"])


@pytest.mark.parametrize("N,K", [(512, 512), (2048, 2048), (144, 320), (1, 64), (11008, 4096)])
def test_weight_qdq_matches_oracle(N, K):
    b = need_gpu()
    _check_qdq(b, S.weights(N, K, seed=N))


def test_weight_qdq_batched_experts():
    b = need_gpu()
    _check_qdq(b, S.weights(256, 128, seed=3, batch=5))
    _check_qdq(b, S.weights(100, 64, seed=4, batch=3), layout=0)


def test_weight_qdq_stacked_clusters():
    """Stacks of several matrices (one launch pair for the whole stack):
    ragged row counts, one and several column tiles, both scale layouts."""
    b = need_gpu()
    _check_qdq(b, S.weights(100, 64, seed=5, batch=12))
    _check_qdq(b, S.weights(300, 320, seed=6, batch=9), layout=0)
    _check_qdq(b, S.weights(128, 1024, seed=8, batch=40))


def test_weight_qdq_stacked_clusters_in_place():
    b = need_gpu()
    w = S.weights(200, 256, seed=9, batch=10)
    wb = bits(w).reshape(10, 200, 256)
    wd = w.cuda()
    b.weight_qdq(wd, want_q=False, want_colamax=False, out=wd)
    torch.cuda.synchronize()
    got = bits(wd).reshape(10, 200, 256)
    for e in range(10):
        assert np.array_equal(got[e], oracle.weight_qdq(wb[e])["w_out"])


def test_weight_qdq_expert_stack_full_size():
    """The prefill step's trainer-side QDQ shape, 64 experts x 1024 x 2048
    (the two passes over the whole stack): four experts checked
    against the oracle in full, every tensor scale against its amax."""
    b = need_gpu()
    w = S.weights(1024, 2048, seed=11, batch=64)
    _check_qdq(b, w, experts=[0, 21, 42, 63])
    _, qw, _ = b.weight_qdq(w.cuda())
    torch.cuda.synchronize()
    wf = w.float().numpy().reshape(64, 1024 * 2048)     # bf16 values, exact in fp32
    st = qw.tensor_scale.cpu().numpy()
    for e in range(64):
        assert np.float32(st[e]) == oracle.nvfp4.tensor_scale(oracle.nvfp4.amax(wf[e]))


def test_weight_qdq_tensor_scales_across_fast_bound():
    """Stacked experts whose tensor scales lie on both sides of 2^-55 (the
    bound above which the quotients take the reciprocal-table path), down to
    a subnormal s_t: W4A16 outputs, codes, scales and colamax bit for bit."""
    b = need_gpu()
    w = S.weights(256, 192, seed=11, batch=7).float()
    for e, k in enumerate((0, 40, 41, 44, 60, 100, 120)):
        w[e] *= 2.0 ** -k
    _check_qdq(b, w.to(torch.bfloat16))


def test_weight_qdq_in_place():
    b = need_gpu()
    w = S.weights(256, 512, seed=7)
    ref = oracle.weight_qdq(bits(w))
    wd = w.cuda()
    b.weight_qdq(wd, want_q=False, want_colamax=False, out=wd)
    torch.cuda.synchronize()
    assert np.array_equal(bits(wd), ref["w_out"])


@pytest.mark.parametrize("N,K,k", [(512, 512, 50.0), (144, 1024, 25.0), (2048, 2048, 100.0), (300, 448, 12.5),
                                   (11008, 4096, 50.0), (16, 64, 1.5625),
                                   # one row per pass (shared-memory bound) and the generic
                                   # gather (K beyond 16-bit channel indices)
                                   (48, 16384, 0.5), (16, 65600, 0.1)])
def test_weight_select_quant_matches_oracle(N, K, k):
    b = need_gpu()
    w = S.weights(N, K, seed=K)
    rng = np.random.default_rng(N)
    n_sel = oracle.n_selected(k, K)
    sel = np.sort(rng.choice(K, n_sel, replace=False)).astype(np.int32)
    wd = w.cuda()
    _, _, colamax = b.weight_qdq(wd, want_q=False)
    q = b.rac_weight_quant(wd, torch.from_numpy(sel).cuda(), n_sel, colamax[0])
    torch.cuda.synchronize()
    wf = oracle.bf16_to_f32(bits(w))
    width = oracle.padded_width(n_sel)
    c, s, st = oracle.gather_quantize(wf, sel, width, oracle.column_amax(wf)[sel].max())
    assert np.float32(q.tensor_scale.cpu().numpy()[0]) == st
    assert np.array_equal(untile_scales(q.scales.cpu().numpy(), N, width), s)
    assert np.array_equal(unpack_codes(q.codes.cpu().numpy()), c)
