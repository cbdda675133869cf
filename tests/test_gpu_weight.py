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


def _check_qdq(b, w, layout=1):
    wd = w.cuda()
    batch, N, K = (1, *w.shape) if w.dim() == 2 else w.shape
    w_out, qw, colamax = b.weight_qdq(wd, layout=layout)
    torch.cuda.synchronize()
    wb = bits(w).reshape(batch, N, K)
    got_out = bits(w_out).reshape(batch, N, K)
    codes = unpack_codes(qw.codes.cpu().numpy())
    sc = qw.scales.cpu().numpy()
    scales = untile_scales(sc, batch * N, K) if layout == 1 else sc[: batch * N * K // 16].reshape(batch * N, K // 16)
    for e in range(batch):
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
