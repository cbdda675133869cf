"""moe_grouped_w4a4_rac_gemm (each expert its own RAC linear, one call)
against the oracle, on ragged groups with empty experts and on the full MoE
expert-FFN workload (sampled rows)."""
import numpy as np
import pytest
import torch

import oracle
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import REL_TOL, bits, need_gpu, rel_err

pytestmark = pytest.mark.gpu


def _run(b, x_perm, offsets, w, k):
    xd, wd = x_perm.cuda(), w.cuda()
    _, qw, colamax = b.weight_qdq(wd)
    off = torch.from_numpy(np.asarray(offsets, np.int64)).cuda()
    y, masks = b.moe_rac(xd, off, wd, qw, colamax, k)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    return y.cpu().numpy(), masks.cpu().numpy()


@pytest.mark.parametrize("counts,N,K,k", [([70, 0, 130, 5], 128, 256, 50.0),
                                          ([0, 300, 128, 129, 0], 256, 192, 25.0),
                                          ([1], 128, 64, 100.0), ([0, 0, 17], 128, 128, 0.0)])
def test_moe_small_matches_oracle(counts, N, K, k):
    b = need_gpu()
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    E = len(counts)
    x = S.activations(int(off[-1]), K, seed=E)
    w = S.weights(N, K, seed=E, batch=E)
    y, masks = _run(b, x, off, w, k)
    y_ref, masks_ref, _ = oracle.moe_rac(bits(x), off, bits(w).reshape(E, N, K), k)
    assert np.array_equal(masks, masks_ref)
    assert rel_err(y, y_ref) < REL_TOL


def test_moe_full_size_sampled():
    """8192 tokens, top-8 of 64 Zipf(1.1) experts, up projection 2048 -> 1024."""
    b = need_gpu()
    tok, off = S.moe_routing(8192)
    x = S.activations(8192, 2048)[torch.from_numpy(tok)]
    w = S.weights(1024, 2048, batch=64)
    y, masks = _run(b, x, off, w, 50.0)
    xb, wb = bits(x), bits(w).reshape(64, 1024, 2048)
    rng = np.random.default_rng(0)
    for e in [0, 1, 7, 31, 63] + list(rng.choice(64, 3, replace=False)):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        rows = np.unique(np.concatenate([[0, r1 - r0 - 1], rng.integers(0, r1 - r0, 24)]))
        ref = oracle.rac_linear(xb[r0:r1], wb[e], 50.0, rows=rows)
        assert np.array_equal(masks[e], ref["mask"])
        assert rel_err(y[r0:r1][rows], ref["y"]) < REL_TOL
