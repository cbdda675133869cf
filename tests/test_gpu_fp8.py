"""The FP8 comparator through the C ABI against the MXFP8 oracle: codes and
UE8M0 scales bit for bit, and the kind::mxf8f6f4 tensor-core GEMM within the
1e-3 bar against the fp64 product of the same dequantized operands."""
import numpy as np
import pytest
import torch

from oracle import mxfp8 as mx
from oracle.formats import bf16_to_f32
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import REL_TOL, bits, need_gpu, rel_err

pytestmark = pytest.mark.gpu


def _tiled_index(rows, cols):
    r = np.arange(rows, dtype=np.int64)[:, None]
    c = np.arange(cols // 32, dtype=np.int64)[None, :]
    return ((r >> 7) * (cols // 128) + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3)


def _check_q(b, x, layout):
    M, K = x.shape
    q = b.mxfp8_quantize(x.cuda(), layout=layout)
    torch.cuda.synchronize()
    codes, scales = mx.quantize(bf16_to_f32(S.bf16_bits(x)))
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    sc = q.scales.cpu().numpy()
    got = sc[_tiled_index(M, K)] if layout == 1 else sc.reshape(M, K // 32)
    assert np.array_equal(got, scales)
    return q, codes, scales


@pytest.mark.parametrize("M,K", [(64, 512), (1, 256), (300, 768), (4096, 2048)])
@pytest.mark.parametrize("layout", [0, 1])
def test_mxfp8_quantize_matches_oracle(M, K, layout):
    b = need_gpu()
    _check_q(b, S.activations(M, K, seed=M + K), layout)


def test_mxfp8_quantize_edges():
    b = need_gpu()
    rng = np.random.default_rng(2)
    x = rng.standard_normal((40, 256)).astype(np.float32)
    x[0, :32] = 0.0                                   # zero block
    x[1, 5] = -0.0
    x[2, :32] *= 1e-38                                # subnormal-range block
    x[3, 0] = 500.0                                   # saturates to 448 2^E
    x[4, :32] = np.float32(1.0625)                    # ties
    x[5, 32:64] = 3e38
    xt = torch.from_numpy(x).to(torch.bfloat16)
    _check_q(b, xt, 1)


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (300, 144, 512), (1, 16, 256), (1024, 2048, 4096),
                                   (4000, 2000, 512), (2560, 1040, 256),   # CTA-pair kernel, ragged
                                   (256, 11008, 4096)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_w8a8_gemm_matches_oracle(M, N, K, out):
    b = need_gpu()
    x = S.activations(M, K, seed=M)
    w = S.weights(N, K, seed=N)
    qa, ac, asc = _check_q(b, x, 1)
    qb, bc, bsc = _check_q(b, w, 1)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    y = b.w8a8_gemm(qa, qb, out_dtype=dt)
    torch.cuda.synchronize()
    assert b.stream_status() == 0
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(1).integers(0, M, 64)]))
    ref = mx.gemm_fp64(ac, asc, bc, bsc, rows=rows)
    tol = REL_TOL if out == "f32" else REL_TOL + 2.0 ** -8
    assert rel_err(y.float().cpu().numpy()[rows], ref) < tol
