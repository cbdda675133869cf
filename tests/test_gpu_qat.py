"""Trainer-side QAT linear (W4A16 and the symmetric W4A4 ablation): the
fake-quantized operands bit for bit, and the bf16 forward and
straight-through backward against the oracle's fp64 products."""
import numpy as np
import pytest
import torch

import oracle
from oracle import qat as oqat
from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import bits, need_gpu, rel_err

pytestmark = pytest.mark.gpu

# bf16 outputs of library GEMMs of exact bf16 operands: the final bf16
# rounding (2^-9 relative), fp32 summation, and possibly bf16-rounded split-K
# partial sums (torch allows reduced-precision bf16 reductions by default); a
# wrong operand or a missing fake quantizer is off by far more
GEMM_TOL = 1e-2


@pytest.mark.parametrize("M,K,N", [(64, 256, 128), (300, 192, 144), (1024, 2048, 2048)])
@pytest.mark.parametrize("act_quant", [False, True])
def test_qat_linear_matches_oracle(M, K, N, act_quant):
    b = need_gpu()
    x = S.activations(M, K, seed=M)
    w = S.weights(N, K, seed=M)
    dy = (0.01 * torch.randn(M, N, generator=torch.Generator().manual_seed(M))).to(torch.bfloat16)
    xd = x.cuda().requires_grad_(True)
    wd = w.cuda().requires_grad_(True)
    y = b.qat_linear(xd, wd, act_quant=act_quant)
    y.backward(dy.cuda())
    torch.cuda.synchronize()
    ref = oqat.qat_linear(bits(x), bits(w), dy.float().numpy(), act_quant=act_quant)
    # the fake-quantized operands are the oracle's, bit for bit
    assert np.array_equal(bits(b.fake_quant(wd.detach())), ref["w_q"])
    if act_quant:
        assert np.array_equal(bits(b.fake_quant(xd.detach())), ref["x_q"])
    assert rel_err(y.detach().float().cpu().numpy(), ref["y"]) < GEMM_TOL
    assert rel_err(xd.grad.float().cpu().numpy(), ref["dx"]) < GEMM_TOL
    assert rel_err(wd.grad.float().cpu().numpy(), ref["dw"]) < GEMM_TOL


def test_fake_quant_gradient_is_straight_through():
    b = need_gpu()
    w = S.weights(64, 128, seed=9).cuda().requires_grad_(True)
    g = torch.randn(64, 128, device="cuda").to(torch.bfloat16)
    b.fake_quant(w).backward(g)
    torch.cuda.synchronize()
    assert torch.equal(w.grad, g)
