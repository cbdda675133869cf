"""CPU oracle for the NVFP4 W4A4 + RAC rollout path.  TEST INFRASTRUCTURE.

This package is the plain, slow reference the CUDA library is checked
against.  Only the tests, the smoke check in ``__graft_entry__`` and the CPU
baseline leg of ``bench.py`` may import it; the library itself never does,
and there is no CPU fallback of the product path through it.  It shares no
code, tables or constants with the CUDA sources.

Modules
  formats  E2M1 / E4M3 / bf16 encoders and decoders from their definitions.
  nvfp4    tensor Q / DQ with 16-element blocks and an fp32 tensor scale.
  rac      residual, channel score, top-k% mask, second-pass quantization,
           fp64 products, the trainer-side weight fake quantization, MoE.
  scalar   an independent pure-Python restatement for tiny shapes.
  qat      the trainer-side QAT linear (W4A16, symmetric W4A4 ablation) with
           the straight-through gradient.
  mxfp8    the FP8 comparator's operand format (E4M3 elements, one UE8M0
           scale per 32 elements) and its fp64 product.

Floating point: the quantization steps are fp32 operations rounded to nearest
even (numpy float32 arithmetic, no fused multiply-add, no flush to zero),
because the codes they decide must match the kernels bit for bit; the output
products are exact block values multiplied and summed in fp64.

Parity pins (see tests/test_oracle_*.py): the element formats against their
closed-form bit-field definitions and an exhaustive nearest search, the count
of 8 magnitudes per sign, round trips of every code under every scale,
QDQ idempotence, the error bound of the grid, brute-force top-k on tiny
inputs, k = 0 / k = 100 reductions, the fp64 product against a plain loop,
the scalar restatement, and "RAC error <= plain W4A4 error" against the bf16
product.  The MXFP8 comparator format is pinned by closed-form blocks (a
block maximum of 448 2^k gives scale 2^k), round trips of every E4M3 code,
saturation, ties, signed zeros and its own scalar restatement.  The opt-in variants are pinned the same way: W_sel from the NVFP4
weights (scalar restatement, weights already on the grid), a channel mask
kept from an earlier call (equal to the per-call linear under its own mask;
an empty mask gives the plain product), and the QAT linear (grid-exact
operands reduce it to the plain linear and the textbook gradients).
"""
from . import formats, mxfp8, nvfp4, qat, rac, scalar  # noqa: F401
from .formats import (bf16_to_f32, e2m1_decode, e2m1_encode, e4m3_decode,  # noqa: F401
                      e4m3_encode, f32_to_bf16)
from .nvfp4 import amax, dequantize, quantize, quantize_tensor, tensor_scale  # noqa: F401
from .rac import (channel_score, column_amax, gather_quantize, gemm_fp64,  # noqa: F401
                  moe_rac, n_selected, padded_width, quantize_activations,
                  rac_linear, residual, select_channels, weight_qdq,
                  weight_sel_from_fp4)
