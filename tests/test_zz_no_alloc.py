"""nvfp4_quantize_static_ws: the quantizer for callers that cannot allocate.

Callers such as plugin hooks that only receive input and output pointers, or
processes whose device memory is fully reserved by another allocator, cannot
pass a workspace.  This entry point uses a fixed device array inside the
library instead.  The test compares it, through the C ABI, with the
workspace-taking nvfp4_quantize on the same input, bit for bit (the tolerance
of the quantizer tests), over two calls in a row (the array keeps the first
call's contents), and checks that a shape needing more scratch than the array
holds is refused before anything runs.  It lives in a file of its own that
pytest collects last.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _need():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from precision_rl_rollout_nvfp4_b200 import binding
    return binding


@pytest.mark.parametrize("M,K", [(4096, 2048), (300, 192)])
@pytest.mark.parametrize("scores", [True, "colamax", False])
@pytest.mark.parametrize("caller_amax", [False, True])
def test_static_scratch_matches_workspace_quantize(M, K, scores, caller_amax):
    b = _need()
    from precision_rl_rollout_nvfp4_b200 import synthetic as S
    # a call of another shape first, so the array holds that call's leftover
    # partial maxima and strip counters when the calls under test run
    other = S.activations(1000, 640, seed=7).cuda()
    b.quantize_static_ws(other, layout=1, scores=True)
    x = S.activations(M, K, seed=M + 1).cuda()
    amax = x.float().abs().max().reshape(1) if caller_amax else None
    ref_q, ref_score, ref_cm = b.quantize(x, amax=amax, layout=1, scores=scores)
    torch.cuda.synchronize()
    for _ in range(2):
        q, score, cm = b.quantize_static_ws(x, amax=amax, layout=1, scores=scores)
        torch.cuda.synchronize()
        assert b.stream_status() == 0
        assert torch.equal(q.codes, ref_q.codes)
        assert torch.equal(q.scales, ref_q.scales)
        assert torch.equal(q.tensor_scale, ref_q.tensor_scale)
        if scores is True:
            assert torch.equal(score, ref_score)
        if scores:
            assert torch.equal(cm, ref_cm)


def test_static_scratch_refuses_oversize_shapes():
    b = _need()
    x = torch.zeros(32768, 4096, dtype=torch.bfloat16, device="cuda")   # needs ~12.6 MB of scratch
    with pytest.raises(b.NvFP4Error) as e:
        b.quantize_static_ws(x, layout=1)
    assert e.value.status == 4          # NVFP4_ERR_WORKSPACE
