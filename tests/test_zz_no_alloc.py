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
def test_static_scratch_matches_workspace_quantize(M, K):
    b = _need()
    from precision_rl_rollout_nvfp4_b200 import synthetic as S
    x = S.activations(M, K, seed=M + 1).cuda()
    ref_q, ref_score, ref_cm = b.quantize(x, layout=1)
    torch.cuda.synchronize()
    for _ in range(2):
        q, score, cm = b.quantize_static_ws(x, layout=1)
        torch.cuda.synchronize()
        assert b.stream_status() == 0
        assert torch.equal(q.codes, ref_q.codes)
        assert torch.equal(q.scales, ref_q.scales)
        assert torch.equal(q.tensor_scale, ref_q.tensor_scale)
        assert torch.equal(score, ref_score)
        assert torch.equal(cm, ref_cm)


def test_static_scratch_refuses_oversize_shapes():
    b = _need()
    x = torch.zeros(32768, 4096, dtype=torch.bfloat16, device="cuda")   # needs ~12.6 MB of scratch
    with pytest.raises(b.NvFP4Error) as e:
        b.quantize_static_ws(x, layout=1)
    assert e.value.status == 4          # NVFP4_ERR_WORKSPACE
