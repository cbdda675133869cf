"""Device-side bounded waits: a wait that nothing completes gives up after
its limit, records NVFP4_ERR_TIMEOUT, and the context stays usable."""
import time

import pytest
import torch

from tests.gpu_common import need_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    b = need_gpu()
    assert b.stream_status() == 0
    t0 = time.time()
    b.check_bounded_wait(200)
    status = b.stream_status()
    dt = time.time() - t0
    assert status == 6                 # NVFP4_ERR_TIMEOUT
    assert dt < 5.0
    assert b.stream_status() == 0      # the word is cleared once reported
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0    # the context still works


def test_invalid_arguments_rejected_before_launch():
    b = need_gpu()
    x = torch.zeros(64, 96, dtype=torch.bfloat16, device="cuda")   # K % 64 != 0
    with pytest.raises(b.NvFP4Error) as e:
        b.quantize(x)
    assert e.value.status == 3
    with pytest.raises(b.NvFP4Error):
        b.rac_select(torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda"),
                     b.NvFP4Tensor.empty(64, 64), torch.zeros(64, dtype=torch.float64, device="cuda"),
                     torch.zeros(64, device="cuda"), 101.0)
