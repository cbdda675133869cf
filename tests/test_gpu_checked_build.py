"""The whole path in the index-checked build (libnvfp4rac_checked.so, compiled
with NVFP4_CHECKS): on small ragged shapes every kernel's stores and gathered
loads test their indices, and a failure would make nvfp4_stream_status return
NVFP4_ERR_BOUNDS.  The calls run in a child process (one library per
process), which also checks the results against the oracle."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import numpy as np, torch
import oracle
from precision_rl_rollout_nvfp4_b200 import binding as b, synthetic as S
from tests.gpu_common import rel_err
assert b._lib.nvfp4_build_flags() & 1, "not the checked build"
for (M, K, N, k) in [(300, 192, 144, 50.0), (1, 64, 16, 100.0), (130, 1088, 272, 12.5), (257, 512, 400, 25.0)]:
    x, w = S.activations(M, K, seed=M), S.weights(N, K, seed=N)
    for wsel in ("bf16", "fp4"):
        y, st = b.rac_linear(x.cuda(), w.cuda(), k, wsel=wsel)
        torch.cuda.synchronize()
        assert b.stream_status() == 0, (M, K, N, wsel)
        ref = oracle.rac_linear(S.bf16_bits(x), S.bf16_bits(w), k, wsel_source=wsel)
        assert np.array_equal(st["mask"].cpu().numpy(), ref["mask"])
        assert rel_err(y.cpu().numpy(), ref["y"]) < 1e-3
    if K % 256 == 0:
        qa, qb = b.mxfp8_quantize(x.cuda()), b.mxfp8_quantize(w.cuda())
        b.w8a8_gemm(qa, qb)
        torch.cuda.synchronize()
        assert b.stream_status() == 0
counts = [70, 0, 130, 5, 300]
off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
E, N, K = len(counts), 256, 192
x = S.activations(int(off[-1]), K, seed=3)
w = S.weights(N, K, seed=3, batch=E)
_, qw, cm = b.weight_qdq(w.cuda())
y, masks = b.moe_rac(x.cuda(), torch.from_numpy(off).cuda(), w.cuda(), qw, cm, 50.0)
torch.cuda.synchronize()
assert b.stream_status() == 0
y_ref, m_ref, _ = oracle.moe_rac(S.bf16_bits(x), off, S.bf16_bits(w).reshape(E, N, K), 50.0)
assert np.array_equal(masks.cpu().numpy(), m_ref)
assert rel_err(y.cpu().numpy(), y_ref) < 1e-3
q, sc, cmx = b.quantize_static_ws(S.activations(200, 256, seed=9).cuda())
torch.cuda.synchronize()
assert b.stream_status() == 0
print("checked build ok")
'''


def test_whole_path_in_checked_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = os.path.join(ROOT, "precision_rl_rollout_nvfp4_b200", "libnvfp4rac_checked.so")
    assert os.path.exists(lib), "build the checked library (build_lib.build(checked=True))"
    env = dict(os.environ, NVFP4_LIB="checked", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "checked build ok" in r.stdout
