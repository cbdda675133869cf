"""GPU element conversions (used by every quantizing kernel) against the
oracle, around every decision boundary and on random bit patterns."""
import numpy as np
import pytest
import torch

import oracle
from oracle import formats as F
from tests.gpu_common import need_gpu

pytestmark = pytest.mark.gpu


def _around(points, span, seed, n_random):
    rng = np.random.default_rng(seed)
    parts = []
    for p in points:
        b = np.float32(p).view(np.uint32).astype(np.int64)
        parts.append((np.arange(b - span, b + span + 1) & 0xFFFFFFFF).astype(np.uint32))
    parts.append(rng.integers(0, 2**32, n_random, dtype=np.uint64).astype(np.uint32))
    v = np.concatenate(parts).view(np.float32)
    return v[np.isfinite(v)]


def test_e2m1_conversion_matches_oracle():
    b = need_gpu()
    grid = F.E2M1_MAGNITUDES
    pts = list(grid) + list((grid[1:] + grid[:-1]) / 2)
    v = _around(pts, 1 << 15, 0, 1 << 23)
    v = np.concatenate([v, -v, np.float32([0.0, -0.0, np.inf, -np.inf, 1e38, -1e38, 1e-45, -1e-45])])
    got = b.encode_e2m1(torch.from_numpy(v).cuda()).cpu().numpy()
    want = oracle.e2m1_encode(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:8]], got[bad[:8]], want[bad[:8]])


def test_e4m3_conversion_matches_oracle():
    b = need_gpu()
    table = F.E4M3_POSITIVE
    pts = list(table) + list((table[1:] + table[:-1]) / 2)
    v = np.abs(_around(pts, 1 << 11, 1, 1 << 22))
    v = np.concatenate([v, np.float32([0.0, np.inf, 3e38, 1e-45])])
    got = b.encode_e4m3(torch.from_numpy(v).cuda()).cpu().numpy()
    want = oracle.e4m3_encode(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:8]], got[bad[:8]], want[bad[:8]])
