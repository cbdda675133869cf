"""Shared fixtures of the GPU parity tests."""
import numpy as np
import pytest
import torch

from precision_rl_rollout_nvfp4_b200 import synthetic as S

REL_TOL = 1e-3     # max relative error of Y against the fp64 oracle


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from precision_rl_rollout_nvfp4_b200 import binding
    return binding


def rel_err(y_gpu, y_ref):
    """max_ij |Y - Y_ref| / max(|Y_ref_ij|, 1e-3 max|Y_ref|): element-wise
    relative error with a floor so cancellation near zero does not dominate."""
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    floor = 1e-3 * np.max(np.abs(y_ref)) if y_ref.size else 0.0
    den = np.maximum(np.abs(y_ref), floor)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(y_gpu - y_ref) / den)) if y_ref.size else 0.0


def bits(t):
    return S.bf16_bits(t.cpu())
