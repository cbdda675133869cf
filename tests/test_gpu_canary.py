"""Out-of-bounds writes: every output buffer of every C-ABI entry point sits
between two 4 KiB guard bands filled with a canary pattern, on ragged shapes
(rows and columns that are not multiples of the kernels' tiles); after the
calls every guard byte must still hold the pattern.  compute-sanitizer is not
available here, so this is the host-observable check of the kernels' stores."""
import ctypes

import numpy as np
import pytest
import torch

from precision_rl_rollout_nvfp4_b200 import synthetic as S
from tests.gpu_common import need_gpu

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5


class Guarded:
    """Device buffers carved out of one allocation, each between guards."""

    def __init__(self):
        self.parts = []

    def take(self, nbytes, dtype=torch.uint8):
        nbytes = max(int(nbytes), 16)
        nbytes = (nbytes + 15) // 16 * 16
        raw = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.parts.append((raw, nbytes))
        return raw[GUARD:GUARD + nbytes].view(dtype)

    def check(self):
        torch.cuda.synchronize()
        for raw, n in self.parts:
            r = raw.cpu().numpy()
            assert np.all(r[:GUARD] == CANARY) and np.all(r[GUARD + n:] == CANARY)


def _nv(b, g, rows, cols, layout=1, n_scales=1):
    T = b._Tensor
    codes = g.take(rows * cols // 2)
    scales = g.take(b.scale_bytes(rows, cols, layout))
    st = g.take(4 * n_scales, torch.float32)
    return T(codes.data_ptr(), scales.data_ptr(), st.data_ptr(), rows, cols, layout)


@pytest.mark.parametrize("M,K,N,k", [(300, 192, 144, 50.0), (1, 64, 16, 100.0), (130, 1088, 272, 12.5),
                                     (300, 512, 144, 25.0)])
def test_dense_calls_write_inside_their_buffers(M, K, N, k):
    b = need_gpu()
    lib, P = b._lib, ctypes.c_void_p
    x = S.activations(M, K, seed=M).cuda()
    w = S.weights(N, K, seed=N).cuda()
    s = b._stream()
    g = Guarded()
    # weight_qdq -> W', Q(W), colamax
    w_out = g.take(2 * N * K, torch.bfloat16)
    qw = _nv(b, g, N, K)
    cm_w = g.take(4 * K, torch.float32)
    ws = torch.empty(b.workspace_size(b.OP_WEIGHT_QDQ, 0, N, K, 1), dtype=torch.uint8, device="cuda")
    assert lib.weight_qdq(P(w.data_ptr()), N, K, K, 1, P(w_out.data_ptr()), ctypes.byref(qw), P(cm_w.data_ptr()),
                          P(ws.data_ptr()), ws.numel(), s) == 0
    # nvfp4_quantize -> Q(X), scores, residual column maxima
    qx = _nv(b, g, M, K)
    score = g.take(8 * K, torch.float64)
    rcm = g.take(4 * K, torch.float32)
    wsq = torch.empty(b.workspace_size(b.OP_QUANTIZE, M, 0, K), dtype=torch.uint8, device="cuda")
    assert lib.nvfp4_quantize(P(x.data_ptr()), M, K, K, None, ctypes.byref(qx), P(score.data_ptr()),
                              P(rcm.data_ptr()), P(wsq.data_ptr()), wsq.numel(), s) == 0
    # rac_select -> mask, sel, Q(dX_sel)
    n_sel = b.rac_nsel(k, K)
    width = b.rac_width(n_sel)
    mask = g.take(K)
    sel = g.take(4 * n_sel, torch.int32)
    qr = _nv(b, g, M, width)
    n_out = ctypes.c_int64(-1)
    wss = torch.empty(b.workspace_size(b.OP_RAC_SELECT, M, 0, K), dtype=torch.uint8, device="cuda")
    assert lib.rac_select(P(x.data_ptr()), M, K, K, ctypes.byref(qx), P(score.data_ptr()), P(rcm.data_ptr()),
                          float(k), P(mask.data_ptr()), P(sel.data_ptr()), ctypes.byref(n_out), ctypes.byref(qr),
                          P(wss.data_ptr()), wss.numel(), s) == 0
    # rac_weight_quant and rac_weight_quant_fp4 -> Q(W_sel)
    qs = _nv(b, g, N, width)
    assert lib.rac_weight_quant(P(w.data_ptr()), N, K, K, P(sel.data_ptr()), n_sel, P(cm_w.data_ptr()),
                                ctypes.byref(qs), s) == 0
    dq_cm = g.take(4 * K, torch.float32)
    assert lib.nvfp4_dq_colamax(ctypes.byref(qw), 1, P(dq_cm.data_ptr()), s) == 0
    qs4 = _nv(b, g, N, width)
    assert lib.rac_weight_quant_fp4(ctypes.byref(qw), P(sel.data_ptr()), n_sel, P(dq_cm.data_ptr()),
                                    ctypes.byref(qs4), s) == 0
    # the GEMM, fp32 and bf16 Y, with a row stride wider than N
    for dt, esz in ((0, 4), (1, 2)):
        ldy = N + 16
        y = g.take(esz * M * ldy)
        assert lib.w4a4_gemm_quantized(ctypes.byref(qx), ctypes.byref(qw), ctypes.byref(qr), ctypes.byref(qs),
                                       P(y.data_ptr()), dt, ldy, s) == 0
    # the FP8 comparator
    if K % 256 == 0:
        MT = b._MxTensor
        def mx(rows):
            c = g.take(rows * K)
            sc = g.take(b._lib.mxfp8_scale_bytes(rows, K, 1))
            return MT(c.data_ptr(), sc.data_ptr(), rows, K, 1)
        qa8, qb8 = mx(M), mx(N)
        assert lib.mxfp8_quantize(P(x.data_ptr()), M, K, K, ctypes.byref(qa8), s) == 0
        assert lib.mxfp8_quantize(P(w.data_ptr()), N, K, K, ctypes.byref(qb8), s) == 0
        y8 = g.take(4 * M * N)
        assert lib.w8a8_gemm_quantized(ctypes.byref(qa8), ctypes.byref(qb8), P(y8.data_ptr()), 0, N, s) == 0
    assert b.stream_status() == 0
    g.check()


def test_moe_call_writes_inside_its_buffers():
    b = need_gpu()
    lib, P = b._lib, ctypes.c_void_p
    counts = [70, 0, 130, 5, 300]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    E, N, K, k = len(counts), 256, 192, 50.0
    T = int(off[-1])
    x = S.activations(T, K, seed=3).cuda()
    w = S.weights(N, K, seed=3, batch=E).cuda()
    _, qw_t, cm = b.weight_qdq(w)
    offd = torch.from_numpy(off).cuda()
    g = Guarded()
    y = g.take(4 * T * N, torch.float32)
    masks = g.take(E * K)
    ws = torch.empty(b.workspace_size(b.OP_MOE, T, N, K, E), dtype=torch.uint8, device="cuda")
    qw = qw_t.c()
    assert lib.moe_grouped_w4a4_rac_gemm(P(x.data_ptr()), T, K, P(offd.data_ptr()), E, P(w.data_ptr()), N,
                                         ctypes.byref(qw), P(cm.data_ptr()), float(k), P(y.data_ptr()), 0,
                                         P(masks.data_ptr()), P(ws.data_ptr()), ws.numel(), b._stream()) == 0
    assert b.stream_status() == 0
    g.check()
