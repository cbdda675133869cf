"""ctypes binding of libnvfp4rac.so (C ABI in include/nvfp4rac.h).

Argument marshalling only: torch provides device memory and the current
stream; every step of the path runs in the library's CUDA kernels.  Importing
this module fails loudly when the library is missing -- there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# NVFP4_LIB=checked loads the index-checked build (libnvfp4rac_checked.so)
LIB_PATH = os.path.join(_PKG, "libnvfp4rac_checked.so" if os.environ.get("NVFP4_LIB") == "checked"
                        else "libnvfp4rac.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m precision_rl_rollout_nvfp4_b200.build_lib` (needs nvcc)")
_lib = ctypes.CDLL(LIB_PATH)

OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "misaligned", 3: "unsupported shape",
                4: "workspace too small", 5: "CUDA error", 6: "timeout", 7: "not sm_100",
                8: "index check failed"}
OP_QUANTIZE, OP_RAC_SELECT, OP_GEMM, OP_MOE, OP_WEIGHT_QDQ = range(5)
EXPORTS = ["nvfp4_scale_bytes", "nvfp4_workspace_size", "nvfp4_quantize", "rac_select",
           "nvfp4_rac_nsel", "nvfp4_rac_width", "rac_weight_quant", "w4a4_rac_gemm",
           "w4a4_gemm_quantized", "moe_grouped_w4a4_rac_gemm", "weight_qdq",
           "nvfp4_encode_e2m1", "nvfp4_encode_e4m3", "nvfp4_stream_status",
           "nvfp4_check_bounded_wait", "nvfp4_status_string", "nvfp4_quantize_static_ws",
           "nvfp4_dq_colamax", "rac_weight_quant_fp4", "rac_select_channels", "rac_residual_quant",
           "rac_sel_tensor_scale", "mxfp8_scale_bytes", "mxfp8_quantize", "w8a8_gemm_quantized",
           "nvfp4_build_flags", "rac_quantize_select", "rac_second_pass"]


class _Tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("scale_layout", ctypes.c_int32)]


class _MxTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("scale_layout", ctypes.c_int32)]


P, I64, I32, F32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
TP = ctypes.POINTER(_Tensor)
MP = ctypes.POINTER(_MxTensor)
_sig = {
    "nvfp4_scale_bytes": (SZ, [I64, I64, I32]),
    "nvfp4_workspace_size": (SZ, [I32, I64, I64, I64, I32]),
    "nvfp4_quantize": (I32, [P, I64, I64, I64, P, TP, P, P, P, SZ, P]),
    "nvfp4_quantize_static_ws": (I32, [P, I64, I64, I64, P, TP, P, P, P]),
    "rac_select": (I32, [P, I64, I64, I64, TP, P, P, F32, P, P, ctypes.POINTER(I64), TP, P, SZ, P]),
    "nvfp4_rac_nsel": (I64, [F32, I64]),
    "nvfp4_rac_width": (I64, [I64]),
    "rac_weight_quant": (I32, [P, I64, I64, I64, P, I64, P, TP, P]),
    "nvfp4_dq_colamax": (I32, [TP, I32, P, P]),
    "rac_select_channels": (I32, [P, P, I64, F32, P, P, ctypes.POINTER(I64), P, P]),
    "rac_residual_quant": (I32, [P, I64, I64, I64, TP, P, I64, TP, P]),
    "rac_sel_tensor_scale": (I32, [P, I64, P, I64, P, P]),
    "rac_weight_quant_fp4": (I32, [TP, P, I64, P, TP, P]),
    "w4a4_rac_gemm": (I32, [TP, TP, P, I64, P, I64, I64, TP, P, P, I32, I64, P, SZ, P]),
    "w4a4_gemm_quantized": (I32, [TP, TP, TP, TP, P, I32, I64, P]),
    "moe_grouped_w4a4_rac_gemm": (I32, [P, I64, I64, P, I32, P, I64, TP, P, F32, P, I32, P, P, SZ, P]),
    "weight_qdq": (I32, [P, I64, I64, I64, I32, P, TP, P, P, SZ, P]),
    "nvfp4_encode_e2m1": (I32, [P, P, I64, P]),
    "nvfp4_encode_e4m3": (I32, [P, P, I64, P]),
    "nvfp4_stream_status": (I32, [P]),
    "nvfp4_check_bounded_wait": (I32, [I32, P]),
    "nvfp4_status_string": (ctypes.c_char_p, [I32]),
    "mxfp8_scale_bytes": (SZ, [I64, I64, I32]),
    "nvfp4_build_flags": (I32, []),
    "rac_quantize_select": (I32, [P, I64, I64, I64, P, TP, P, P, F32, P, P, ctypes.POINTER(I64), P, P, SZ, P]),
    "rac_second_pass": (I32, [P, I64, I64, I64, TP, P, I64, TP, P, I64, I64, TP, P, TP, P]),
    "mxfp8_quantize": (I32, [P, I64, I64, I64, MP, P]),
    "w8a8_gemm_quantized": (I32, [MP, MP, P, I32, I64, P]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


class NvFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_lib.nvfp4_status_string(status).decode()} (status {status})")
        self.status = status


def _check(status: int, where: str):
    if status != OK:
        raise NvFP4Error(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def scale_bytes(rows: int, cols: int, layout: int) -> int:
    return int(_lib.nvfp4_scale_bytes(rows, cols, layout))


def workspace_size(op: int, M: int = 0, N: int = 0, K: int = 0, E: int = 1) -> int:
    return int(_lib.nvfp4_workspace_size(op, M, N, K, E))


def rac_nsel(k_percent: float, K: int) -> int:
    return int(_lib.nvfp4_rac_nsel(k_percent, K))


def rac_width(n_sel: int) -> int:
    return int(_lib.nvfp4_rac_width(n_sel))


@dataclass
class NvFP4Tensor:
    """Device buffers of one NVFP4 tensor (see nvfp4_tensor in the header)."""
    codes: torch.Tensor          # uint8 [rows, cols/2]
    scales: torch.Tensor         # uint8 [scale_bytes]
    tensor_scale: torch.Tensor   # float32 [n]
    rows: int
    cols: int
    layout: int

    @staticmethod
    def empty(rows, cols, layout=1, n_scales=1, device="cuda"):
        return NvFP4Tensor(torch.empty(rows, cols // 2, dtype=torch.uint8, device=device),
                           torch.empty(max(scale_bytes(rows, cols, layout), 1), dtype=torch.uint8, device=device),
                           torch.empty(n_scales, dtype=torch.float32, device=device),
                           rows, cols, layout)

    def c(self) -> _Tensor:
        return _Tensor(self.codes.data_ptr(), self.scales.data_ptr(), self.tensor_scale.data_ptr(),
                       self.rows, self.cols, self.layout)


class Workspace:
    """Grow-only device workspace reused across calls on one stream."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = torch.empty(0, dtype=torch.uint8, device=device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


_WS: dict = {}


def _ws(nbytes: int, device) -> torch.Tensor:
    key = torch.device(device)
    if key not in _WS:
        _WS[key] = Workspace(key)
    return _WS[key].get(nbytes)


def _bits(x: torch.Tensor) -> torch.Tensor:
    if x.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return x


def quantize(x, amax=None, layout=1, scores=True, out=None, stream=None):
    """Q(X) of bf16 x [M, K]; returns (qx, score fp64 [K], res_colamax fp32 [K])
    (the last two None when scores=False; scores="colamax" gives the residual
    column maxima without the scores)."""
    x = _bits(x)
    M, K = x.shape
    qx = out if out is not None else NvFP4Tensor.empty(M, K, layout, device=x.device)
    score = torch.empty(K, dtype=torch.float64, device=x.device) if scores is True else None
    colamax = torch.empty(K, dtype=torch.float32, device=x.device) if scores else None
    nbytes = workspace_size(OP_QUANTIZE, M, 0, K)
    ws = _ws(nbytes, x.device)
    st = qx.c()
    _check(_lib.nvfp4_quantize(_ptr(x), M, K, x.stride(0), _ptr(amax), ctypes.byref(st),
                               _ptr(score), _ptr(colamax), _ptr(ws), ws.numel(), _stream(stream)),
           "nvfp4_quantize")
    return qx, score, colamax


def quantize_static_ws(x, amax=None, layout=1, scores=True, out=None, stream=None):
    """Same as quantize() but through nvfp4_quantize_static_ws: no workspace
    is passed; the library uses its own fixed 4 MiB device scratch array."""
    x = _bits(x)
    M, K = x.shape
    qx = out if out is not None else NvFP4Tensor.empty(M, K, layout, device=x.device)
    score = torch.empty(K, dtype=torch.float64, device=x.device) if scores is True else None
    colamax = torch.empty(K, dtype=torch.float32, device=x.device) if scores else None
    st = qx.c()
    _check(_lib.nvfp4_quantize_static_ws(_ptr(x), M, K, x.stride(0), _ptr(amax), ctypes.byref(st),
                                         _ptr(score), _ptr(colamax), _stream(stream)),
           "nvfp4_quantize_static_ws")
    return qx, score, colamax


def rac_select(x, qx, score, colamax, k_percent, layout=1, stream=None):
    """Top-k% mask and Q(dX_sel); returns (mask u8 [K], sel i32 [n_sel],
    n_sel, q_res or None)."""
    x = _bits(x)
    M, K = x.shape
    n_sel = rac_nsel(k_percent, K)
    mask = torch.empty(K, dtype=torch.uint8, device=x.device)
    sel = torch.empty(max(n_sel, 1), dtype=torch.int32, device=x.device)
    q_res = NvFP4Tensor.empty(M, rac_width(n_sel), layout, device=x.device) if n_sel > 0 else None
    ws = _ws(workspace_size(OP_RAC_SELECT, M, 0, K), x.device)
    n_out = ctypes.c_int64(-1)
    qs, rs = qx.c(), (q_res.c() if q_res is not None else None)
    _check(_lib.rac_select(_ptr(x), M, K, x.stride(0), ctypes.byref(qs), _ptr(score), _ptr(colamax),
                           float(k_percent), _ptr(mask), _ptr(sel), ctypes.byref(n_out),
                           ctypes.byref(rs) if rs is not None else None, _ptr(ws), ws.numel(),
                           _stream(stream)), "rac_select")
    assert n_out.value == n_sel
    return mask, sel[:n_sel], n_sel, q_res


def quantize_select(x, k_percent, amax=None, layout=1, stream=None):
    """Q(X), scores and the top-k% selection in one pass (rac_quantize_select).
    Returns (qx, score, res_colamax, mask, sel [n_sel], n_sel, res_tensor_scale)."""
    x = _bits(x)
    M, K = x.shape
    n_sel = rac_nsel(k_percent, K)
    qx = NvFP4Tensor.empty(M, K, layout, device=x.device)
    score = torch.empty(K, dtype=torch.float64, device=x.device)
    colamax = torch.empty(K, dtype=torch.float32, device=x.device)
    mask = torch.empty(K, dtype=torch.uint8, device=x.device)
    sel = torch.empty(max(n_sel, 1), dtype=torch.int32, device=x.device)
    st = torch.empty(1, dtype=torch.float32, device=x.device)
    ws = _ws(workspace_size(OP_QUANTIZE, M, 0, K), x.device)
    n_out = ctypes.c_int64(-1)
    q = qx.c()
    _check(_lib.rac_quantize_select(_ptr(x), M, K, x.stride(0), _ptr(amax), ctypes.byref(q), _ptr(score),
                                    _ptr(colamax), float(k_percent), _ptr(mask), _ptr(sel), ctypes.byref(n_out),
                                    _ptr(st), _ptr(ws), ws.numel(), _stream(stream)), "rac_quantize_select")
    assert n_out.value == n_sel
    return qx, score, colamax, mask, sel[:n_sel], n_sel, st


def second_pass(x, qx, sel, n_sel, res_tensor_scale, w, qw, w_colamax, layout=1, stream=None):
    """Q(dX_sel) and Q(W_sel) in one call (rac_second_pass); w = None takes
    W_sel from qw (w_colamax = dq_colamax(qw)).  Returns (q_res, q_wsel)."""
    x = _bits(x)
    M, K = x.shape
    N = qw.rows
    q_res = NvFP4Tensor.empty(M, rac_width(n_sel), layout, device=x.device)
    q_res.tensor_scale.copy_(res_tensor_scale.reshape(1))
    q_ws = NvFP4Tensor.empty(N, rac_width(n_sel), layout, device=x.device)
    a, r, wq, ws_ = qx.c(), q_res.c(), qw.c(), q_ws.c()
    w = _bits(w) if w is not None else None
    _check(_lib.rac_second_pass(_ptr(x), M, K, x.stride(0), ctypes.byref(a), _ptr(sel), n_sel, ctypes.byref(r),
                                _ptr(w), N, w.stride(0) if w is not None else K, ctypes.byref(wq), _ptr(w_colamax),
                                ctypes.byref(ws_), _stream(stream)), "rac_second_pass")
    return q_res, q_ws


def rac_select_channels(score, colamax, k_percent, res_tensor_scale=None, stream=None):
    """Top-k% mask, sel and the residual tensor scale (the first half of
    rac_select).  Returns (mask, sel [n_sel], n_sel, res_tensor_scale)."""
    K = score.numel()
    n_sel = rac_nsel(k_percent, K)
    mask = torch.empty(K, dtype=torch.uint8, device=score.device)
    sel = torch.empty(max(n_sel, 1), dtype=torch.int32, device=score.device)
    st = res_tensor_scale if res_tensor_scale is not None else torch.empty(1, dtype=torch.float32,
                                                                           device=score.device)
    n_out = ctypes.c_int64(-1)
    _check(_lib.rac_select_channels(_ptr(score), _ptr(colamax), K, float(k_percent), _ptr(mask), _ptr(sel),
                                    ctypes.byref(n_out), _ptr(st), _stream(stream)), "rac_select_channels")
    assert n_out.value == n_sel
    return mask, sel[:n_sel], n_sel, st


def rac_sel_tensor_scale(colamax, sel, n_sel, out=None, stream=None):
    """RN(max_{j in sel} colamax_j / 2688) as a device fp32 [1]."""
    out = out if out is not None else torch.empty(1, dtype=torch.float32, device=colamax.device)
    _check(_lib.rac_sel_tensor_scale(_ptr(colamax), colamax.numel(), _ptr(sel), n_sel, _ptr(out),
                                     _stream(stream)), "rac_sel_tensor_scale")
    return out


def rac_residual_quant(x, qx, sel, n_sel, res_tensor_scale, layout=1, out=None, stream=None):
    """Q(dX_sel) (the second half of rac_select) with the residual tensor
    scale written by rac_select_channels."""
    x = _bits(x)
    M, K = x.shape
    q = out if out is not None else NvFP4Tensor.empty(M, rac_width(n_sel), layout, device=x.device)
    if out is None:
        q.tensor_scale.copy_(res_tensor_scale.reshape(1))
    a, qs = qx.c(), q.c()
    _check(_lib.rac_residual_quant(_ptr(x), M, K, x.stride(0), ctypes.byref(a), _ptr(sel), n_sel,
                                   ctypes.byref(qs), _stream(stream)), "rac_residual_quant")
    return q


def rac_weight_quant(w, sel, n_sel, w_colamax, layout=1, out=None, stream=None):
    w = _bits(w)
    N, K = w.shape
    q = out if out is not None else NvFP4Tensor.empty(N, rac_width(n_sel), layout, device=w.device)
    qs = q.c()
    _check(_lib.rac_weight_quant(_ptr(w), N, K, w.stride(0), _ptr(sel), n_sel, _ptr(w_colamax),
                                 ctypes.byref(qs), _stream(stream)), "rac_weight_quant")
    return q


def dq_colamax(q, batch=1, out=None, stream=None):
    """max_n |DQ(Q(W))_nk| per column of each of `batch` stacked matrices
    held in the NVFP4 tensor q (rows = batch * N).  Returns fp32 [batch, K]."""
    out = out if out is not None else torch.empty(batch, q.cols, dtype=torch.float32, device=q.codes.device)
    qc = q.c()
    _check(_lib.nvfp4_dq_colamax(ctypes.byref(qc), batch, _ptr(out), _stream(stream)), "nvfp4_dq_colamax")
    return out


def rac_weight_quant_fp4(qw, sel, n_sel, dq_cm, layout=1, out=None, stream=None):
    """Q(W_sel) re-quantized from the NVFP4 weight qw alone (dq_cm from
    dq_colamax(qw))."""
    q = out if out is not None else NvFP4Tensor.empty(qw.rows, rac_width(n_sel), layout, device=qw.codes.device)
    a, qs = qw.c(), q.c()
    _check(_lib.rac_weight_quant_fp4(ctypes.byref(a), _ptr(sel), n_sel, _ptr(dq_cm), ctypes.byref(qs),
                                     _stream(stream)), "rac_weight_quant_fp4")
    return q


def gemm_quantized(qa, qb, q_res=None, q_wsel=None, out_dtype=torch.float32, out=None, stream=None):
    y = out if out is not None else torch.empty(qa.rows, qb.rows, dtype=out_dtype, device=qa.codes.device)
    a, b = qa.c(), qb.c()
    r = q_res.c() if q_res is not None else None
    s = q_wsel.c() if q_wsel is not None else None
    _check(_lib.w4a4_gemm_quantized(ctypes.byref(a), ctypes.byref(b),
                                    ctypes.byref(r) if r is not None else None,
                                    ctypes.byref(s) if s is not None else None, _ptr(y),
                                    0 if y.dtype == torch.float32 else 1, y.stride(0), _stream(stream)),
           "w4a4_gemm_quantized")
    return y


def rac_gemm(qx, q_res, sel, n_sel, w, qw, w_colamax, out_dtype=torch.float32, out=None, stream=None):
    """w = None takes W_sel from qw (then w_colamax = dq_colamax(qw))."""
    N, K = qw.rows, qx.cols
    dev = qx.codes.device
    w = _bits(w) if w is not None else None
    y = out if out is not None else torch.empty(qx.rows, N, dtype=out_dtype, device=dev)
    ws = _ws(workspace_size(OP_GEMM, 0, N, K), dev)
    a, b = qx.c(), qw.c()
    r = q_res.c() if q_res is not None else None
    _check(_lib.w4a4_rac_gemm(ctypes.byref(a), ctypes.byref(r) if r is not None else None, _ptr(sel),
                              n_sel, _ptr(w), N, w.stride(0) if w is not None else K, ctypes.byref(b),
                              _ptr(w_colamax), _ptr(y),
                              0 if y.dtype == torch.float32 else 1, y.stride(0), _ptr(ws), ws.numel(),
                              _stream(stream)), "w4a4_rac_gemm")
    return y


def weight_qdq(w, want_q=True, want_colamax=True, layout=1, out=None, stream=None, ws=None):
    """W4A16 fake quantization of bf16 w [N, K] or [batch, N, K].  Returns
    (w_out bf16, qw or None, colamax fp32 [batch, K] or None).  ws: an
    optional caller-owned uint8 workspace (else a shared per-device one)."""
    w = _bits(w)
    batch, N, K = (1, *w.shape) if w.dim() == 2 else w.shape
    w_out = out if out is not None else torch.empty_like(w)
    qw = NvFP4Tensor.empty(batch * N, K, layout, n_scales=batch, device=w.device) if want_q else None
    colamax = torch.empty(batch, K, dtype=torch.float32, device=w.device) if want_colamax else None
    if ws is None:
        ws = _ws(workspace_size(OP_WEIGHT_QDQ, 0, N, K, batch), w.device)
    qs = qw.c() if qw is not None else None
    _check(_lib.weight_qdq(_ptr(w), N, K, K, batch, _ptr(w_out), ctypes.byref(qs) if qs is not None else None,
                           _ptr(colamax), _ptr(ws), ws.numel(), _stream(stream)), "weight_qdq")
    return w_out, qw, colamax


def moe_rac(x_perm, offsets, w, qw, w_colamax, k_percent, out_dtype=torch.float32, masks=True,
            out=None, stream=None):
    """Grouped RAC linears of E experts.  offsets: int64 [E+1] on the device.
    w = None takes every W_sel from qw (then w_colamax = dq_colamax(qw, E))."""
    x_perm = _bits(x_perm)
    T, K = x_perm.shape
    if w is not None:
        w = _bits(w)
        E, N, _ = w.shape
    else:
        E = w_colamax.shape[0]
        N = qw.rows // E
    y = out if out is not None else torch.empty(T, N, dtype=out_dtype, device=x_perm.device)
    mk = torch.empty(E, K, dtype=torch.uint8, device=x_perm.device) if masks else None
    ws = _ws(workspace_size(OP_MOE, T, N, K, E), x_perm.device)
    q = qw.c()
    _check(_lib.moe_grouped_w4a4_rac_gemm(_ptr(x_perm), T, K, _ptr(offsets), E, _ptr(w), N, ctypes.byref(q),
                                          _ptr(w_colamax), float(k_percent), _ptr(y),
                                          0 if y.dtype == torch.float32 else 1, _ptr(mk), _ptr(ws),
                                          ws.numel(), _stream(stream)), "moe_grouped_w4a4_rac_gemm")
    return y, mk


def rac_linear(x, w, k_percent, out_dtype=torch.float32, prepared=None, wsel="bf16", stream=None):
    """The whole rollout linear: weight prep (or `prepared` = (qw, colamax)),
    Q(X) + scores, mask + Q(dX_sel), Q(W_sel), and the two-segment GEMM.
    wsel="fp4" re-quantizes W_sel from Q(W) (colamax then holds the column
    maxima of DQ(Q(W)))."""
    assert wsel in ("bf16", "fp4")
    if prepared is None:
        _, qw, colamax = weight_qdq(w, want_colamax=wsel == "bf16", stream=stream)
        colamax = colamax[0] if wsel == "bf16" else dq_colamax(qw, stream=stream)[0]
    else:
        qw, colamax = prepared
    qx, score, rcm = quantize(x, stream=stream)
    mask, sel, n_sel, q_res = rac_select(x, qx, score, rcm, k_percent, stream=stream)
    y = rac_gemm(qx, q_res, sel, n_sel, w if wsel == "bf16" else None, qw, colamax, out_dtype=out_dtype,
                 stream=stream)
    return y, dict(qx=qx, score=score, res_colamax=rcm, mask=mask, sel=sel, n_sel=n_sel, q_res=q_res,
                   qw=qw, w_colamax=colamax)


class _FakeQuantSTE(torch.autograd.Function):
    """bf16(DQ(Q(t))) of a 2-D bf16 tensor with its own tensor scale, by the
    library's weight_qdq; backward: the straight-through estimator (the
    gradient crosses the fake quantizer unchanged)."""

    @staticmethod
    def forward(ctx, t):
        out, _, _ = weight_qdq(t.contiguous(), want_q=False, want_colamax=False)
        return out

    @staticmethod
    def backward(ctx, g):
        return g


def fake_quant(t):
    """Trainer-side NVFP4 fake quantization with a straight-through gradient."""
    return _FakeQuantSTE.apply(t)


def qat_linear(x, w, act_quant=False):
    """Trainer-side QAT linear Y = X' W'^T as a bf16 GEMM (torch matmul):
    W' = fake_quant(W) (asymmetric W4A16), and X' = fake_quant(X) for the
    symmetric W4A4 ablation (act_quant=True), else X' = X.  Autograd gives
    dX = dY W' and dW = dY^T X' through the straight-through quantizers."""
    wq = fake_quant(w)
    xq = fake_quant(x) if act_quant else x
    return xq @ wq.t()


@dataclass
class MxFP8Tensor:
    """Device buffers of one MXFP8 tensor (mxfp8_tensor in the header): the
    FP8 comparator's operand format."""
    codes: torch.Tensor          # uint8 [rows, cols] E4M3
    scales: torch.Tensor         # uint8 [mxfp8_scale_bytes] UE8M0
    rows: int
    cols: int
    layout: int

    @staticmethod
    def empty(rows, cols, layout=1, device="cuda"):
        return MxFP8Tensor(torch.empty(rows, cols, dtype=torch.uint8, device=device),
                           torch.empty(max(int(_lib.mxfp8_scale_bytes(rows, cols, layout)), 1), dtype=torch.uint8,
                                       device=device), rows, cols, layout)

    def c(self) -> _MxTensor:
        return _MxTensor(self.codes.data_ptr(), self.scales.data_ptr(), self.rows, self.cols, self.layout)


def mxfp8_quantize(x, layout=1, out=None, stream=None):
    """MXFP8 of bf16 x [M, K] (K % 256 == 0)."""
    x = _bits(x)
    M, K = x.shape
    q = out if out is not None else MxFP8Tensor.empty(M, K, layout, device=x.device)
    qs = q.c()
    _check(_lib.mxfp8_quantize(_ptr(x), M, K, x.stride(0), ctypes.byref(qs), _stream(stream)), "mxfp8_quantize")
    return q


def w8a8_gemm(qa, qb, out_dtype=torch.float32, out=None, stream=None):
    """Y = A B^T of two MXFP8 operands (the FP8 comparator GEMM)."""
    y = out if out is not None else torch.empty(qa.rows, qb.rows, dtype=out_dtype, device=qa.codes.device)
    a, b = qa.c(), qb.c()
    _check(_lib.w8a8_gemm_quantized(ctypes.byref(a), ctypes.byref(b), _ptr(y), 0 if y.dtype == torch.float32 else 1,
                                    y.stride(0), _stream(stream)), "w8a8_gemm_quantized")
    return y


def encode_e2m1(v: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    _check(_lib.nvfp4_encode_e2m1(_ptr(v), _ptr(out), v.numel(), _stream(stream)), "nvfp4_encode_e2m1")
    return out


def encode_e4m3(v: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    _check(_lib.nvfp4_encode_e4m3(_ptr(v), _ptr(out), v.numel(), _stream(stream)), "nvfp4_encode_e4m3")
    return out


def stream_status(stream=None) -> int:
    return int(_lib.nvfp4_stream_status(_stream(stream)))


def check_bounded_wait(timeout_ms: int, stream=None):
    _check(_lib.nvfp4_check_bounded_wait(timeout_ms, _stream(stream)), "nvfp4_check_bounded_wait")


def library_handle():
    return _lib


class RacLinearPlan:
    """All buffers of one rollout linear Y = X W^T (NVFP4 W4A4 + RAC) for fixed
    shapes, allocated once; every call below only enqueues library work on
    the current stream (no allocation, no host synchronization), so a step
    can also be captured in a CUDA graph.

    Steps (each one C ABI call):
      prepare_weight  weight_qdq(W) -> Q(W), colamax_W     (per weight sync)
      quantize        nvfp4_quantize(X) -> Q(X), scores, residual col-max
      select          rac_select -> mask, sel, Q(dX_sel)
                      (the steps call its halves, rac_select_channels and
                      rac_residual_quant, so the two gathers overlap)
      weight_select   rac_weight_quant -> Q(W_sel)
      gemm            w4a4_gemm_quantized -> Y
    reuse_step() keeps the channel mask, sel and Q(W_sel) of the last step
    that selected (the mask-reuse variant): it quantizes X with the residual
    column maxima only (no scores, no top-k), takes the residual tensor scale
    over the kept sel (rac_sel_tensor_scale), gathers Q(dX_sel) and runs the
    GEMM.
    With wsel="fp4" the weight preparation also takes the column maxima of
    DQ(Q(W)) (nvfp4_dq_colamax) and weight_select re-quantizes W_sel from
    Q(W) (rac_weight_quant_fp4) instead of reading the bf16 W.
    """

    def __init__(self, M, K, N, k_percent, out_dtype=torch.bfloat16, device="cuda", wsel="bf16"):
        assert wsel in ("bf16", "fp4")
        self.M, self.K, self.N, self.k = M, K, N, float(k_percent)
        self.wsel = wsel
        self.launches = dict(self.LAUNCHES)
        if wsel == "fp4":
            self.launches["prepare_weight"] += 1        # nvfp4_dq_colamax
        self.n_sel = rac_nsel(k_percent, K)
        self.width = rac_width(self.n_sel)
        dev = torch.device(device)
        self.qw = NvFP4Tensor.empty(N, K, 1, device=dev)
        self.w_out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        self.w_colamax = torch.empty(K, dtype=torch.float32, device=dev)
        self.dq_colamax = torch.empty(K, dtype=torch.float32, device=dev) if wsel == "fp4" else None
        self.qx = NvFP4Tensor.empty(M, K, 1, device=dev)
        self.score = torch.empty(K, dtype=torch.float64, device=dev)
        self.res_colamax = torch.empty(K, dtype=torch.float32, device=dev)
        self.mask = torch.empty(K, dtype=torch.uint8, device=dev)
        self.sel = torch.empty(max(self.n_sel, 1), dtype=torch.int32, device=dev)
        self.q_res = NvFP4Tensor.empty(M, self.width, 1, device=dev) if self.n_sel else None
        self.q_wsel = NvFP4Tensor.empty(N, self.width, 1, device=dev) if self.n_sel else None
        self.y = torch.empty(M, N, dtype=out_dtype, device=dev)
        sizes = [workspace_size(OP_QUANTIZE, M, 0, K), workspace_size(OP_RAC_SELECT, M, 0, K),
                 workspace_size(OP_WEIGHT_QDQ, 0, N, K, 1)]
        self.ws = torch.empty(max(sizes), dtype=torch.uint8, device=dev)
        # weight preparation may run concurrently on a side stream: own workspace
        self.ws_w = torch.empty(workspace_size(OP_WEIGHT_QDQ, 0, N, K, 1), dtype=torch.uint8, device=dev)
        self.side = torch.cuda.Stream(device=dev)
        self._fork = torch.cuda.Event()
        self._join = torch.cuda.Event()
        self._sel_ready = torch.cuda.Event()
        self._wsel_done = torch.cuda.Event()
        self.res_st = (self.q_res.tensor_scale if self.q_res is not None
                       else torch.empty(1, dtype=torch.float32, device=dev))
        self._qw, self._qx = self.qw.c(), self.qx.c()
        self._qr = self.q_res.c() if self.q_res is not None else None
        self._qs = self.q_wsel.c() if self.q_wsel is not None else None
        self._nout = ctypes.c_int64(-1)
        self.x = None
        self.w = None
        self.amax = None

    def bind(self, x, w, amax=None):
        """Point the plan at device inputs x [M, K] and w [N, K] (bf16).
        amax: optional device fp32 [1], a caller-supplied max|X| (e.g. from
        calibration or an earlier step); the quantizer then skips its amax
        pass (values above it saturate)."""
        assert tuple(x.shape) == (self.M, self.K) and tuple(w.shape) == (self.N, self.K)
        self.x, self.w = _bits(x), _bits(w)
        self.amax = amax
        return self

    def prepare_weight(self, stream=None):
        fp4 = self.wsel == "fp4"
        _check(_lib.weight_qdq(_ptr(self.w), self.N, self.K, self.w.stride(0), 1, _ptr(self.w_out),
                               ctypes.byref(self._qw), None if fp4 else _ptr(self.w_colamax),
                               _ptr(self.ws_w), self.ws_w.numel(), _stream(stream)), "weight_qdq")
        if fp4:
            _check(_lib.nvfp4_dq_colamax(ctypes.byref(self._qw), 1, _ptr(self.dq_colamax), _stream(stream)),
                   "nvfp4_dq_colamax")

    def quantize(self, stream=None, scores=True):
        """scores: True (scores and residual column maxima), False (codes
        only) or "colamax" (residual column maxima only)."""
        _check(_lib.nvfp4_quantize(_ptr(self.x), self.M, self.K, self.x.stride(0), _ptr(self.amax),
                                   ctypes.byref(self._qx),
                                   _ptr(self.score) if scores is True else None,
                                   _ptr(self.res_colamax) if scores else None, _ptr(self.ws),
                                   self.ws.numel(), _stream(stream)), "nvfp4_quantize")

    def select(self, stream=None):
        _check(_lib.rac_select(_ptr(self.x), self.M, self.K, self.x.stride(0), ctypes.byref(self._qx),
                               _ptr(self.score), _ptr(self.res_colamax), self.k, _ptr(self.mask),
                               _ptr(self.sel), ctypes.byref(self._nout),
                               ctypes.byref(self._qr) if self._qr is not None else None,
                               _ptr(self.ws), self.ws.numel(), _stream(stream)), "rac_select")

    def quantize_select(self, stream=None):
        """Q(X), scores, mask, sel and the residual tensor scale in one pass."""
        _check(_lib.rac_quantize_select(_ptr(self.x), self.M, self.K, self.x.stride(0), _ptr(self.amax),
                                        ctypes.byref(self._qx), _ptr(self.score), _ptr(self.res_colamax), self.k,
                                        _ptr(self.mask), _ptr(self.sel), ctypes.byref(self._nout),
                                        _ptr(self.res_st), _ptr(self.ws), self.ws.numel(), _stream(stream)),
               "rac_quantize_select")

    def second_pass(self, stream=None):
        """Q(dX_sel) and Q(W_sel) in one call."""
        if self.n_sel == 0:
            return
        fp4 = self.wsel == "fp4"
        _check(_lib.rac_second_pass(_ptr(self.x), self.M, self.K, self.x.stride(0), ctypes.byref(self._qx),
                                    _ptr(self.sel), self.n_sel, ctypes.byref(self._qr),
                                    None if fp4 else _ptr(self.w), self.N, self.K if fp4 else self.w.stride(0),
                                    ctypes.byref(self._qw), _ptr(self.dq_colamax if fp4 else self.w_colamax),
                                    ctypes.byref(self._qs), _stream(stream)), "rac_second_pass")

    def select_channels(self, stream=None):
        _check(_lib.rac_select_channels(_ptr(self.score), _ptr(self.res_colamax), self.K, self.k, _ptr(self.mask),
                                        _ptr(self.sel), ctypes.byref(self._nout), _ptr(self.res_st),
                                        _stream(stream)), "rac_select_channels")

    def residual_quant(self, stream=None):
        if self.n_sel == 0:
            return
        _check(_lib.rac_residual_quant(_ptr(self.x), self.M, self.K, self.x.stride(0), ctypes.byref(self._qx),
                                       _ptr(self.sel), self.n_sel, ctypes.byref(self._qr), _stream(stream)),
               "rac_residual_quant")

    def _gathers_overlapped(self):
        """After select_channels: the W_sel gather on the side stream (after
        any weight preparation queued there) concurrently with the residual
        gather on the current stream; the current stream then waits for it."""
        main = torch.cuda.current_stream()
        if self.n_sel == 0:
            return
        self._sel_ready.record(main)
        self.side.wait_event(self._sel_ready)
        self.weight_select(stream=self.side)
        self._wsel_done.record(self.side)
        self.residual_quant()
        main.wait_event(self._wsel_done)

    def weight_select(self, stream=None):
        if self.n_sel == 0:
            return
        if self.wsel == "fp4":
            _check(_lib.rac_weight_quant_fp4(ctypes.byref(self._qw), _ptr(self.sel), self.n_sel,
                                             _ptr(self.dq_colamax), ctypes.byref(self._qs), _stream(stream)),
                   "rac_weight_quant_fp4")
            return
        _check(_lib.rac_weight_quant(_ptr(self.w), self.N, self.K, self.w.stride(0), _ptr(self.sel), self.n_sel,
                                     _ptr(self.w_colamax), ctypes.byref(self._qs), _stream(stream)),
               "rac_weight_quant")

    def gemm(self, stream=None, plain=False):
        r = None if plain or self._qr is None else ctypes.byref(self._qr)
        s = None if plain or self._qs is None else ctypes.byref(self._qs)
        _check(_lib.w4a4_gemm_quantized(ctypes.byref(self._qx), ctypes.byref(self._qw), r, s, _ptr(self.y),
                                        0 if self.y.dtype == torch.float32 else 1, self.y.stride(0),
                                        _stream(stream)), "w4a4_gemm_quantized")

    def rollout_step(self):
        """The rollout linear on an already-prepared weight: quantize with the
        fused selection, both second passes, the GEMM (current stream)."""
        self.quantize_select()
        self.second_pass()
        self.gemm()

    def full_step(self):
        """Weight preparation and the rollout linear.  The weight preparation
        (independent of X) runs on a side stream that forks from the current
        stream and joins it before the second passes, which read Q(W)'s
        source and the weight's column maxima; it overlaps the quantize pass."""
        main = torch.cuda.current_stream()
        self._fork.record(main)
        self.side.wait_event(self._fork)
        self.prepare_weight(stream=self.side)
        self._join.record(self.side)
        self.quantize_select()
        main.wait_event(self._join)
        self.second_pass()
        self.gemm()

    def split_step(self):
        """The same linear as full_step through the separate calls (quantize,
        select_channels, the two gathers on two streams, GEMM)."""
        main = torch.cuda.current_stream()
        self._fork.record(main)
        self.side.wait_event(self._fork)
        self.prepare_weight(stream=self.side)
        self._join.record(self.side)
        self.quantize()
        self.select_channels()
        self._gathers_overlapped()                 # W_sel queued behind the weight preparation
        main.wait_event(self._join)
        self.gemm()

    def reuse_step(self):
        """The rollout linear with the channel mask, sel and Q(W_sel) kept
        from the last step that selected (see the class notes)."""
        if self.n_sel == 0:
            self.plain_step()
            return
        self.quantize(scores="colamax")
        _check(_lib.rac_sel_tensor_scale(_ptr(self.res_colamax), self.K, _ptr(self.sel), self.n_sel,
                                         _ptr(self.res_st), _stream(None)), "rac_sel_tensor_scale")
        self.residual_quant()
        self.gemm()

    def plain_step(self, stream=None):
        """Plain NVFP4 W4A4 (no RAC): Q(X) without scores, one-segment GEMM."""
        self.quantize(stream, scores=False)
        self.gemm(stream, plain=True)

    # kernels each call launches (for launch accounting)
    LAUNCHES = dict(prepare_weight=2, quantize=2, quantize_plain=2, select=2, weight_select=1, gemm=1,
                    reuse_step=5, quantize_select=2, second_pass=1)
