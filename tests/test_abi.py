"""The C ABI library loads and exports every symbol the header declares; pure
host-side behaviour (sizes, n_sel, argument checks) needs no GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from precision_rl_rollout_nvfp4_b200 import build_lib
    build_lib.build()
    return ctypes.CDLL(build_lib.LIB)


def declared_functions():
    text = open(os.path.join(ROOT, "include", "nvfp4rac.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z0-9_]+)\s*\(", text)) - {"defined", "sizeof"})


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n


def test_binding_matches_header():
    from precision_rl_rollout_nvfp4_b200 import binding
    assert sorted(binding.EXPORTS) == declared_functions()


def test_nsel_and_width(lib):
    import oracle
    f = lib.nvfp4_rac_nsel
    f.restype, f.argtypes = ctypes.c_int64, [ctypes.c_float, ctypes.c_int64]
    for k in (0.0, 12.5, 25.0, 33.3, 50.0, 99.99, 100.0, 0.1):
        for K in (64, 1000, 2048, 11008):
            assert f(k, K) == oracle.n_selected(k, K)
    assert f(-1.0, 64) == -1 and f(100.5, 64) == -1
    w = lib.nvfp4_rac_width
    w.restype, w.argtypes = ctypes.c_int64, [ctypes.c_int64]
    assert [w(n) for n in (0, 1, 64, 65, 5504)] == [0, 64, 64, 128, 5504]


def test_scale_bytes_and_workspace(lib):
    f = lib.nvfp4_scale_bytes
    f.restype, f.argtypes = ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32]
    assert f(64, 512, 0) == 64 * 32
    assert f(64, 512, 1) == 128 * 32
    assert f(300, 192, 1) == 384 * 4 * 3
    ws = lib.nvfp4_workspace_size
    ws.restype = ctypes.c_size_t
    ws.argtypes = [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32]
    assert ws(0, 4096, 0, 2048, 1) >= 32 * 2048 * 12
    assert ws(9, 1, 1, 64, 1) == 0


def test_argument_errors_without_gpu(lib):
    q = lib.nvfp4_quantize
    q.restype = ctypes.c_int32
    # null input -> NVFP4_ERR_INVALID_ARG before any CUDA call
    assert q(None, 64, 64, 64, None, None, None, None, None, 0, None) == 1
    s = lib.nvfp4_status_string
    s.restype, s.argtypes = ctypes.c_char_p, [ctypes.c_int32]
    assert s(6) == b"device-side wait timed out"


class _T(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("scale_layout", ctypes.c_int32)]


def _fake_tensor(rows, cols, layout=1):
    # aligned, never dereferenced: every call below returns before any CUDA work
    return _T(0x10000, 0x20000, 0x30000, rows, cols, layout)


def test_nvfp4_weight_variant_argument_errors_without_gpu(lib):
    """nvfp4_dq_colamax and rac_weight_quant_fp4 reject bad arguments with
    the documented codes before any CUDA call."""
    TP = ctypes.POINTER(_T)
    cm = lib.nvfp4_dq_colamax
    cm.restype, cm.argtypes = ctypes.c_int32, [TP, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    q = _fake_tensor(256, 512)
    assert cm(None, 1, ctypes.c_void_p(0x40000), None) == 1            # null tensor
    assert cm(ctypes.byref(q), 1, None, None) == 1                     # null output
    assert cm(ctypes.byref(q), 0, ctypes.c_void_p(0x40000), None) == 3   # batch 0
    assert cm(ctypes.byref(q), 3, ctypes.c_void_p(0x40000), None) == 3   # rows % batch
    bad = _fake_tensor(256, 500)
    assert cm(ctypes.byref(bad), 1, ctypes.c_void_p(0x40000), None) == 3  # cols % 64
    assert cm(ctypes.byref(q), 1, ctypes.c_void_p(0x40004), None) == 2    # misaligned output
    wq = lib.rac_weight_quant_fp4
    wq.restype = ctypes.c_int32
    wq.argtypes = [TP, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, TP, ctypes.c_void_p]
    out = _fake_tensor(256, 256)
    sel, dq = ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000)
    assert wq(None, sel, 200, dq, ctypes.byref(out), None) == 1
    assert wq(ctypes.byref(q), None, 200, dq, ctypes.byref(out), None) == 1
    assert wq(ctypes.byref(q), sel, 0, dq, ctypes.byref(out), None) == 3       # n_sel 0
    assert wq(ctypes.byref(q), sel, 513, dq, ctypes.byref(out), None) == 3     # n_sel > K
    assert wq(ctypes.byref(q), sel, 100, dq, ctypes.byref(out), None) == 3     # width 128 != 256
    wrong_rows = _fake_tensor(128, 256)
    assert wq(ctypes.byref(q), sel, 200, dq, ctypes.byref(wrong_rows), None) == 3


def test_split_select_argument_errors_without_gpu(lib):
    f = lib.rac_select_channels
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64), ctypes.c_void_p, ctypes.c_void_p]
    n = ctypes.c_int64(-1)
    p = ctypes.c_void_p
    assert f(None, p(0x100), 512, 50.0, p(0x200), p(0x300), ctypes.byref(n), p(0x400), None) == 1
    assert f(p(0x100), p(0x100), 512, 50.0, p(0x200), p(0x300), ctypes.byref(n), None, None) == 1
    assert f(p(0x100), p(0x100), 512, 150.0, p(0x200), p(0x300), ctypes.byref(n), p(0x400), None) == 1
    assert f(p(0x100), p(0x100), 500, 50.0, p(0x200), p(0x300), ctypes.byref(n), p(0x400), None) == 3
    assert f(p(0x100), p(0x100), 512, 50.0, p(0x200), None, ctypes.byref(n), p(0x400), None) == 1
    g = lib.rac_residual_quant
    TP = ctypes.POINTER(_T)
    g.restype = ctypes.c_int32
    g.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, TP, ctypes.c_void_p,
                  ctypes.c_int64, TP, ctypes.c_void_p]
    qx, qr = _fake_tensor(64, 512), _fake_tensor(64, 256)
    assert g(None, 64, 512, 512, ctypes.byref(qx), p(0x300), 256, ctypes.byref(qr), None) == 1
    assert g(p(0x1000), 64, 512, 512, ctypes.byref(qx), p(0x300), 300, ctypes.byref(qr), None) == 3   # width 320
    assert g(p(0x1000), 64, 512, 512, ctypes.byref(qx), p(0x300), 0, ctypes.byref(qr), None) == 3
    assert g(p(0x1008), 64, 512, 512, ctypes.byref(qx), p(0x300), 256, ctypes.byref(qr), None) == 2


def test_sel_tensor_scale_argument_errors_without_gpu(lib):
    f = lib.rac_sel_tensor_scale
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    p = ctypes.c_void_p
    assert f(None, 512, p(0x100), 8, p(0x200), None) == 1
    assert f(p(0x100), 512, None, 8, p(0x200), None) == 1
    assert f(p(0x100), 512, p(0x100), 8, None, None) == 1
    assert f(p(0x100), 512, p(0x100), 0, p(0x200), None) == 3
    assert f(p(0x100), 512, p(0x100), 513, p(0x200), None) == 3


def test_quantize_refuses_scores_without_colamax(lib):
    q = lib.nvfp4_quantize
    q.restype = ctypes.c_int32
    t = _fake_tensor(64, 64)
    q.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.POINTER(_T), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                  ctypes.c_void_p]
    assert q(ctypes.c_void_p(0x1000), 64, 64, 64, None, ctypes.byref(t), ctypes.c_void_p(0x2000), None,
             None, 0, None) == 1


def test_header_is_plain_c_and_links(tmp_path):
    """include/nvfp4rac.h compiles as strict C99 and a C program links
    against the library and calls its host-side size functions."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use_abi.c"
    src.write_text(
        '#include "nvfp4rac.h"\n'
        "int main(void) {\n"
        "  if (nvfp4_rac_width(1) != 64 || nvfp4_rac_width(65) != 128) return 1;\n"
        "  if (nvfp4_rac_nsel(50.0f, 2048) != 1024) return 2;\n"
        "  if (nvfp4_scale_bytes(300, 192, 1) != 384 * 4 * 3) return 3;\n"
        "  if (nvfp4_workspace_size(99, 1, 1, 64, 1) != 0) return 4;\n"
        "  return 0;\n}\n")
    pkg = os.path.join(root, "precision_rl_rollout_nvfp4_b200")
    exe = tmp_path / "use_abi"
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(root, "include"),
           str(src), os.path.join(pkg, "libnvfp4rac.so"), "-Wl,-rpath," + pkg, "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0
