"""Scalar pure-Python restatement of the RAC linear, for tiny inputs only.

Test infrastructure: see the package header in ``oracle/__init__.py``.

It is written independently of the numpy oracle (formats by exhaustive search
over every code, fp32 rounding through ``struct``) so that the two can check
each other on shapes of a few rows and channels.  Python floats are binary64;
an fp32 operation is done in binary64 and rounded once to binary32, which
equals the fp32-rounded exact result for +, -, * and / because binary64
carries more than 2 x 24 + 2 bits.
"""
from __future__ import annotations

import math
import struct


def f32(v: float) -> float:
    """Round a binary64 value to the nearest binary32 (ties to even)."""
    if math.isinf(v) or abs(v) >= 3.4028235677973366e38:
        return math.copysign(math.inf, v)   # no overflow occurs on valid inputs
    return struct.unpack("<f", struct.pack("<f", v))[0]


def bf16_bits_to_float(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (b & 0xFFFF) << 16))[0]


def e2m1_value(code: int) -> float:
    exp, man = (code >> 1) & 3, code & 1
    mag = man * 0.5 if exp == 0 else (1.0 + man * 0.5) * 2.0 ** (exp - 1)
    return -mag if code & 8 else mag


def e4m3_value(code: int) -> float:
    exp, man = (code >> 3) & 15, code & 7
    return man * 2.0 ** -9 if exp == 0 else (1.0 + man / 8.0) * 2.0 ** (exp - 7)


def e2m1_code(v: float) -> int:
    a = abs(v)
    best = 0
    for c in range(8):
        d_c, d_b = abs(a - e2m1_value(c)), abs(a - e2m1_value(best))
        if d_c < d_b or (d_c == d_b and c % 2 == 0 and best % 2 == 1):
            best = c
    return best | (8 if math.copysign(1.0, v) < 0 else 0)


def e4m3_code(s: float) -> int:
    best = 0
    for c in range(0x7F):
        d_c, d_b = abs(s - e4m3_value(c)), abs(s - e4m3_value(best))
        if d_c < d_b or (d_c == d_b and c % 2 == 0 and best % 2 == 1):
            best = c
    return best


def quantize_rows(rows, s_t):
    """rows: list of lists of floats (fp32 values), length % 16 == 0."""
    codes, scales = [], []
    for row in rows:
        rc, rs = [], []
        for b0 in range(0, len(row), 16):
            blk = row[b0:b0 + 16]
            if s_t == 0.0:
                rs.append(0)
                rc.extend(8 if math.copysign(1.0, v) < 0 else 0 for v in blk)
                continue
            d = f32(6.0 * s_t)
            sb = e4m3_code(f32(max(abs(v) for v in blk) / d))
            s_dec = f32(e4m3_value(sb) * s_t)
            rs.append(sb)
            for v in blk:
                q = f32(v / s_dec) if s_dec > 0 else math.copysign(0.0, v)
                rc.append(e2m1_code(q))
        codes.append(rc)
        scales.append(rs)
    return codes, scales


def dequantize_rows(codes, scales, s_t):
    return [[f32(f32(e2m1_value(c) * e4m3_value(scales[i][j // 16])) * s_t)
             for j, c in enumerate(row)] for i, row in enumerate(codes)]


def rac_linear(x_bits, w_bits, k_percent, wsel_source="bf16"):
    """x_bits [M][K], w_bits [N][K]: bf16 bit patterns.  Returns a dict with
    the codes, scales, scores, sel and the fp64 outputs.  wsel_source="fp4"
    takes the selected weight columns from the dequantized NVFP4 weights."""
    X = [[bf16_bits_to_float(b) for b in row] for row in x_bits]
    W = [[bf16_bits_to_float(b) for b in row] for row in w_bits]
    M, K, N = len(X), len(X[0]), len(W)

    def t_scale(rows):
        a = max((abs(v) for row in rows for v in row), default=0.0)
        return a, f32(a / 2688.0)

    ax, stx = t_scale(X)
    cx, sx = quantize_rows(X, stx)
    dqx = dequantize_rows(cx, sx, stx)
    dx = [[f32(X[i][j] - dqx[i][j]) for j in range(K)] for i in range(M)]
    score = [0.0] * K
    for j in range(K):
        total = 0.0
        for c0 in range(0, M, 128):
            part = 0.0
            for i in range(c0, min(c0 + 128, M)):
                part += abs(dx[i][j])
            total += part
        score[j] = total
    n_sel = math.floor(k_percent * K / 100)
    ranked = sorted(range(K), key=lambda j: (-score[j], j))
    sel = sorted(ranked[:n_sel])

    aw, stw = t_scale(W)
    cw, sw = quantize_rows(W, stw)

    def block_val(codes, scales, i, j):
        return e2m1_value(codes[i][j]) * e4m3_value(scales[i][j // 16])

    def product(ca, sa, sta, cb, sb_, stb, width):
        return [[sta * stb * sum(block_val(ca, sa, i, k) * block_val(cb, sb_, n, k)
                                 for k in range(width)) for n in range(len(cb))]
                for i in range(len(ca))]

    y_plain = product(cx, sx, stx, cw, sw, stw, K)
    out = dict(codes=cx, scales=sx, s_t=stx, dx=dx, score=score, sel=sel,
               w_codes=cw, w_scales=sw, w_st=stw, y_plain=y_plain)
    if n_sel == 0:
        out["y"] = y_plain
        return out
    width = -(-n_sel // 64) * 64
    R = [[dx[i][j] for j in sel] + [0.0] * (width - n_sel) for i in range(M)]
    Wsrc = dequantize_rows(cw, sw, stw) if wsel_source == "fp4" else W
    Ws = [[Wsrc[n][j] for j in sel] + [0.0] * (width - n_sel) for n in range(N)]
    ar, str_ = t_scale(R)
    aws, stws = t_scale(Ws)
    cr, sr = quantize_rows(R, str_)
    cws, sws = quantize_rows(Ws, stws)
    y_corr = product(cr, sr, str_, cws, sws, stws, width)
    out.update(r_codes=cr, r_scales=sr, r_st=str_, ws_codes=cws, ws_scales=sws,
               ws_st=stws, y=[[y_plain[i][n] + y_corr[i][n] for n in range(N)]
                              for i in range(M)])
    return out


def mxfp8_quantize_rows(rows):
    """MXFP8 (E4M3 elements, one UE8M0 scale per 32 elements) of fp32 rows,
    restated independently of oracle.mxfp8: the block exponent from a loop
    over powers of two, the element code by exhaustive nearest search over
    the 127 finite E4M3 magnitudes (ties to the even code, 448 saturates)."""
    codes, scales = [], []
    for row in rows:
        rc, rs = [], []
        for b0 in range(0, len(row), 32):
            blk = row[b0:b0 + 32]
            amax = max(abs(v) for v in blk)
            if amax == 0.0:
                e = -127
            else:
                p = 0
                while 2.0 ** (p + 1) <= amax:
                    p += 1
                while 2.0 ** p > amax:
                    p -= 1
                e = max(-127, min(127, p - 8))
            rs.append(e + 127)
            for v in blk:
                q = v / 2.0 ** e
                rc.append(e4m3_code(abs(q)) | (0x80 if math.copysign(1.0, v) < 0 else 0))
        codes.append(rc)
        scales.append(rs)
    return codes, scales
