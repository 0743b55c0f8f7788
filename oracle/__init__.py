"""CPU oracle for the block-scaled FP4 routed-expert MoE FFN.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's ``cpu_baseline`` / ``--impl reference`` legs may import this package.
It is a numpy front end over the plain-C fp64 oracle in ``ds4g_oracle.c``
(sources and readings are listed in ``ds4g_oracle.h``); it shares no code with
the CUDA library.

Formats: ``MX`` = E2M1 + UE8M0 scale per 32 along K; ``NV`` = E2M1 + UE4M3
scale per 16 along K + an fp32 tensor scale ``g``; ``MX8`` = E4M3 (one byte
per element) + UE8M0 scale per 32 (the FP8 activations of the FP8 x FP4
variant).  A block-scaled tensor is the tuple
``Fp4(data uint8 [rows][K/2] (K for MX8), scales uint8 [rows][K/blk], g float, fmt)``.
"""
import ctypes
from collections import namedtuple

import numpy as np

from . import build as _build

MX = 0
NV = 1
MX8 = 2
BLOCK = {MX: 32, NV: 16, MX8: 32}


def _row_bytes(fmt, K):
    return K if fmt == MX8 else K // 2


def _K_of(t):
    return t.data.shape[1] if t.fmt == MX8 else t.data.shape[1] * 2

Fp4 = namedtuple("Fp4", ["data", "scales", "g", "fmt"])

_lib = None


def _L():
    global _lib
    if _lib is None:
        _build.build()
        L = ctypes.CDLL(_build.LIB)
        vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.orc_e2m1_decode.restype = dbl
        L.orc_e2m1_decode.argtypes = [i32]
        L.orc_e2m1_encode.restype = i32
        L.orc_e2m1_encode.argtypes = [dbl]
        L.orc_ue8m0_decode.restype = dbl
        L.orc_ue8m0_decode.argtypes = [i32]
        L.orc_ue4m3_decode.restype = dbl
        L.orc_ue4m3_decode.argtypes = [i32]
        L.orc_ue4m3_encode.restype = i32
        L.orc_ue4m3_encode.argtypes = [dbl]
        L.orc_lut_decode_check.restype = i32
        L.orc_lut_decode_check.argtypes = []
        L.orc_e4m3_decode.restype = dbl
        L.orc_e4m3_decode.argtypes = [i32]
        L.orc_e4m3_encode.restype = i32
        L.orc_e4m3_encode.argtypes = [dbl]
        L.orc_quantize_mx8.argtypes = [vp, i64, i64, vp, vp]
        L.orc_quantize_mx8.restype = None
        L.orc_expert_gemm_rows_mixed.argtypes = [vp, vp, dbl, i32, vp, i64, vp, vp, dbl, i32, i32, i32, i64, vp,
                                                 vp]
        L.orc_expert_gemm_rows_mixed.restype = None
        L.orc_quantize_mx.argtypes = [vp, i64, i64, vp, vp]
        L.orc_quantize_nv.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.orc_dequantize.argtypes = [vp, vp, i32, dbl, i64, i64, vp]
        L.orc_route_topk.argtypes = [vp, i32, i32, i32, vp, vp]
        L.orc_moe_permute.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.orc_gather_rows.argtypes = [vp, vp, i64, i32, vp, i64, i32, vp, vp]
        L.orc_grouped_gemm.argtypes = [vp, vp, dbl, vp, i32, vp, vp, dbl, i32, i64, i32,
                                       i64, i64, i32, i32, vp, vp]
        L.orc_expert_gemm_rows.argtypes = [vp, vp, dbl, vp, i64, vp, vp, dbl, i32, i32, i64, i32, vp, vp]
        L.orc_swiglu.argtypes = [vp, i64, i32, vp]
        L.orc_moe_combine.argtypes = [vp, vp, vp, i32, i32, i32, vp]
        for f in (L.orc_quantize_mx, L.orc_quantize_nv, L.orc_dequantize, L.orc_route_topk,
                  L.orc_moe_permute, L.orc_gather_rows, L.orc_grouped_gemm, L.orc_expert_gemm_rows,
                  L.orc_swiglu, L.orc_moe_combine):
            f.restype = None
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data if a is not None else None


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ---- codecs ----------------------------------------------------------------

def e2m1_decode(code):
    return _L().orc_e2m1_decode(int(code))


def e2m1_encode(y):
    return _L().orc_e2m1_encode(float(y))


def ue8m0_decode(b):
    return _L().orc_ue8m0_decode(int(b))


def ue4m3_decode(b):
    return _L().orc_ue4m3_decode(int(b))


def ue4m3_encode(r):
    return _L().orc_ue4m3_encode(float(r))


def lut_decode_check():
    return _L().orc_lut_decode_check()


def e4m3_decode(code):
    return _L().orc_e4m3_decode(int(code))


def e4m3_encode(y):
    return _L().orc_e4m3_encode(float(y))


# ---- quantisation ----------------------------------------------------------

def quantize(x, fmt, g=None):
    """x: fp32 array [rows][K] (bf16 inputs widened exactly by the caller)"""
    x = _c(x, np.float32)
    rows, K = x.shape
    blk = BLOCK[fmt]
    data = np.zeros((rows, _row_bytes(fmt, K)), np.uint8)
    scales = np.zeros((rows, K // blk), np.uint8)
    if fmt == MX8:
        _L().orc_quantize_mx8(_p(x), rows, K, _p(data), _p(scales))
        return Fp4(data, scales, 1.0, MX8)
    if fmt == MX:
        _L().orc_quantize_mx(_p(x), rows, K, _p(data), _p(scales))
        return Fp4(data, scales, 1.0, MX)
    gin = None if g is None else np.array([g], np.float32)
    gout = np.zeros(1, np.float32)
    _L().orc_quantize_nv(_p(x), rows, K, _p(gin), _p(data), _p(scales), _p(gout))
    return Fp4(data, scales, float(gout[0]), NV)


def dequantize(t):
    rows = t.data.shape[0]
    K = _K_of(t)
    out = np.empty((rows, K), np.float64)
    _L().orc_dequantize(_p(_c(t.data, np.uint8)), _p(_c(t.scales, np.uint8)), t.fmt, float(t.g),
                        rows, K, _p(out))
    return out


# ---- routing / permutation -------------------------------------------------

def route_topk(logits, k):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    _L().orc_route_topk(_p(logits), T, E, k, _p(idx), _p(w))
    return idx, w


def moe_permute(idx, E):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    S = T * k
    offsets = np.zeros(E + 1, np.int32)
    r2s = np.zeros(S, np.int32)
    s2r = np.zeros(S, np.int32)
    _L().orc_moe_permute(_p(idx), T, k, E, _p(offsets), _p(r2s), _p(s2r))
    return offsets, r2s, s2r


def gather_rows(t, row_to_slot, k):
    data = _c(t.data, np.uint8)
    scales = _c(t.scales, np.uint8)
    K = _K_of(t)
    r2s = _c(row_to_slot, np.int32)
    S = r2s.shape[0]
    od = np.zeros((S, data.shape[1]), np.uint8)
    os_ = np.zeros((S, scales.shape[1]), np.uint8)
    _L().orc_gather_rows(_p(data), _p(scales), K, t.fmt, _p(r2s), S, k, _p(od), _p(os_))
    return Fp4(od, os_, t.g, t.fmt)


# ---- GEMM / SwiGLU / combine -----------------------------------------------

def grouped_gemm(a, offsets, w, N, rows=None, cols=None):
    """Returns (out f64 [S][N], abssum f64 [S][N]); only rows[0]:rows[1] and
    cols[0]:cols[1] are filled when given (the rest stays NaN)."""
    ad, as_ = _c(a.data, np.uint8), _c(a.scales, np.uint8)
    wd, ws = _c(w.data, np.uint8), _c(w.scales, np.uint8)
    offsets = _c(offsets, np.int32)
    E = offsets.shape[0] - 1
    S = ad.shape[0]
    K = _K_of(a)
    r0, r1 = rows if rows is not None else (0, S)
    c0, c1 = cols if cols is not None else (0, N)
    out = np.full((S, N), np.nan)
    ab = np.full((S, N), np.nan)
    _L().orc_grouped_gemm(_p(ad), _p(as_), float(a.g), _p(offsets), E, _p(wd), _p(ws), float(w.g),
                          N, K, a.fmt, r0, r1, c0, c1, _p(out), _p(ab))
    return out, ab


def expert_gemm_rows(a, rows, w_e, cols):
    """rows of A (indices) against one expert's weights w_e (an Fp4 of that
    expert's N rows); returns (out, abssum) of shape [len(rows)][cols span]."""
    ad, as_ = _c(a.data, np.uint8), _c(a.scales, np.uint8)
    wd, ws = _c(w_e.data, np.uint8), _c(w_e.scales, np.uint8)
    rows = _c(rows, np.int64)
    K = _K_of(a)
    c0, c1 = cols
    out = np.empty((rows.shape[0], c1 - c0))
    ab = np.empty((rows.shape[0], c1 - c0))
    if a.fmt == w_e.fmt:
        _L().orc_expert_gemm_rows(_p(ad), _p(as_), float(a.g), _p(rows), rows.shape[0], _p(wd), _p(ws),
                                  float(w_e.g), c0, c1, K, a.fmt, _p(out), _p(ab))
    else:
        _L().orc_expert_gemm_rows_mixed(_p(ad), _p(as_), float(a.g), a.fmt, _p(rows), rows.shape[0], _p(wd),
                                        _p(ws), float(w_e.g), w_e.fmt, c0, c1, K, _p(out), _p(ab))
    return out, ab


def swiglu(y1):
    y1 = _c(y1, np.float32)
    rows, two_i = y1.shape
    h = np.empty((rows, two_i // 2), np.float32)
    _L().orc_swiglu(_p(y1), rows, two_i // 2, _p(h))
    return h


def moe_combine(y2, slot_to_row, w):
    y2 = _c(y2, np.float64)
    w = _c(w, np.float64)
    T, k = w.shape
    d = y2.shape[1]
    out = np.empty((T, d), np.float64)
    _L().orc_moe_combine(_p(y2), _p(_c(slot_to_row, np.int32)), _p(w), T, k, d, _p(out))
    return out


# ---- the whole layer -------------------------------------------------------

def moe_layer(x, logits, w1, w2, k, fmt, g_h=None):
    """The full routed-expert FFN on fp32 inputs x [T][d] (already widened from
    bf16), router logits [T][E], expert weights w1 (Fp4 of [E*2I][d]) and w2
    (Fp4 of [E*d][I]).  Returns a dict of every stage's result."""
    T, d = x.shape
    E = logits.shape[1]
    idx, w = route_topk(logits, k)
    xq = quantize(x, fmt)
    offsets, r2s, s2r = moe_permute(idx, E)
    a = gather_rows(xq, r2s, k)
    two_i = w1.data.shape[0] // E
    y1, y1_abs = grouped_gemm(a, offsets, w1, two_i)
    y1f = y1.astype(np.float32)
    h = swiglu(y1f)
    hq = quantize(h, fmt, g=g_h if fmt == NV else None)
    y2, y2_abs = grouped_gemm(hq, offsets, w2, d)
    y2f = y2.astype(np.float32)
    out = moe_combine(y2f.astype(np.float64), s2r, w)
    return dict(idx=idx, w=w, xq=xq, offsets=offsets, row_to_slot=r2s, slot_to_row=s2r, a=a,
                y1=y1, y1_abs=y1_abs, h=h, hq=hq, y2=y2, y2_abs=y2_abs, out=out)
