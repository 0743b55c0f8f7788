"""The C-ABI library loads on a machine without a GPU and exports every
function include/ds4g.h declares; the host-only helpers answer without a
device (no compute call is made here)."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ds4g.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ds4g_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_path_calls():
    names = _declared()
    for n in ("ds4g_quantize_mx", "ds4g_route_topk", "ds4g_moe_permute", "ds4g_grouped_gemm_fp4",
              "ds4g_swiglu_requant", "ds4g_moe_combine"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from block_scaled_fp4_topk_b200 import build
    build.build()
    lib = ctypes.CDLL(build.LIB)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_host_only_helpers():
    from block_scaled_fp4_topk_b200 import ds4g
    L = ds4g._lib
    assert L.ds4g_status_str(0) == b"ok"
    assert b"64" in L.ds4g_status_str(2)
    assert L.ds4g_quantize_workspace_bytes(1, 0) >= 4 and L.ds4g_quantize_workspace_bytes(0, 0) == 0
    # per-expert counts of each 256-slot chunk: E * ceil(T*k / 256) int32
    assert L.ds4g_permute_workspace_bytes(2048, 6, 256) == 256 * 48 * 4
    # dispatch: the permutation's counts (16-byte rounded), plus the NVFP4 amax word without g_in
    assert L.ds4g_dispatch_workspace_bytes(2048, 6, 256, 0, 0) == 256 * 48 * 4
    assert L.ds4g_dispatch_workspace_bytes(2048, 6, 256, 1, 0) == 256 * 48 * 4 + 16
    assert L.ds4g_dispatch_workspace_bytes(2048, 6, 256, 1, 1) == 256 * 48 * 4
    assert L.ds4g_permute_static_max_bytes() == 256 * 1024


def test_bad_arguments_rejected_before_any_launch():
    # shape / argument validation happens on the host and needs no device
    from block_scaled_fp4_topk_b200 import ds4g
    L = ds4g._lib
    assert L.ds4g_route_topk(None, 4, 8, 9, None, None, None) == 1          # k > E
    assert L.ds4g_moe_combine(None, None, None, 2, 2, 6, None, None) == 2   # d % 4 != 0
    out = ds4g._Fp4C(None, None, None, 4, 96, 0, 0)
    assert L.ds4g_quantize_mx(None, 0, 4, 96, 0, None, ctypes.byref(out), None, 0, None) == 2   # K % 64


def _fp4(rows, K, fmt=0, buf=None):
    """a ds4g_fp4 descriptor whose data / scale pointers are host addresses:
    the calls below must reject their arguments before touching them"""
    from block_scaled_fp4_topk_b200 import ds4g
    p = buf.ctypes.data if buf is not None else None
    return ds4g._Fp4C(p, p, p, rows, K, fmt, 0)


def test_grouped_gemm_shapes_rejected_on_the_host():
    import numpy as np
    from block_scaled_fp4_topk_b200 import ds4g
    L = ds4g._lib
    buf = np.zeros(1 << 16, np.uint8)              # 64-byte aligned host buffer, never read
    offs = np.zeros(5, np.int32)
    op = offs.ctypes.data_as(ctypes.c_void_p)
    out = buf.ctypes.data_as(ctypes.c_void_p)
    a = _fp4(8, 96, buf=buf)
    w = _fp4(4 * 128, 96, buf=buf)
    # K % 64 != 0 (the FP4 path's K rule)
    assert L.ds4g_grouped_gemm_fp4(ctypes.byref(a), op, 4, 8, ctypes.byref(w), 128, 0, out, None, None, None) == 2
    a, w = _fp4(8, 128, buf=buf), _fp4(4 * 128, 128, buf=buf)
    # no experts / missing operands
    assert L.ds4g_grouped_gemm_fp4(ctypes.byref(a), op, 0, 8, ctypes.byref(w), 128, 0, out, None, None, None) == 1
    assert L.ds4g_grouped_gemm_fp4(None, op, 4, 8, ctypes.byref(w), 128, 0, out, None, None, None) == 1
    # an epilogue the call does not have
    assert L.ds4g_grouped_gemm_fp4(ctypes.byref(a), op, 4, 8, ctypes.byref(w), 128, 7, out, None, None, None) == 1
    # weights whose K differs from the activations'
    wk = _fp4(4 * 128, 256, buf=buf)
    assert L.ds4g_grouped_gemm_fp4(ctypes.byref(a), op, 4, 8, ctypes.byref(wk), 128, 0, out, None, None, None) == 2
    # SwiGLU: N = 2I with I % 32 != 0
    w80 = _fp4(4 * 80, 128, buf=buf)
    hq = _fp4(8, 40, buf=buf)
    assert L.ds4g_grouped_gemm_fp4(ctypes.byref(a), op, 4, 8, ctypes.byref(w80), 80, 1, None, ctypes.byref(hq),
                                   None, None) == 2
    # FC2 + combine: a must have T * k rows; k >= 1
    r2s = offs.ctypes.data_as(ctypes.c_void_p)
    assert L.ds4g_grouped_gemm_fp4_combine(ctypes.byref(a), op, 4, 8, ctypes.byref(w), 128, r2s, out, 3, 2, out,
                                           None) == 2
    assert L.ds4g_grouped_gemm_fp4_combine(ctypes.byref(a), op, 4, 8, ctypes.byref(w), 128, r2s, out, 8, 0, out,
                                           None) == 1


def test_chained_combine_and_zero_fill_rejected_on_the_host():
    import numpy as np
    from block_scaled_fp4_topk_b200 import ds4g
    L = ds4g._lib
    buf = np.zeros(1 << 16, np.uint8)              # 64-byte aligned host buffer, never read
    offs = np.zeros(5, np.int32)
    op = offs.ctypes.data_as(ctypes.c_void_p)
    out = buf.ctypes.data_as(ctypes.c_void_p)
    a, w = _fp4(8, 128, buf=buf), _fp4(4 * 128, 128, buf=buf)
    # a must have T * k rows; k >= 1; T >= 0; the routing arrays when T > 0
    assert L.ds4g_grouped_gemm_fp4_combine_chained(ctypes.byref(a), op, 4, 8, ctypes.byref(w), 128, op, out, 3, 2,
                                                   out, None) == 2
    assert L.ds4g_grouped_gemm_fp4_combine_chained(ctypes.byref(a), op, 4, 8, ctypes.byref(w), 128, op, out, 8, 0,
                                                   out, None) == 1
    assert L.ds4g_grouped_gemm_fp4_combine_chained(ctypes.byref(a), op, 4, 8, ctypes.byref(w), 128, None, out, 4, 2,
                                                   out, None) == 1
    # zero-fill: nothing to do for 0 bytes; a null pointer otherwise is rejected
    assert L.ds4g_zero_fill(None, 0, None) == 0
    assert L.ds4g_zero_fill(None, 64, None) == 1


def test_empty_combine_is_a_no_op():
    from block_scaled_fp4_topk_b200 import ds4g
    # zero tokens: validated, nothing to launch
    assert ds4g._lib.ds4g_moe_combine(None, None, None, 0, 6, 7168, None, None) == 0


def test_ffn_call_rejected_on_the_host():
    import numpy as np
    from block_scaled_fp4_topk_b200 import ds4g
    L = ds4g._lib
    buf = np.zeros(1 << 16, np.uint8)              # 64-byte aligned host buffer, never read
    offs = np.zeros(5, np.int32)
    op = offs.ctypes.data_as(ctypes.c_void_p)
    out = buf.ctypes.data_as(ctypes.c_void_p)
    E, d, I, T, k = 4, 512, 512, 4, 2
    a, h = _fp4(T * k, d, buf=buf), _fp4(T * k, I, buf=buf)
    w1, w2 = _fp4(E * 2 * I, d, buf=buf), _fp4(E * d, I, buf=buf)

    def call(a=a, max_rows=4, w1=w1, w2=w2, d=d, I=I, h=h, T=T, k=k, ctr=out):
        return L.ds4g_moe_ffn_fp4(ctypes.byref(a), op, E, max_rows, ctypes.byref(w1), ctypes.byref(w2), d, I,
                                  ctypes.byref(h), op, out, T, k, out, ctr, None)
    assert call(a=_fp4(T * k + 1, d, buf=buf)) == 2            # a must have T * k rows
    assert call(max_rows=17) == 2                              # decode sizes only
    assert call(a=_fp4(T * k, 96, buf=buf), d=96) == 2         # the decode kernel's K rule
    assert call(w2=_fp4(E * d, 256, buf=buf)) == 2             # w2's K must be I
    assert call(h=_fp4(T * k, 256, buf=buf)) == 2              # h_q rows of I
    assert call(ctr=None) == 1                                 # the counters are required
    assert call(k=0) == 1
    a8 = _fp4(T * k, d, fmt=2, buf=buf)
    assert call(a=a8) == 1                                     # FP4 activations only
