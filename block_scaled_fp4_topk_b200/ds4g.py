"""Thin Python binding of libds4g (include/ds4g.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  If the compiled
library is missing, importing this module raises: there is no fallback.
"""
import ctypes
import os

import torch

from . import build as _build

MXFP4 = 0
NVFP4 = 1
MXFP8 = 2
BF16 = 0
F32 = 1
EPI_NONE = 0
EPI_SWIGLU_REQUANT = 1
BLOCK = {MXFP4: 32, NVFP4: 16, MXFP8: 32}


def row_bytes(fmt, K):
    """bytes of one row of K elements: E4M3 (MXFP8) one per byte, E2M1 two"""
    return K if fmt == MXFP8 else K // 2

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "unsupported device", 4: "CUDA error",
           5: "device-side wait gave up", 6: "workspace missing or too small"}


class Ds4gError(RuntimeError):
    def __init__(self, call, status):
        self.status = status
        super().__init__(f"{call}: {_STATUS.get(status, status)} (status {status})")


class _Fp4C(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("g", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("K", ctypes.c_int64), ("fmt", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


if not os.path.exists(_build.LIB):
    raise ImportError(f"libds4g.so is not built ({_build.LIB}); run block_scaled_fp4_topk_b200/build.py")

_lib = ctypes.CDLL(_build.LIB)
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_P = ctypes.POINTER(_Fp4C)
_SIGS = {
    "ds4g_status_str": ([_i32], ctypes.c_char_p),
    "ds4g_device_supported": ([], _i32),
    "ds4g_check_device": ([_vp], _i32),
    "ds4g_quantize_workspace_bytes": ([_i32, _i32], _sz),
    "ds4g_quantize_mx": ([_vp, _i32, _i64, _i64, _i32, _vp, _P, _vp, _sz, _vp], _i32),
    "ds4g_route_topk": ([_vp, _i32, _i32, _i32, _vp, _vp, _vp], _i32),
    "ds4g_permute_workspace_bytes": ([_i32, _i32, _i32], _sz),
    "ds4g_moe_permute": ([_vp, _i32, _i32, _i32, _P, _vp, _vp, _vp, _P, _vp, _sz, _vp], _i32),
    "ds4g_dispatch_workspace_bytes": ([_i32, _i32, _i32, _i32, _i32], _sz),
    "ds4g_moe_dispatch": ([_vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _P, _vp, _vp, _vp, _P, _vp, _sz,
                           _vp], _i32),
    "ds4g_grouped_gemm_fp4": ([_P, _vp, _i32, _i32, _P, _i32, _i32, _vp, _P, _vp, _vp], _i32),
    "ds4g_swiglu_requant": ([_vp, _i64, _i32, _i32, _P, _vp, _vp], _i32),
    "ds4g_grouped_gemm_fp4_combine": ([_P, _vp, _i32, _i32, _P, _i32, _vp, _vp, _i32, _i32, _vp, _vp], _i32),
    "ds4g_moe_combine": ([_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp], _i32),
    "ds4g_segment_ids": ([_vp, _i32, _i32, _i64, _vp, _vp], _i32),
    "ds4g_grouped_gemm_fp4_combine_chained": ([_P, _vp, _i32, _i32, _P, _i32, _vp, _vp, _i32, _i32, _vp, _vp],
                                              _i32),
    "ds4g_moe_ffn_fp4": ([_P, _vp, _i32, _i32, _P, _P, _i32, _i32, _P, _vp, _vp, _i32, _i32, _vp, _vp, _vp], _i32),
    "ds4g_zero_fill": ([_vp, _sz, _vp], _i32),
    "ds4g_permute_static_max_bytes": ([], _sz),
    "ds4g_moe_permute_static": ([_vp, _i32, _i32, _i32, _P, _vp, _vp, _vp, _P, _vp], _i32),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res

LIB_PATH = _build.LIB
EXPORTED = tuple(_SIGS)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _check(name, st):
    if st != 0:
        raise Ds4gError(name, st)


class Fp4Tensor:
    """Device block-scaled tensor: data uint8 [rows][K/2] (FP4) or [rows][K]
    (MXFP8), scales uint8 [rows][K/blk], g float32 [1] (NVFP4 tensor scale)
    or None, fmt."""

    def __init__(self, data, scales, g, fmt):
        self.data, self.scales, self.g, self.fmt = data, scales, g, fmt

    @property
    def rows(self):
        return self.data.shape[0]

    @property
    def K(self):
        return self.data.shape[1] * (1 if self.fmt == MXFP8 else 2)

    @staticmethod
    def empty(rows, K, fmt, device="cuda"):
        g = torch.ones(1, dtype=torch.float32, device=device) if fmt == NVFP4 else None
        return Fp4Tensor(torch.empty((rows, row_bytes(fmt, K)), dtype=torch.uint8, device=device),
                         torch.empty((rows, K // BLOCK[fmt]), dtype=torch.uint8, device=device), g, fmt)

    def c(self):
        return _Fp4C(self.data.data_ptr(), self.scales.data_ptr(), _ptr(self.g), self.rows, self.K, self.fmt, 0)

    def view_rows(self, r0, r1):
        return Fp4Tensor(self.data[r0:r1], self.scales[r0:r1], self.g, self.fmt)


def ds4g_device_supported():
    return _lib.ds4g_device_supported() == 0


def ds4g_check_device():
    _check("ds4g_check_device", _lib.ds4g_check_device(_stream()))


def ds4g_quantize_mx(x, fmt, g_in=None, out=None, workspace=None):
    rows, K = x.shape
    dtype = BF16 if x.dtype == torch.bfloat16 else F32
    if out is None:
        out = Fp4Tensor.empty(rows, K, fmt, x.device)
    need = _lib.ds4g_quantize_workspace_bytes(fmt, 1 if g_in is not None else 0)
    if need and workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    c = out.c()
    _check("ds4g_quantize_mx", _lib.ds4g_quantize_mx(x.data_ptr(), dtype, rows, K, fmt, _ptr(g_in), ctypes.byref(c),
                                                     _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                                     _stream()))
    return out


def ds4g_route_topk(logits, k, idx=None, w=None):
    T, E = logits.shape
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if w is None:
        w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _check("ds4g_route_topk", _lib.ds4g_route_topk(logits.data_ptr(), T, E, k, idx.data_ptr(), w.data_ptr(), _stream()))
    return idx, w


def permute_workspace(T, k, E, device="cuda"):
    n = _lib.ds4g_permute_workspace_bytes(T, k, E)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def ds4g_moe_permute(idx, E, x_q, offsets=None, row_to_slot=None, slot_to_row=None, a_perm=None, workspace=None):
    T, k = idx.shape
    S = T * k
    dev = idx.device
    if offsets is None:
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_to_slot is None:
        row_to_slot = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    if slot_to_row is None:
        slot_to_row = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    if a_perm is None:
        a_perm = Fp4Tensor.empty(S, x_q.K, x_q.fmt, dev)
    if workspace is None:
        workspace = permute_workspace(T, k, E, dev)
    xc, ac = x_q.c(), a_perm.c()
    _check("ds4g_moe_permute", _lib.ds4g_moe_permute(idx.data_ptr(), T, k, E, ctypes.byref(xc), offsets.data_ptr(),
                                                     row_to_slot.data_ptr(), slot_to_row.data_ptr(), ctypes.byref(ac),
                                                     workspace.data_ptr(), workspace.numel(), _stream()))
    return offsets, row_to_slot[:S], slot_to_row[:S], a_perm


def dispatch_workspace(T, k, E, fmt, has_g_in=False, device="cuda"):
    n = _lib.ds4g_dispatch_workspace_bytes(T, k, E, fmt, 1 if has_g_in else 0)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def ds4g_moe_dispatch(logits, x, k, fmt, g_in=None, idx=None, w=None, x_q=None, offsets=None, row_to_slot=None,
                      slot_to_row=None, a_perm=None, workspace=None):
    """route + quantise + permute in one call; returns
    (idx, w, x_q, offsets, row_to_slot[:S], slot_to_row[:S], a_perm)"""
    T, E = logits.shape
    d = x.shape[1]
    S = T * k
    dev = x.device
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if w is None:
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
    if x_q is None:
        x_q = Fp4Tensor.empty(T, d, fmt, dev)
    if offsets is None:
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_to_slot is None:
        row_to_slot = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    if slot_to_row is None:
        slot_to_row = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    if a_perm is None:
        a_perm = Fp4Tensor.empty(S, d, fmt, dev)
    if workspace is None:
        workspace = dispatch_workspace(T, k, E, fmt, g_in is not None, dev)
    dtype = BF16 if x.dtype == torch.bfloat16 else F32
    xc, ac = x_q.c(), a_perm.c()
    _check("ds4g_moe_dispatch",
           _lib.ds4g_moe_dispatch(logits.data_ptr(), x.data_ptr(), dtype, T, E, k, fmt, _ptr(g_in), idx.data_ptr(),
                                  w.data_ptr(), ctypes.byref(xc), offsets.data_ptr(), row_to_slot.data_ptr(),
                                  slot_to_row.data_ptr(), ctypes.byref(ac), workspace.data_ptr(), workspace.numel(),
                                  _stream()))
    return idx, w, x_q, offsets, row_to_slot[:S], slot_to_row[:S], a_perm


def ds4g_moe_permute_static(idx, E, x_q, offsets=None, row_to_slot=None, slot_to_row=None, a_perm=None):
    """ds4g_moe_permute with the library's own static scratch (no workspace)."""
    T, k = idx.shape
    S = T * k
    dev = idx.device
    if offsets is None:
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_to_slot is None:
        row_to_slot = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    if slot_to_row is None:
        slot_to_row = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    if a_perm is None:
        a_perm = Fp4Tensor.empty(S, x_q.K, x_q.fmt, dev)
    xc, ac = x_q.c(), a_perm.c()
    _check("ds4g_moe_permute_static",
           _lib.ds4g_moe_permute_static(idx.data_ptr(), T, k, E, ctypes.byref(xc), offsets.data_ptr(),
                                        row_to_slot.data_ptr(), slot_to_row.data_ptr(), ctypes.byref(ac), _stream()))
    return offsets, row_to_slot[:S], slot_to_row[:S], a_perm


def ds4g_grouped_gemm_fp4(a, offsets, E, max_rows_per_expert, w, N, epilogue=EPI_NONE, out=None, out_q=None,
                          h_debug=None):
    S = a.rows
    if epilogue == EPI_NONE and out is None:
        out = torch.empty((S, N), dtype=torch.float32, device=a.data.device)
    if epilogue == EPI_SWIGLU_REQUANT and out_q is None:
        raise ValueError("SWIGLU_REQUANT needs out_q (and out_q.g for NVFP4)")
    ac, wc = a.c(), w.c()
    qc = out_q.c() if out_q is not None else None
    _check("ds4g_grouped_gemm_fp4",
           _lib.ds4g_grouped_gemm_fp4(ctypes.byref(ac), offsets.data_ptr(), E, max_rows_per_expert, ctypes.byref(wc),
                                      N, epilogue, _ptr(out), ctypes.byref(qc) if qc is not None else None,
                                      _ptr(h_debug), _stream()))
    return out if epilogue == EPI_NONE else out_q


def ds4g_grouped_gemm_fp4_combine(a, offsets, E, max_rows_per_expert, w, N, row_to_slot, route_w, out=None):
    """FC2 with the weighted combine fused: out [T][N] (zeroed by the call)."""
    T, k = route_w.shape
    if out is None:
        out = torch.empty((T, N), dtype=torch.float32, device=a.data.device)
    ac, wc = a.c(), w.c()
    _check("ds4g_grouped_gemm_fp4_combine",
           _lib.ds4g_grouped_gemm_fp4_combine(ctypes.byref(ac), offsets.data_ptr(), E, max_rows_per_expert,
                                              ctypes.byref(wc), N, row_to_slot.data_ptr(), route_w.data_ptr(), T, k,
                                              out.data_ptr(), _stream()))
    return out


def ds4g_grouped_gemm_fp4_combine_chained(a, offsets, E, max_rows_per_expert, w, N, row_to_slot, route_w, out):
    """FC2 with the combine added into out [T][N] (not zeroed), launched to
    overlap the previous kernel on the stream (the FC1 call that wrote a)."""
    T, k = route_w.shape
    ac, wc = a.c(), w.c()
    _check("ds4g_grouped_gemm_fp4_combine_chained",
           _lib.ds4g_grouped_gemm_fp4_combine_chained(ctypes.byref(ac), offsets.data_ptr(), E, max_rows_per_expert,
                                                      ctypes.byref(wc), N, row_to_slot.data_ptr(),
                                                      route_w.data_ptr(), T, k, out.data_ptr(), _stream()))
    return out


def ffn_supported(fmt, d, I, E):
    """whether ds4g_moe_ffn_fp4 takes these shapes (the decode kernel's tiling
    of both GEMMs, as include/ds4g.h states it)"""
    kmul = 512 if fmt == MXFP4 else 256
    return (fmt in (MXFP4, NVFP4) and 1 <= E <= 512 and d % kmul == 0 and I % kmul == 0 and I % 64 == 0
            and d % 128 == 0)


def ffn_counters(E, device="cuda"):
    """the zeroed per-expert counters [E + 1] that ds4g_moe_ffn_fp4 needs"""
    return torch.zeros(E + 1, dtype=torch.int32, device=device)


def ds4g_moe_ffn_fp4(a, offsets, E, max_rows_per_expert, w1, w2, d, I, h_q, row_to_slot, route_w, out, counters):
    """FC1 + SwiGLU/requantisation into h_q, then FC2 with the combine added
    into out [T][d] (not zeroed), as one launch (decode sizes); counters:
    int32 [E + 1], zero before the call and after it."""
    T, k = route_w.shape
    ac, w1c, w2c, hc = a.c(), w1.c(), w2.c(), h_q.c()
    _check("ds4g_moe_ffn_fp4",
           _lib.ds4g_moe_ffn_fp4(ctypes.byref(ac), offsets.data_ptr(), E, max_rows_per_expert, ctypes.byref(w1c),
                                 ctypes.byref(w2c), d, I, ctypes.byref(hc), row_to_slot.data_ptr(),
                                 route_w.data_ptr(), T, k, out.data_ptr(), counters.data_ptr(), _stream()))
    return out


def ds4g_zero_fill(t):
    """zero-fills a device tensor on the current stream"""
    _check("ds4g_zero_fill", _lib.ds4g_zero_fill(t.data_ptr(), t.numel() * t.element_size(), _stream()))
    return t


def ds4g_swiglu_requant(y1, fmt, h_q=None, h_debug=None, g_h=None):
    rows, two_i = y1.shape
    I = two_i // 2
    if h_q is None:
        h_q = Fp4Tensor.empty(rows, I, fmt, y1.device)
        if fmt == NVFP4 and g_h is not None:
            h_q.g.copy_(g_h)
    hc = h_q.c()
    _check("ds4g_swiglu_requant", _lib.ds4g_swiglu_requant(y1.data_ptr(), rows, I, fmt, ctypes.byref(hc),
                                                           _ptr(h_debug), _stream()))
    return h_q


def ds4g_moe_combine(y2, slot_to_row, w, out=None):
    T, k = w.shape
    d = y2.shape[1]
    if out is None:
        out = torch.empty((T, d), dtype=torch.float32, device=y2.device)
    _check("ds4g_moe_combine", _lib.ds4g_moe_combine(y2.data_ptr(), slot_to_row.data_ptr(), w.data_ptr(), T, k, d,
                                                     out.data_ptr(), _stream()))
    return out


def ds4g_segment_ids(offsets, nseg, modulo, rows, out=None):
    """out[r] = (group of row offsets[0] + r) % modulo, int32 [rows]"""
    if out is None:
        out = torch.empty(max(rows, 1), dtype=torch.int32, device=offsets.device)
    _check("ds4g_segment_ids", _lib.ds4g_segment_ids(offsets.data_ptr(), nseg, modulo, rows, out.data_ptr(),
                                                     _stream()))
    return out[:rows]
