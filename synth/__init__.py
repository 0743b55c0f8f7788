"""Seeded synthetic inputs for the FP4 MoE path (shared by the oracle side and
the GPU side; holds none of the method's arithmetic).

The generator is splitmix64 evaluated at a counter, turned into standard
normals by Box-Muller with its own log / sin / cos written with IEEE double
+ - * / and sqrt only (see synth_core.h), so the host fill (``fill_*``) and
the device fill (``cuda_fill_*``) return identical bits for the same
(seed, stream, index).

Stream numbering (one stream per tensor, one per expert for weights, so one
expert's weights can be regenerated on its own):
    STREAM_X       layer input activations x [T][d]
    STREAM_LOGITS  router logits [T][E]
    STREAM_BIAS    per-expert router bias [E]
    STREAM_W1 + e  expert e FC1 weights [2I][d] (gate rows then up rows)
    STREAM_W2 + e  expert e FC2 weights [d][I]
    STREAM_WS1 / STREAM_WS2  the shared expert's FC1 [2I][d] / FC2 [d][I] weights
"""
import ctypes
import os

import numpy as np

from . import build as _build

STREAM_X = 1
STREAM_LOGITS = 2
STREAM_BIAS = 3
STREAM_AUX = 4
STREAM_W1 = 1 << 20
STREAM_W2 = 2 << 20
STREAM_WS1 = 1 << 22
STREAM_WS2 = (1 << 22) + 1

_host = None
_cuda = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(_build.HOST_LIB):
            _build.build(cuda=False)
        L = ctypes.CDLL(_build.HOST_LIB)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.synth_u64.restype = u64
        L.synth_u64.argtypes = [u64, u64, u64]
        L.synth_normal.restype = dbl
        L.synth_normal.argtypes = [u64, u64, u64]
        L.synth_fill_normal_f32.argtypes = [vp, i64, u64, u64, dbl, i64]
        L.synth_fill_normal_bf16.argtypes = [vp, i64, u64, u64, dbl, i64]
        L.synth_fill_logits.argtypes = [vp, i64, i64, u64, u64, u64, dbl]
        _host = L
    return _host


def _cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(_build.CUDA_LIB):
            raise RuntimeError("synth: device generator library missing; run synth/build.py")
        L = ctypes.CDLL(_build.CUDA_LIB)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.synth_cuda_fill_normal_f32.argtypes = [vp, i64, u64, u64, dbl, i64, vp]
        L.synth_cuda_fill_normal_bf16.argtypes = [vp, i64, u64, u64, dbl, i64, vp]
        L.synth_cuda_fill_logits.argtypes = [vp, i64, i64, u64, u64, u64, dbl, vp]
        for f in (L.synth_cuda_fill_normal_f32, L.synth_cuda_fill_normal_bf16, L.synth_cuda_fill_logits):
            f.restype = ctypes.c_int
        _cuda = L
    return _cuda


# ---- host fills (numpy) ----------------------------------------------------

def u64(seed, stream, i):
    return _host_lib().synth_u64(seed, stream, i)


def normal(seed, stream, i):
    return _host_lib().synth_normal(seed, stream, i)


def normal_f32(shape, seed, stream, sigma=1.0, offset=0):
    out = np.empty(shape, dtype=np.float32)
    _host_lib().synth_fill_normal_f32(out.ctypes.data, out.size, seed, stream, float(sigma), int(offset))
    return out


def normal_bf16_bits(shape, seed, stream, sigma=1.0, offset=0):
    """bf16 values as their uint16 bit patterns"""
    out = np.empty(shape, dtype=np.uint16)
    _host_lib().synth_fill_normal_bf16(out.ctypes.data, out.size, seed, stream, float(sigma), int(offset))
    return out


def bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def logits(T, E, seed, bias_sigma=0.0):
    out = np.empty((T, E), dtype=np.float32)
    _host_lib().synth_fill_logits(out.ctypes.data, T, E, seed, STREAM_LOGITS, STREAM_BIAS, float(bias_sigma))
    return out


# ---- device fills (raw device pointers; stream = cudaStream_t as int) ------

def _chk(rc, what):
    if rc != 0:
        raise RuntimeError(f"synth: {what} failed with CUDA error {rc}")


def cuda_fill_normal_f32(ptr, n, seed, stream, sigma=1.0, offset=0, cuda_stream=0):
    _chk(_cuda_lib().synth_cuda_fill_normal_f32(ptr, n, seed, stream, float(sigma), int(offset), cuda_stream),
         "fill_normal_f32")


def cuda_fill_normal_bf16(ptr, n, seed, stream, sigma=1.0, offset=0, cuda_stream=0):
    _chk(_cuda_lib().synth_cuda_fill_normal_bf16(ptr, n, seed, stream, float(sigma), int(offset), cuda_stream),
         "fill_normal_bf16")


def cuda_fill_logits(ptr, T, E, seed, bias_sigma=0.0, cuda_stream=0):
    _chk(_cuda_lib().synth_cuda_fill_logits(ptr, T, E, seed, STREAM_LOGITS, STREAM_BIAS, float(bias_sigma),
                                            cuda_stream), "fill_logits")
