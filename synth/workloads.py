"""The seeded synthetic workloads (shapes, distributions, streams).

Each workload follows the problem statement's configurations; all draws come
from the splitmix64 / Box-Muller generator of this package with seed 0:
    x       bf16 [T][d]   ~ N(0, 1)                      stream STREAM_X
    logits  fp32 [T][E]   ~ N(0, 1) (+ bias_e ~ N(0, 1.5) added in fp32 for
                          the prefill workloads)          STREAM_LOGITS / _BIAS
    W1[e]   fp32 [2I][d]  ~ N(0, 0.02), gate rows then up rows   STREAM_W1 + e
    W2[e]   fp32 [d][I]   ~ N(0, 0.02)                            STREAM_W2 + e
The dense workload is one expert (E = 1, k = 1) whose FC1 is skipped: only
W = W1[0] rows [0, N) against M rows of x, so it uses the same streams.

NVFP4 tensor scale of h (the SwiGLU output, quantised inside the FC1
epilogue where its amax is not yet known) is a static calibration constant:
g_h = fp32(H_CAL / 2688) with H_CAL = 128, i.e. |h| up to 128 is covered
without saturating the UE4M3 block scale.
"""
from dataclasses import dataclass

import numpy as np

from . import STREAM_BIAS, STREAM_LOGITS, STREAM_W1, STREAM_W2, STREAM_WS1, STREAM_WS2, STREAM_X

W_SIGMA = 0.02
BIAS_SIGMA = 1.5
H_CAL = 128.0
G_H = float(np.float32(np.float32(H_CAL) / np.float32(2688.0)))
MX, NV, MX8 = 0, 1, 2


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    E: int
    k: int
    d: int
    I: int
    fmt: int
    bias_sigma: float
    dense: bool = False   # one expert, FC1-shaped single GEMM only (N = I rows)
    act_fmt: int = -1     # activations' format: the weights' by default; 2 = MXFP8 (FP8 x FP4)

    @property
    def afmt(self):
        return self.fmt if self.act_fmt < 0 else self.act_fmt

    @property
    def S(self):
        return self.T * self.k

    @property
    def N1(self):
        return 2 * self.I


WORKLOADS = {
    "tiny": Workload("tiny", T=16, E=8, k=2, d=256, I=128, fmt=MX, bias_sigma=0.0),
    "dense_m1": Workload("dense_m1", T=1, E=1, k=1, d=7168, I=4096, fmt=MX, bias_sigma=0.0, dense=True),
    "dense_m64": Workload("dense_m64", T=64, E=1, k=1, d=7168, I=4096, fmt=MX, bias_sigma=0.0, dense=True),
    "decode_t1": Workload("decode_t1", T=1, E=256, k=6, d=7168, I=2048, fmt=MX, bias_sigma=0.0),
    "decode_t4": Workload("decode_t4", T=4, E=256, k=6, d=7168, I=2048, fmt=MX, bias_sigma=0.0),
    "decode_t8": Workload("decode_t8", T=8, E=256, k=6, d=7168, I=2048, fmt=MX, bias_sigma=0.0),
    "prefill": Workload("prefill", T=2048, E=256, k=6, d=7168, I=2048, fmt=MX, bias_sigma=BIAS_SIGMA),
    "prefill16k": Workload("prefill16k", T=16384, E=256, k=6, d=7168, I=2048, fmt=NV, bias_sigma=BIAS_SIGMA),
    # profiling stand-in for "prefill": same per-expert shapes and skew, 64
    # experts (1.5 GB of weights) so that ncu's multi-pass replay stays small
    "prof_prefill": Workload("prof_prefill", T=512, E=64, k=6, d=7168, I=2048, fmt=MX, bias_sigma=BIAS_SIGMA),
    # FP8 activations (MXFP8: E4M3 + UE8M0 per 32) x MXFP4 weights, the
    # m_grouped_fp8_fp4_gemm_nt_contiguous variant, at the prefill layer's shape
    "prefill_fp8": Workload("prefill_fp8", T=2048, E=256, k=6, d=7168, I=2048, fmt=MX, bias_sigma=BIAS_SIGMA,
                            act_fmt=MX8),
    # the same for "prefill16k": NVFP4, 64 experts (1.6 GB of weights) and
    # 4096 tokens, i.e. the same 384 rows per expert on average
    "prof_prefill16k": Workload("prof_prefill16k", T=4096, E=64, k=6, d=7168, I=2048, fmt=NV,
                                bias_sigma=BIAS_SIGMA),
    # profiling stand-in for "decode_t8": 64 experts (1.5 GB of weights per
    # layer) and the same 48 routed slots
    "prof_decode_t8": Workload("prof_decode_t8", T=8, E=64, k=6, d=7168, I=2048, fmt=MX, bias_sigma=0.0),
}


def host_w1(wl: Workload, e: int, seed: int = 0):
    from . import normal_f32
    rows = wl.I if wl.dense else 2 * wl.I
    return normal_f32((rows, wl.d), seed, STREAM_W1 + e, W_SIGMA)


def host_w2(wl: Workload, e: int, seed: int = 0):
    from . import normal_f32
    return normal_f32((wl.d, wl.I), seed, STREAM_W2 + e, W_SIGMA)


def host_ws1(wl: Workload, seed: int = 0):
    """the shared expert's FC1 weights, fp32 [2I][d] ~ N(0, 0.02)"""
    from . import normal_f32
    return normal_f32((2 * wl.I, wl.d), seed, STREAM_WS1, W_SIGMA)


def host_ws2(wl: Workload, seed: int = 0):
    """the shared expert's FC2 weights, fp32 [d][I] ~ N(0, 0.02)"""
    from . import normal_f32
    return normal_f32((wl.d, wl.I), seed, STREAM_WS2, W_SIGMA)


def host_x_bits(wl: Workload, seed: int = 0):
    from . import normal_bf16_bits
    return normal_bf16_bits((wl.T, wl.d), seed, STREAM_X, 1.0)


def host_logits(wl: Workload, seed: int = 0):
    from . import logits
    return logits(wl.T, wl.E, seed, wl.bias_sigma)
