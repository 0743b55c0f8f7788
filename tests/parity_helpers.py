"""Shared helpers of the GPU parity tests: moving FP4 tensors between the
oracle (numpy) and the library (torch device tensors), and the acceptance
rules: bit-exact for bytes / indices, the per-element GEMM bound
|gpu - ref| <= 1e-5 * sum_k |a_k w_k| + 1e-6, and a validity rule for FP4
codes that the GPU derives from fp32 values that legitimately differ from the
oracle's in the last bits."""
import numpy as np
import torch

import oracle
from block_scaled_fp4_topk_b200 import ds4g

E2M1_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
GEMM_REL = 1e-5
GEMM_ABS = 1e-6


def dev():
    return torch.device("cuda:0")


def to_dev(t, device=None, g_per_expert=None):
    device = device or dev()
    g = None
    if t.fmt == oracle.NV:
        gv = g_per_expert if g_per_expert is not None else [t.g]
        g = torch.tensor(np.asarray(gv, np.float32), device=device)
    return ds4g.Fp4Tensor(torch.from_numpy(np.ascontiguousarray(t.data)).to(device),
                          torch.from_numpy(np.ascontiguousarray(t.scales)).to(device), g, t.fmt)


def from_dev(t):
    g = float(t.g[0].item()) if t.g is not None else 1.0
    return oracle.Fp4(t.data.cpu().numpy(), t.scales.cpu().numpy(), g, t.fmt)


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev())


def unpack(data):
    data = np.asarray(data, np.uint8)
    out = np.empty(data.shape[:-1] + (data.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = data & 0x0F
    out[..., 1::2] = data >> 4
    return out


def swiglu_eval_bound(g, h):
    """Bound on |h_gpu - silu(g) u| for the kernels' fp32 evaluation
    g u / (1 + e^-g) from their own g and u, with the hardware's fast
    exponential and division.  Documented bounds (CUDA C Programming Guide,
    intrinsic functions): __expf(x) within 2 + floor(1.173 |x|) ulp,
    __fdividef within 2 ulp for divisors in [2^-126, 2^126], 0 when the
    divisor is beyond 2^126 (|g| above ~87, where |h| < 1e-36).  To first
    order the relative error is (2 + 1.173 |g|) 2^-23 from e^-g, plus
    2^-24 for the add, 2^-24 for g u and 2^-22 for the division:
    (5 + 1.173 |g|) 2^-23; (6 + 1.2 |g|) 2^-23 leaves room for the
    second-order terms.  A further 2^-22 |h| covers the NVFP4 codes, which
    the fused epilogues take from h times the correctly rounded reciprocal of
    the block's divisor (within 1.5 ulp of the quotient)."""
    g = np.abs(np.asarray(g, np.float64))
    return ((6.0 + 1.2 * g) * 2.0 ** -23 + 2.0 ** -22) * np.abs(h) + 1e-30


def assert_gemm_close(gpu, ref, abssum, what=""):
    gpu = np.asarray(gpu, np.float64)
    bound = GEMM_REL * abssum + GEMM_ABS
    err = np.abs(gpu - ref)
    bad = err > bound
    assert not np.any(np.isnan(gpu)), f"{what}: NaN in GPU output"
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements outside the bound; worst excess "
                           f"{(err - bound).max():.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}")


def _scale_values(t):
    blk = oracle.BLOCK[t.fmt]
    sb = np.repeat(np.asarray(t.scales, np.int64), blk, axis=1)
    if t.fmt == oracle.MX:
        return np.ldexp(1.0, sb - 127)
    vals = np.array([oracle.ue4m3_decode(b) for b in range(128)])
    return vals[sb & 0x7F] * t.g


def check_requant(gpu_q, h_ref, delta, fmt, g=1.0, min_exact=0.999):
    """gpu_q: oracle.Fp4 read back from the GPU; h_ref: the oracle's h
    (float64); delta: per-element bound on |h_gpu - h_ref| from the fp32
    arithmetic.  Codes must match the oracle's quantisation of h_ref, except
    where a value within delta of h_ref would round (or scale) differently:
    there the GPU's decoded value must be a valid rounding of such a value."""
    ref_q = oracle.quantize(h_ref.astype(np.float32), fmt, g=g if fmt == oracle.NV else None)
    cg, cr = unpack(gpu_q.data), unpack(ref_q.data)
    same_codes = cg == cr
    blk = oracle.BLOCK[fmt]
    same_scale = np.repeat(gpu_q.scales == ref_q.scales, blk, axis=1)
    exact = same_codes & same_scale
    frac = exact.mean()
    assert frac >= min_exact, f"only {frac:.6f} of the codes match the oracle"
    if exact.all():
        return frac
    sc = _scale_values(gpu_q)
    mag = E2M1_POS[cg & 7]
    val = np.where(cg & 8, -mag, mag) * sc
    # grid spacing around each code (0.5 below 2, 1 below 4, 2 above)
    step = np.where((cg & 7) >= 6, 2.0, np.where((cg & 7) >= 4, 1.0, 0.5)) * sc
    tol = 0.5 * step + delta * 1.000001 + 1e-12
    sat = ((cg & 7) == 7) & (np.abs(h_ref) + delta >= 5.0 * sc)
    ok = exact | (np.abs(h_ref - val) <= tol) | sat
    # a differing scale must come from a block amax that sits within delta of
    # the decision threshold; check that every differing block's ratio is one step
    if not (gpu_q.scales == ref_q.scales).all():
        d = np.abs(gpu_q.scales.astype(np.int64) - ref_q.scales.astype(np.int64))
        assert d.max() <= 1, "a block scale differs by more than one step"
    assert ok.all(), f"{(~ok).sum()} FP4 codes are not a valid rounding of the oracle's values"
    return frac
