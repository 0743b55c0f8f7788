"""GPU parity of the FP8-activation x FP4-weight variant (the
m_grouped_fp8_fp4_gemm_nt_contiguous API of "[DeepSeek V4] Triton FP4
optimisation in practice", "Step 0"; the SwiGLU + FP8 quantisation pattern of
"Moore Threads full-link adaptation of DeepSeek-V4"): activations and h in
MXFP8 (E4M3 + UE8M0 per 32), weights in MXFP4, the block-scaled MMA
kind::mxf8f6f4.  Against the CPU oracle on the same seeded inputs, through the
C ABI:
  - MXFP8 quantisation and the permutation of MXFP8 rows: bit-exact;
  - grouped GEMMs: |gpu - ref| <= 1e-5 * sum|a w| + 1e-6 per element;
  - fused SwiGLU + FP8 requantisation: h within its propagated bound, and
    its E4M3 codes and scales bit-exact against the oracle's quantisation of
    the GPU's own h (the step is exact power-of-two scaling and one RNE
    conversion);
  - FC2 with the weighted combine: per element; a whole layer: relative
    L2 <= 1e-2 against the oracle's chain."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_helpers import assert_gemm_close, bf16_dev, dev, from_dev, swiglu_eval_bound, to_dev

pytestmark = pytest.mark.gpu

ds4g = pytest.importorskip("block_scaled_fp4_topk_b200.ds4g")
MX, MX8 = oracle.MX, oracle.MX8


def _x(rows, K, stream, sigma=1.0):
    return synth.normal_f32((rows, K), 0, stream, sigma)


@pytest.mark.parametrize("src", ["bf16", "f32"])
@pytest.mark.parametrize("rows,K", [(37, 7168), (5, 64), (3, 2048)])
def test_quantize_mx8_bitexact(src, rows, K):
    x = _x(rows, K, 71, 2.0)
    x[0, :64] = 0.0
    x[0, 64:96] = -0.0
    if rows >= 3:
        x[1, :32] *= 1e-38            # subnormal-range block
        x[1, 32:64] = 3e4             # large block
        x[2, :32] = 1.0
        x[2, 5] = 1.0625 / 256        # ties of the E4M3 grid at the block's scale
        x[2, 6] = 1.1875 / 256
    if src == "bf16":
        bits = ((x.view(np.uint32) + 0x7FFF + ((x.view(np.uint32) >> 16) & 1)) >> 16).astype(np.uint16)
        xin, xf = bf16_dev(bits), synth.bf16_bits_to_f32(bits)
    else:
        xin, xf = torch.from_numpy(x).to(dev()), x
    q = ds4g.ds4g_quantize_mx(xin, MX8)
    ref = oracle.quantize(xf, MX8)
    assert q.data.shape == (rows, K)
    assert np.array_equal(q.scales.cpu().numpy(), ref.scales)
    assert np.array_equal(q.data.cpu().numpy(), ref.data)


@pytest.mark.parametrize("T,k,E", [(16, 2, 8), (300, 6, 64), (1, 6, 256)])
def test_permute_mx8_bitexact(T, k, E):
    K = 512
    lg = synth.logits(T, E, 0, 1.5)
    idx, _ = oracle.route_topk(lg, k)
    xq = oracle.quantize(_x(T, K, 72), MX8)
    x_d = ds4g.Fp4Tensor(torch.from_numpy(xq.data).to(dev()), torch.from_numpy(xq.scales).to(dev()), None, MX8)
    offs, r2s, s2r, a = ds4g.ds4g_moe_permute(torch.from_numpy(idx).to(dev()), E, x_d)
    roffs, rr2s, rs2r = oracle.moe_permute(idx, E)
    assert np.array_equal(offs.cpu().numpy(), roffs)
    assert np.array_equal(r2s.cpu().numpy(), rr2s) and np.array_equal(s2r.cpu().numpy(), rs2r)
    ra = oracle.gather_rows(xq, rr2s, k)
    assert np.array_equal(a.data.cpu().numpy(), ra.data) and np.array_equal(a.scales.cpu().numpy(), ra.scales)


def _problem(seg, N, K, stream):
    E = len(seg)
    offsets = np.concatenate([[0], np.cumsum(seg)]).astype(np.int32)
    S = int(offsets[-1])
    a = oracle.quantize(_x(S, K, stream), MX8)
    w = oracle.quantize(synth.normal_f32((E * N, K), 0, stream + 1, 0.02), MX)
    return offsets, a, w


def _dev8(t):
    return ds4g.Fp4Tensor(torch.from_numpy(np.ascontiguousarray(t.data)).to(dev()),
                          torch.from_numpy(np.ascontiguousarray(t.scales)).to(dev()), None, t.fmt)


def _ref(a, offsets, w, N):
    S = a.data.shape[0]
    out, ab = np.full((S, N), np.nan), np.full((S, N), np.nan)
    for e in range(len(offsets) - 1):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            we = oracle.Fp4(w.data[e * N:(e + 1) * N], w.scales[e * N:(e + 1) * N], 1.0, MX)
            out[r0:r1], ab[r0:r1] = oracle.expert_gemm_rows(a, np.arange(r0, r1), we, (0, N))
    return out, ab


# the tensor-core kernel takes every FP8 call (K % 512, N % 224 or % 256);
# short segments, empty experts and the dense shape included
CASES = [([300, 0, 1, 129, 77], 512, 512), ([130, 20], 448, 1024), ([5, 3], 256, 512), ([17, 600], 672, 1024),
         ([64], 4096, 7168)]


@pytest.mark.parametrize("case", CASES)
def test_grouped_gemm_fp8_fp4(case):
    seg, N, K = case
    offsets, a, w = _problem(seg, N, K, 73)
    out = ds4g.ds4g_grouped_gemm_fp4(_dev8(a), torch.from_numpy(offsets).to(dev()), len(seg), max(seg), to_dev(w), N)
    ds4g.ds4g_check_device()
    ref, ab = _ref(a, offsets, w, N)
    assert_gemm_close(out.cpu().numpy(), ref, ab, f"fp8 x fp4 {case}")


def _h_bound(y1, ab1, I):
    g, u = y1[:, :I], y1[:, I:]
    dg, du = 1e-5 * ab1[:, :I] + 1e-6, 1e-5 * ab1[:, I:] + 1e-6
    sig = 1.0 / (1.0 + np.exp(-g))
    h = g * sig * u
    return h, np.abs(sig * (1 + g * (1 - sig))) * np.abs(u) * dg + np.abs(g * sig) * du + swiglu_eval_bound(g, h)


@pytest.mark.parametrize("case", [([300, 0, 1, 129, 77], 256, 512), ([17, 140], 384, 1024), ([3, 5], 128, 512)])
def test_fc1_fp8_swiglu_fp8_requant(case):
    seg, I, K = case
    offsets, a, w = _problem(seg, 2 * I, K, 74)
    S = int(offsets[-1])
    hq = ds4g.Fp4Tensor.empty(S, I, MX8, dev())
    hdbg = torch.empty((S, I), dtype=torch.float32, device=dev())
    ds4g.ds4g_grouped_gemm_fp4(_dev8(a), torch.from_numpy(offsets).to(dev()), len(seg), max(seg), to_dev(w), 2 * I,
                               ds4g.EPI_SWIGLU_REQUANT, out_q=hq, h_debug=hdbg)
    ds4g.ds4g_check_device()
    y1, ab1 = _ref(a, offsets, w, 2 * I)
    h_ref, dh = _h_bound(y1, ab1, I)
    h_gpu = hdbg.cpu().numpy()
    assert np.all(np.abs(h_gpu.astype(np.float64) - h_ref) <= dh * 1.000001), "h outside its bound"
    requant = oracle.quantize(h_gpu, MX8)
    assert np.array_equal(hq.scales.cpu().numpy(), requant.scales)
    assert np.array_equal(hq.data.cpu().numpy(), requant.data)


@pytest.mark.parametrize("T,k,E,N,K", [(300, 6, 16, 512, 1024), (300, 6, 16, 448, 1024), (3, 6, 64, 256, 512)])
def test_fc2_fp8_combine(T, k, E, N, K):
    lg = synth.logits(T, E, 0, 1.5)
    idx, rw = oracle.route_topk(lg, k)
    offsets, r2s, s2r = oracle.moe_permute(idx, E)
    a = oracle.quantize(_x(T * k, K, 75), MX8)
    W = oracle.quantize(synth.normal_f32((E * N, K), 0, 76, 0.02), MX)
    w32 = rw.astype(np.float32)
    out = ds4g.ds4g_grouped_gemm_fp4_combine(_dev8(a), torch.from_numpy(offsets).to(dev()), E, T, to_dev(W), N,
                                             torch.from_numpy(r2s).to(dev()), torch.from_numpy(w32).to(dev()))
    ds4g.ds4g_check_device()
    y2, ab = _ref(a, offsets, W, N)
    w64 = w32.astype(np.float64)
    ref = oracle.moe_combine(y2, s2r, w64)
    bound = (oracle.moe_combine(1e-5 * ab + 1e-6, s2r, np.abs(w64)) +
             1e-6 * oracle.moe_combine(np.abs(y2), s2r, np.abs(w64)) + 1e-7)
    got = out.cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound), f"worst excess {(np.abs(got - ref) - bound).max():.3e}"


def test_layer_fp8_activations():
    """a whole layer with FP8 activations and FP4 weights (64 tokens, 8
    experts, top-2, d = I = 512) against the oracle's chain: routing, MXFP8
    quantisation, FC1, SwiGLU, MXFP8 requantisation, FC2, combine"""
    from synth import workloads
    from block_scaled_fp4_topk_b200.layer import MoeLayer
    from bench import synthetic_weights
    wl = workloads.Workload("fp8_small", T=64, E=8, k=2, d=512, I=512, fmt=MX, bias_sigma=1.5, act_fmt=MX8)
    w1, w2 = synthetic_weights(wl.E, wl.d, wl.I, MX, device=dev())
    layer = MoeLayer(w1, w2, wl.E, wl.k, wl.d, wl.I, MX, act_fmt=ds4g.MXFP8)
    xb, lg = workloads.host_x_bits(wl), workloads.host_logits(wl)
    out = layer.forward(bf16_dev(xb), torch.from_numpy(lg).to(dev())).cpu().numpy().astype(np.float64)
    ds4g.ds4g_check_device()
    W1 = oracle.quantize(np.concatenate([workloads.host_w1(wl, e) for e in range(wl.E)]), MX)
    W2 = oracle.quantize(np.concatenate([workloads.host_w2(wl, e) for e in range(wl.E)]), MX)
    assert np.array_equal(from_dev(w1).data, W1.data)
    idx, w = oracle.route_topk(lg, wl.k)
    xq = oracle.quantize(synth.bf16_bits_to_f32(xb), MX8)
    offsets, r2s, s2r = oracle.moe_permute(idx, wl.E)
    a = oracle.gather_rows(xq, r2s, wl.k)
    y1, _ = _ref(a, offsets, W1, 2 * wl.I)
    hq = oracle.quantize(oracle.swiglu(y1.astype(np.float32)), MX8)
    y2, _ = _ref(hq, offsets, W2, wl.d)
    ref = oracle.moe_combine(y2.astype(np.float32).astype(np.float64), s2r, w)
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel <= 1e-2, rel


@pytest.mark.parametrize("case", [([64], 1024, 512), ([300, 0, 129], 448, 1024), ([64], 4096, 7168)])
def test_grouped_gemm_fp8_fp8(case):
    """MXFP8 activations x MXFP8 weights (the shared expert's Q8 weights of
    "DGX Spark native FP4 matrix instructions ...", sec. 2): per element"""
    seg, N, K = case
    E = len(seg)
    offsets = np.concatenate([[0], np.cumsum(seg)]).astype(np.int32)
    a = oracle.quantize(_x(int(offsets[-1]), K, 77), MX8)
    w = oracle.quantize(synth.normal_f32((E * N, K), 0, 78, 0.02), MX8)
    out = ds4g.ds4g_grouped_gemm_fp4(_dev8(a), torch.from_numpy(offsets).to(dev()), E, max(seg), _dev8(w), N)
    ds4g.ds4g_check_device()
    ref, ab = oracle.grouped_gemm(a, offsets, w, N)
    assert_gemm_close(out.cpu().numpy(), ref, ab, f"fp8 x fp8 {case}")


def test_layer_fp8_with_shared_expert():
    """the FP8-activation layer plus a shared expert with FP8 weights that
    every token goes through (64 tokens, 8 routed experts, top-2, d = I = 512)
    against the oracle's chain of both, summed"""
    from synth import workloads
    from block_scaled_fp4_topk_b200.layer import MoeLayer
    from bench import synthetic_shared_weights, synthetic_weights
    wl = workloads.Workload("fp8_shared", T=64, E=8, k=2, d=512, I=512, fmt=MX, bias_sigma=1.5, act_fmt=MX8)
    w1, w2 = synthetic_weights(wl.E, wl.d, wl.I, MX, device=dev())
    ws1, ws2 = synthetic_shared_weights(wl.d, wl.I, device=dev())
    layer = MoeLayer(w1, w2, wl.E, wl.k, wl.d, wl.I, MX, act_fmt=ds4g.MXFP8, shared=(ws1, ws2))
    xb, lg = workloads.host_x_bits(wl), workloads.host_logits(wl)
    out = layer.forward(bf16_dev(xb), torch.from_numpy(lg).to(dev())).cpu().numpy().astype(np.float64)
    ds4g.ds4g_check_device()
    W1 = oracle.quantize(np.concatenate([workloads.host_w1(wl, e) for e in range(wl.E)]), MX)
    W2 = oracle.quantize(np.concatenate([workloads.host_w2(wl, e) for e in range(wl.E)]), MX)
    WS1, WS2 = oracle.quantize(workloads.host_ws1(wl), MX8), oracle.quantize(workloads.host_ws2(wl), MX8)
    assert np.array_equal(ws1.data.cpu().numpy(), WS1.data) and np.array_equal(ws2.scales.cpu().numpy(), WS2.scales)
    idx, w = oracle.route_topk(lg, wl.k)
    xq = oracle.quantize(synth.bf16_bits_to_f32(xb), MX8)
    offsets, r2s, s2r = oracle.moe_permute(idx, wl.E)
    a = oracle.gather_rows(xq, r2s, wl.k)
    y1, _ = _ref(a, offsets, W1, 2 * wl.I)
    hq = oracle.quantize(oracle.swiglu(y1.astype(np.float32)), MX8)
    y2, _ = _ref(hq, offsets, W2, wl.d)
    routed = oracle.moe_combine(y2.astype(np.float32).astype(np.float64), s2r, w)
    all_rows = np.array([0, wl.T], np.int32)
    ys1, _ = oracle.grouped_gemm(xq, all_rows, WS1, 2 * wl.I)
    hs = oracle.quantize(oracle.swiglu(ys1.astype(np.float32)), MX8)
    ys2, _ = oracle.grouped_gemm(hs, all_rows, WS2, wl.d)
    ref = routed + ys2.astype(np.float32).astype(np.float64)
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel <= 1e-2, rel
