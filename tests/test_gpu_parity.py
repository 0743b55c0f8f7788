"""GPU parity: every library call against the CPU oracle on the same seeded
inputs, through the C ABI.  Bytes, indices and offsets bit-exact; GEMM
outputs within |gpu - ref| <= 1e-5 * sum|a w| + 1e-6 per element; FP4 codes
that the GPU derives from its own fp32 arithmetic checked for validity
against the oracle's values; full layers within relative L2 <= 1e-2."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_helpers import (assert_gemm_close, bf16_dev, check_requant, dev, from_dev, swiglu_eval_bound, to_dev,
                            unpack)
from synth.workloads import G_H

pytestmark = pytest.mark.gpu

ds4g = pytest.importorskip("block_scaled_fp4_topk_b200.ds4g")
MX, NV = oracle.MX, oracle.NV


def _x_f32(rows, K, stream, sigma=1.0):
    return synth.normal_f32((rows, K), 0, stream, sigma)


# ---- generator: host and device produce the same bits ----------------------

def test_generator_device_matches_host():
    n = 1 << 20
    ref = synth.normal_f32((n,), 0, 4242, 0.02, offset=12345)
    buf = torch.empty(n, dtype=torch.float32, device=dev())
    synth.cuda_fill_normal_f32(buf.data_ptr(), n, 0, 4242, 0.02, 12345, torch.cuda.current_stream().cuda_stream)
    assert np.array_equal(buf.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    bits = synth.normal_bf16_bits((n,), 0, synth.STREAM_X)
    bb = torch.empty(n, dtype=torch.int16, device=dev())
    synth.cuda_fill_normal_bf16(bb.data_ptr(), n, 0, synth.STREAM_X, 1.0, 0, torch.cuda.current_stream().cuda_stream)
    assert np.array_equal(bb.cpu().numpy().view(np.uint16), bits)
    lg = synth.logits(64, 256, 0, 1.5)
    lt = torch.empty((64, 256), dtype=torch.float32, device=dev())
    synth.cuda_fill_logits(lt.data_ptr(), 64, 256, 0, 1.5, torch.cuda.current_stream().cuda_stream)
    assert np.array_equal(lt.cpu().numpy().view(np.uint32), lg.view(np.uint32))


# ---- quantisation ------------------------------------------------------------

def _special_rows(x):
    x = x.copy()
    x[0, :64] = 0.0
    x[0, 64:96] = -0.0
    x[1, :32] *= 1e-38          # subnormal-range block
    x[1, 32:64] = 3e4           # large block
    x[2, 5] = 6.0 * 2 ** 10     # exact grid values / ties
    x[2, 6] = 5.0 * 2 ** 10
    x[2, 7] = -2.5 * 2 ** 10
    return x


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("src", ["bf16", "f32"])
@pytest.mark.parametrize("rows,K", [(37, 7168), (5, 64), (1, 2048)])
def test_quantize_bitexact(fmt, src, rows, K):
    x = _special_rows(_x_f32(rows, K, 7)) if rows >= 3 else _x_f32(rows, K, 7)
    if src == "bf16":
        bits = (x.view(np.uint32) + 0x7FFF + ((x.view(np.uint32) >> 16) & 1)) >> 16
        bits = bits.astype(np.uint16)
        xin = bf16_dev(bits)
        xf = synth.bf16_bits_to_f32(bits)
    else:
        xin = torch.from_numpy(x).to(dev())
        xf = x
    q = ds4g.ds4g_quantize_mx(xin, fmt)
    ref = oracle.quantize(xf, fmt)
    got = from_dev(q)
    assert np.array_equal(got.scales, ref.scales)
    assert np.array_equal(got.data, ref.data)
    if fmt == NV:
        assert np.float32(got.g) == np.float32(ref.g)


def test_quantize_nv_given_g():
    x = _x_f32(16, 512, 8, 3.0)
    g = np.float32(0.0123)
    q = ds4g.ds4g_quantize_mx(torch.from_numpy(x).to(dev()), NV, g_in=torch.tensor([g], device=dev()))
    ref = oracle.quantize(x, NV, g=float(g))
    got = from_dev(q)
    assert np.array_equal(got.scales, ref.scales) and np.array_equal(got.data, ref.data)


def test_quantize_rejects_bad_k():
    x = torch.zeros((4, 96), dtype=torch.float32, device=dev())
    with pytest.raises(ds4g.Ds4gError) as ei:
        ds4g.ds4g_quantize_mx(x, MX, out=ds4g.Fp4Tensor.empty(4, 96, MX, dev()))
    assert ei.value.status == 2


# ---- routing -------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,bias", [(16, 8, 2, 0.0), (37, 256, 6, 1.5), (5, 256, 6, 0.0), (3, 1000, 32, 0.0),
                                        (4, 8, 8, 0.0)])
def test_route_topk(T, E, k, bias):
    lg = synth.logits(T, E, 0, bias)
    lg[0, 3] = lg[0, 5] = lg[0].max() + 1.0     # a tie at the top: lower index first
    idx, w = ds4g.ds4g_route_topk(torch.from_numpy(lg).to(dev()), k)
    ridx, rw = oracle.route_topk(lg, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.allclose(w.cpu().numpy(), rw, rtol=0, atol=2e-6)


def _non_finite_logits(T, E, seed):
    lg = synth.logits(T, E, seed, 1.5)
    lg[0, :] = -np.inf
    lg[1, 17] = np.inf
    lg[2, [3, E - 1]] = np.inf
    lg[3, :] = np.nan
    lg[3, E // 2] = 0.0
    lg[4, ::3] = np.nan
    lg[5, :] = np.nan
    lg[6, 1::2] = -np.inf
    return lg


@pytest.mark.parametrize("T,E,k", [(8, 256, 6), (100, 256, 6), (9, 64, 8)])
def test_route_topk_non_finite(T, E, k):
    """NaN ranks as -inf, infinities take the softmax's limit: picks stay
    distinct and in [0, E), identical to the oracle's"""
    lg = _non_finite_logits(T, E, 5)
    idx, w = ds4g.ds4g_route_topk(torch.from_numpy(lg).to(dev()), k)
    ridx, rw = oracle.route_topk(lg, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.allclose(w.cpu().numpy(), rw, rtol=0, atol=2e-6)


@pytest.mark.parametrize("T,k,E", [(8, 6, 256), (200, 6, 256)])
def test_dispatch_non_finite_logits(T, k, E):
    """the fused dispatch (one-CTA path at 48 slots, three kernels at 1200)
    routes non-finite logits like the oracle and permutes in bounds"""
    lg = _non_finite_logits(T, E, 6)
    bits = synth.normal_bf16_bits((T, 256), 0, 62, 1.0)
    idx, w, xq, offs, r2s, s2r, a = ds4g.ds4g_moe_dispatch(torch.from_numpy(lg).to(dev()), bf16_dev(bits), k, MX)
    ds4g.ds4g_check_device()
    ridx, rw = oracle.route_topk(lg, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.allclose(w.cpu().numpy(), rw, rtol=0, atol=2e-6)
    roffs, rr2s, rs2r = oracle.moe_permute(ridx, E)
    assert np.array_equal(offs.cpu().numpy(), roffs)
    assert np.array_equal(r2s.cpu().numpy(), rr2s) and np.array_equal(s2r.cpu().numpy(), rs2r)


# ---- permutation ---------------------------------------------------------------

@pytest.mark.parametrize("T,k,E,fmt", [(16, 2, 8, MX), (1000, 6, 256, MX), (333, 6, 256, NV), (1, 6, 256, MX),
                                       (8, 6, 256, NV), (85, 6, 256, MX), (86, 6, 256, MX), (2048, 6, 256, MX)])
def test_permute_bitexact(T, k, E, fmt):
    K = 256
    lg = synth.logits(T, E, 0, 1.5)
    ridx, _ = oracle.route_topk(lg, k)
    xq = oracle.quantize(_x_f32(T, K, 9), fmt)
    offs, r2s, s2r, a = ds4g.ds4g_moe_permute(torch.from_numpy(ridx).to(dev()), E, to_dev(xq))
    roffs, rr2s, rs2r = oracle.moe_permute(ridx, E)
    assert np.array_equal(offs.cpu().numpy(), roffs)
    assert np.array_equal(r2s.cpu().numpy(), rr2s)
    assert np.array_equal(s2r.cpu().numpy(), rs2r)
    ra = oracle.gather_rows(xq, rr2s, k)
    got = from_dev(a)
    assert np.array_equal(got.data, ra.data) and np.array_equal(got.scales, ra.scales)
    if fmt == NV:
        assert np.float32(got.g) == np.float32(xq.g)


def test_permute_empty():
    E = 8
    idx = torch.empty((0, 2), dtype=torch.int32, device=dev())
    xq = ds4g.Fp4Tensor.empty(0, 64, MX, dev())
    offs, _, _, _ = ds4g.ds4g_moe_permute(idx, E, xq)
    assert np.array_equal(offs.cpu().numpy(), np.zeros(E + 1, np.int32))


# ---- dispatch (route + quantise + permute in one call) --------------------------

@pytest.mark.parametrize("T,k,E,fmt,f32,g_given", [
    (1, 6, 256, MX, False, False), (8, 6, 256, NV, False, False), (85, 6, 256, MX, False, False),
    (86, 6, 256, MX, False, False), (16, 2, 8, NV, True, True), (300, 6, 256, NV, False, False),
    (37, 6, 1000, MX, True, False), (4, 8, 8, NV, False, True), (512, 1, 64, MX, False, False)])
def test_dispatch_bitexact(T, k, E, fmt, f32, g_given):
    """single-CTA path up to 512 slots (T*k), the three-kernel path above;
    every output bit-exact against the oracle's routing, quantisation and
    permutation of the same inputs"""
    K = 512
    lg = synth.logits(T, E, 3, 1.5)
    if f32:
        xr = _x_f32(T, K, 61, 2.0)
        xd = torch.from_numpy(xr).to(dev())
    else:
        bits = synth.normal_bf16_bits((T, K), 0, 61, 2.0)
        xd = bf16_dev(bits)
        xr = synth.bf16_bits_to_f32(bits)
    g = np.float32(0.0117) if g_given else None
    idx, w, xq, offs, r2s, s2r, a = ds4g.ds4g_moe_dispatch(
        torch.from_numpy(lg).to(dev()), xd, k, fmt, g_in=torch.tensor([g], device=dev()) if g_given else None)
    ds4g.ds4g_check_device()
    ridx, rw = oracle.route_topk(lg, k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.allclose(w.cpu().numpy(), rw, rtol=0, atol=2e-6)
    rq = oracle.quantize(xr, fmt, g=float(g) if g_given else None)
    gq = from_dev(xq)
    assert np.array_equal(gq.data, rq.data) and np.array_equal(gq.scales, rq.scales)
    if fmt == NV:
        assert np.float32(gq.g) == np.float32(rq.g)
    roffs, rr2s, rs2r = oracle.moe_permute(ridx, E)
    assert np.array_equal(offs.cpu().numpy(), roffs)
    assert np.array_equal(r2s.cpu().numpy(), rr2s) and np.array_equal(s2r.cpu().numpy(), rs2r)
    ra = oracle.gather_rows(rq, rr2s, k)
    ga = from_dev(a)
    assert np.array_equal(ga.data, ra.data) and np.array_equal(ga.scales, ra.scales)
    if fmt == NV:
        assert np.float32(ga.g) == np.float32(rq.g)


def test_dispatch_empty():
    E = 8
    lg = torch.empty((0, E), dtype=torch.float32, device=dev())
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=dev())
    _, _, _, offs, _, _, _ = ds4g.ds4g_moe_dispatch(lg, x, 2, MX)
    ds4g.ds4g_check_device()
    assert np.array_equal(offs.cpu().numpy(), np.zeros(E + 1, np.int32))


# ---- grouped GEMM ------------------------------------------------------------------

def _grouped_problem(seg, N, K, fmt, stream=11):
    E = len(seg)
    offsets = np.concatenate([[0], np.cumsum(seg)]).astype(np.int32)
    S = int(offsets[-1])
    a = oracle.quantize(_x_f32(max(S, 1), K, stream)[:S] if S else np.zeros((0, K), np.float32), fmt)
    wf = synth.normal_f32((E * N, K), 0, stream + 1, 0.02)
    if fmt == NV:
        ws = [oracle.quantize(wf[e * N:(e + 1) * N], NV) for e in range(E)]
        w = oracle.Fp4(np.concatenate([t.data for t in ws]), np.concatenate([t.scales for t in ws]), 1.0, NV)
        gw = [t.g for t in ws]
    else:
        w = oracle.quantize(wf, MX)
        gw = None
    return offsets, a, w, gw


def _ref_gemm(a, offsets, w, gw, N):
    """oracle result; NV weights carry one scale per expert"""
    if a.fmt == MX:
        return oracle.grouped_gemm(a, offsets, w, N)
    S = a.data.shape[0]
    out = np.full((S, N), np.nan)
    ab = np.full((S, N), np.nan)
    for e in range(len(offsets) - 1):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 == r0:
            continue
        we = oracle.Fp4(w.data[e * N:(e + 1) * N], w.scales[e * N:(e + 1) * N], gw[e], NV)
        o, s = oracle.expert_gemm_rows(a, np.arange(r0, r1), we, (0, N))
        out[r0:r1], ab[r0:r1] = o, s
    return out, ab


# decode-sized segments: the swapped tensor-core kernel where the tiling fits
# (K % 512 MX / % 256 NV), the dp4a kernel otherwise
GEMV_CASES = [([3, 0, 1, 8, 5], 512, 7168), ([1, 1, 1, 1, 1, 1], 256, 2048), ([2, 0, 0, 7], 256, 256),
              ([8], 4096, 256), ([1], 128, 128), ([16, 9, 0, 13], 256, 1024), ([1, 2], 384, 1024),
              ([1], 4096, 7168),                      # the dense configuration at M = 1 (one expert)
              ([3], 2048, 4096)]                      # one expert, few tiles: K split over 8 parts
# tensor-core kernel cases (MX needs K % 512, NV K % 256; others take the
# GEMV kernel with long segments, which is covered as well)
TC_CASES = [([300, 0, 1, 129, 77], 512, 512), ([256, 128], 256, 1024), ([9, 200, 0, 0, 1000], 256, 512),
            ([130], 512, 7168), ([17, 140], 256, 768), ([40, 12], 256, 384),
            # N a multiple of 224: 224-column tiles, two accumulators
            ([300, 0, 1, 129, 77], 448, 512), ([130, 20], 224, 2048), ([17, 600], 672, 1024),
            ([64], 4096, 7168),                       # the dense configuration at M = 64 (one expert)
            ([40], 2048, 4096)]                       # one expert, few tiles: K split over 8 parts


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("case", GEMV_CASES + TC_CASES)
def test_grouped_gemm_plain(fmt, case):
    seg, N, K = case
    offsets, a, w, gw = _grouped_problem(seg, N, K, fmt)
    max_rows = max(seg)
    out = ds4g.ds4g_grouped_gemm_fp4(to_dev(a), torch.from_numpy(offsets).to(dev()), len(seg), max_rows,
                                     to_dev(w, g_per_expert=gw), N)
    ds4g.ds4g_check_device()
    ref, ab = _ref_gemm(a, offsets, w, gw, N)
    assert_gemm_close(out.cpu().numpy(), ref, ab, f"{'gemv' if max_rows <= 8 else 'tcgen05'} {case}")


def _h_bound(y1_ref, ab1, I):
    g, u = y1_ref[:, :I], y1_ref[:, I:]
    dg = 1e-5 * ab1[:, :I] + 1e-6
    du = 1e-5 * ab1[:, I:] + 1e-6
    sig = 1.0 / (1.0 + np.exp(-g))
    dsilu = sig * (1 + g * (1 - sig))
    h = g * sig * u
    # the GEMM's bound on g and u carried through silu(g) u, plus the fp32
    # evaluation of h from the GPU's own g and u (swiglu_eval_bound)
    return h, np.abs(dsilu) * np.abs(u) * dg + np.abs(g * sig) * du + swiglu_eval_bound(g, h)


# decode-sized FC1 (<= 16 rows per expert) runs one CTA per item, or, with
# few items (min(E, rows) x I / 64 <= 296), each item's K range split over a
# CTA pair: ([3, 0, 1, 8, 5], 256, 7168) and ([5, 16, 2], 192, 1024) take the
# split, ([1] * 40, 512, 1024) and ([3, 16, 0, 5] * 20, 384, 1024) do not
@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("case", [([3, 0, 1, 8, 5], 256, 7168), ([300, 0, 1, 129, 77], 256, 512),
                                  ([2, 1], 64, 256), ([131], 128, 2048), ([20, 0, 150], 128, 768),
                                  ([200, 9], 384, 1024), ([100, 30], 96, 1024), ([5, 16, 2], 192, 1024),
                                  ([140, 60], 160, 512), ([700, 3, 260], 2048, 1024), ([1] * 40, 512, 1024),
                                  ([3, 16, 0, 5] * 20, 384, 1024)])
def test_fc1_fused_swiglu_requant(fmt, case):
    seg, I, K = case
    offsets, a, w, gw = _grouped_problem(seg, 2 * I, K, fmt, stream=21)
    S = int(offsets[-1])
    max_rows = max(seg)
    hq = ds4g.Fp4Tensor.empty(S, I, fmt, dev())
    g_h = G_H
    if fmt == NV:
        hq.g.fill_(g_h)
    hdbg = torch.empty((S, I), dtype=torch.float32, device=dev())
    ds4g.ds4g_grouped_gemm_fp4(to_dev(a), torch.from_numpy(offsets).to(dev()), len(seg), max_rows,
                               to_dev(w, g_per_expert=gw), 2 * I, ds4g.EPI_SWIGLU_REQUANT, out_q=hq, h_debug=hdbg)
    ds4g.ds4g_check_device()
    y1, ab1 = _ref_gemm(a, offsets, w, gw, 2 * I)
    h_ref, dh = _h_bound(y1, ab1, I)
    h_gpu = hdbg.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(h_gpu - h_ref) <= dh * 1.000001), "h outside its error bound"
    check_requant(from_dev(hq), h_ref, dh, fmt, g=g_h)


@pytest.mark.parametrize("fmt", [MX, NV])
def test_swiglu_requant(fmt):
    rows, I = 70, 256
    y1 = synth.normal_f32((rows, 2 * I), 0, 31, 2.0)
    g_h = G_H
    hdbg = torch.empty((rows, I), dtype=torch.float32, device=dev())
    hq = ds4g.ds4g_swiglu_requant(torch.from_numpy(y1).to(dev()), fmt, h_debug=hdbg,
                                  g_h=torch.tensor([g_h], device=dev()) if fmt == NV else None)
    h_ref = oracle.swiglu(y1).astype(np.float64)
    h_gpu = hdbg.cpu().numpy().astype(np.float64)
    dh = swiglu_eval_bound(y1[:, :I], h_ref)
    assert np.all(np.abs(h_gpu - h_ref) <= dh)
    check_requant(from_dev(hq), h_ref, dh, fmt, g=g_h, min_exact=0.9999)


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("max_rows", [0, 300])
def test_grouped_gemm_no_rows(fmt, max_rows):
    """no routed rows at all (every expert segment empty): each epilogue
    returns without work, whichever kernel the row bound selects"""
    E, N, K = 4, 448, 512
    offsets = torch.zeros(E + 1, dtype=torch.int32, device=dev())
    a = ds4g.Fp4Tensor.empty(0, K, fmt, dev())
    w = ds4g.Fp4Tensor.empty(E * N, K, fmt, dev())
    if fmt == NV:
        w.g = torch.ones(E, dtype=torch.float32, device=dev())
    out = ds4g.ds4g_grouped_gemm_fp4(a, offsets, E, max_rows, w, N)
    assert out.shape == (0, N)
    hq = ds4g.Fp4Tensor.empty(0, N // 2, fmt, dev())
    ds4g.ds4g_grouped_gemm_fp4(a, offsets, E, max_rows, w, N, ds4g.EPI_SWIGLU_REQUANT, out_q=hq)
    r2s = torch.empty(0, dtype=torch.int32, device=dev())
    rw = torch.empty((0, 6), dtype=torch.float32, device=dev())
    out2 = ds4g.ds4g_grouped_gemm_fp4_combine(a, offsets, E, max_rows, w, N, r2s, rw)
    assert out2.shape == (0, N)
    ds4g.ds4g_check_device()


# ---- FC2 with the combine fused --------------------------------------------------------

@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("T,k,E,N,K", [(300, 6, 16, 512, 1024),    # tensor-core kernel
                                       (300, 6, 16, 448, 1024),    # tensor-core kernel, 224-column tiles
                                       (4096, 2, 8, 7168, 512),    # output of 117 MB: two column bands
                                       (3, 6, 64, 256, 1024),      # decode tensor-core kernel
                                       (4, 2, 8, 128, 256)])       # dp4a kernel (MX) / decode tc (NV)
def test_fc2_combine_fused(fmt, T, k, E, N, K):
    lg = synth.logits(T, E, 0, 1.5)
    idx, w = oracle.route_topk(lg, k)
    offsets, r2s, s2r = oracle.moe_permute(idx, E)
    S = T * k
    a = oracle.quantize(_x_f32(S, K, 51), fmt)
    wf = synth.normal_f32((E * N, K), 0, 52, 0.02)
    if fmt == NV:
        ws = [oracle.quantize(wf[e * N:(e + 1) * N], NV) for e in range(E)]
        W = oracle.Fp4(np.concatenate([t.data for t in ws]), np.concatenate([t.scales for t in ws]), 1.0, NV)
        gw = [t.g for t in ws]
    else:
        W, gw = oracle.quantize(wf, MX), None
    w32 = w.astype(np.float32)
    out = ds4g.ds4g_grouped_gemm_fp4_combine(to_dev(a), torch.from_numpy(offsets).to(dev()), E, T,
                                             to_dev(W, g_per_expert=gw), N, torch.from_numpy(r2s).to(dev()),
                                             torch.from_numpy(w32).to(dev()))
    ds4g.ds4g_check_device()
    y2, ab = _ref_gemm(a, offsets, W, gw, N)
    ref = oracle.moe_combine(y2, s2r, w32.astype(np.float64))
    bound = (oracle.moe_combine(1e-5 * ab + 1e-6, s2r, np.abs(w32.astype(np.float64))) +
             1e-6 * oracle.moe_combine(np.abs(y2), s2r, np.abs(w32.astype(np.float64))) + 1e-7)
    got = out.cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound), f"worst excess {(np.abs(got - ref) - bound).max():.3e}"


@pytest.mark.parametrize("fmt", [MX, NV])
@pytest.mark.parametrize("T,k,E,d,I", [(1, 6, 32, 2048, 1024),     # decode kernel, FC1 split over CTA pairs
                                       (3, 6, 64, 1024, 512),      # decode kernel
                                       (300, 6, 16, 512, 512),     # tensor-core kernel (no overlap)
                                       (4, 2, 8, 256, 128)])       # dp4a kernel (MX)
def test_fc2_combine_chained(fmt, T, k, E, d, I):
    """FC1 writes h, then the chained FC2 + combine, launched right after it
    on the same stream, adds into out: out = (what it held) + the oracle's
    FC2 + combine of the h codes FC1 produced"""
    lg = synth.logits(T, E, 7, 1.5)
    idx, rw = oracle.route_topk(lg, k)
    offsets, r2s, s2r = oracle.moe_permute(idx, E)
    S = T * k
    touched = [e for e in range(E) if offsets[e + 1] > offsets[e]]
    W = []
    for n_rows, K, stream in ((2 * I, d, 82), (d, I, 83)):
        blk = oracle.BLOCK[fmt]
        data = np.zeros((E * n_rows, K // 2), np.uint8)
        scales = np.zeros((E * n_rows, K // blk), np.uint8)
        gw = [1.0] * E
        for e in touched:          # weights of the touched experts only (no row reads the others)
            q = oracle.quantize(synth.normal_f32((n_rows, K), e, stream, 0.02), fmt)
            data[e * n_rows:(e + 1) * n_rows], scales[e * n_rows:(e + 1) * n_rows] = q.data, q.scales
            gw[e] = q.g if fmt == NV else 1.0
        W.append((oracle.Fp4(data, scales, 1.0, fmt), gw if fmt == NV else None))
    (W1, g1), (W2, g2) = W
    a = oracle.quantize(_x_f32(S, d, 81), fmt)
    offs_d, r2s_d = torch.from_numpy(offsets).to(dev()), torch.from_numpy(r2s).to(dev())
    rw32 = rw.astype(np.float32)
    hq = ds4g.Fp4Tensor.empty(S, I, fmt, dev())
    if fmt == NV:
        hq.g.fill_(G_H)
    base = synth.normal_f32((T, d), 0, 84, 1.0)
    out = torch.from_numpy(base).to(dev())
    torch.cuda.synchronize()
    ds4g.ds4g_grouped_gemm_fp4(to_dev(a), offs_d, E, T, to_dev(W1, g_per_expert=g1), 2 * I, ds4g.EPI_SWIGLU_REQUANT,
                               out_q=hq)
    ds4g.ds4g_grouped_gemm_fp4_combine_chained(hq, offs_d, E, T, to_dev(W2, g_per_expert=g2), d, r2s_d,
                                               torch.from_numpy(rw32).to(dev()), out)
    ds4g.ds4g_check_device()
    hq_host = from_dev(hq)
    y1, ab1 = _ref_gemm(a, offsets, W1, g1, 2 * I)
    h_ref, dh = _h_bound(y1, ab1, I)
    check_requant(hq_host, h_ref, dh, fmt, g=G_H)
    y2, ab2 = _ref_gemm(hq_host, offsets, W2, g2, d)
    w64 = rw32.astype(np.float64)
    ref = base.astype(np.float64) + oracle.moe_combine(y2, s2r, w64)
    bound = (oracle.moe_combine(1e-5 * ab2 + 1e-6, s2r, np.abs(w64)) +
             1e-6 * (oracle.moe_combine(np.abs(y2), s2r, np.abs(w64)) + np.abs(base)) + 1e-7)
    got = out.cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound), f"worst excess {(np.abs(got - ref) - bound).max():.3e}"


def _decode_weights(E, touched, n_rows, K, fmt, stream):
    """an expert weight tensor whose touched experts hold random weights (the
    others zero: no row reads them)"""
    blk = oracle.BLOCK[fmt]
    data = np.zeros((E * n_rows, K // 2), np.uint8)
    scales = np.zeros((E * n_rows, K // blk), np.uint8)
    gw = [1.0] * E
    for e in touched:
        q = oracle.quantize(synth.normal_f32((n_rows, K), e, stream, 0.02), fmt)
        data[e * n_rows:(e + 1) * n_rows], scales[e * n_rows:(e + 1) * n_rows] = q.data, q.scales
        gw[e] = q.g if fmt == NV else 1.0
    return oracle.Fp4(data, scales, 1.0, fmt), (gw if fmt == NV else None)


# the one-launch decode FFN (one CTA per SM): few items (fewer FC1 items
# than SMs) and many, and (NV) K stage counts that are odd in both GEMMs
FFN_CASES = {MX: [(1, 6, 32, 2048, 1024), (3, 6, 64, 1024, 512), (8, 6, 64, 1024, 1024), (4, 2, 8, 512, 512)],
             NV: [(1, 6, 32, 2048, 1024), (3, 6, 64, 1024, 512), (8, 6, 64, 1024, 1024), (4, 2, 8, 768, 256)]}


@pytest.mark.parametrize("fmt,T,k,E,d,I", [(f,) + c for f in (MX, NV) for c in FFN_CASES[f]])
def test_moe_ffn_one_launch(fmt, T, k, E, d, I):
    """ds4g_moe_ffn_fp4 twice in a row on the same buffers and counters, with
    new activations and routing the second time: each call's h codes are a
    valid rounding of the oracle's h, and out = (what it held) + the oracle's
    FC2 + combine of those h codes; the counters are zero after each call"""
    routes = []
    for call in range(2):
        lg = synth.logits(T, E, 7 + call, 1.5)
        idx, rw = oracle.route_topk(lg, k)
        routes.append((rw, oracle.moe_permute(idx, E)))
    touched = sorted({e for _, (offsets, _, _) in routes for e in range(E) if offsets[e + 1] > offsets[e]})
    W1, g1 = _decode_weights(E, touched, 2 * I, d, fmt, 92)
    W2, g2 = _decode_weights(E, touched, d, I, fmt, 93)
    w1_d, w2_d = to_dev(W1, g_per_expert=g1), to_dev(W2, g_per_expert=g2)
    S = T * k
    hq = ds4g.Fp4Tensor.empty(S, I, fmt, dev())
    if fmt == NV:
        hq.g.fill_(G_H)
    ctr = ds4g.ffn_counters(E, dev())
    out = torch.empty((T, d), dtype=torch.float32, device=dev())
    for call, (rw, (offsets, r2s, s2r)) in enumerate(routes):
        a = oracle.quantize(_x_f32(S, d, 91 + call), fmt)
        base = synth.normal_f32((T, d), call, 94, 1.0)
        out.copy_(torch.from_numpy(base))
        rw32 = rw.astype(np.float32)
        ds4g.ds4g_moe_ffn_fp4(to_dev(a), torch.from_numpy(offsets).to(dev()), E, T, w1_d, w2_d, d, I, hq,
                              torch.from_numpy(r2s).to(dev()), torch.from_numpy(rw32).to(dev()), out, ctr)
        ds4g.ds4g_check_device()
        assert not ctr.any(), f"call {call}: counters left {ctr.cpu().numpy()}"
        hq_host = from_dev(hq)
        y1, ab1 = _ref_gemm(a, offsets, W1, g1, 2 * I)
        h_ref, dh = _h_bound(y1, ab1, I)
        check_requant(hq_host, h_ref, dh, fmt, g=G_H)
        y2, ab2 = _ref_gemm(hq_host, offsets, W2, g2, d)
        w64 = rw32.astype(np.float64)
        ref = base.astype(np.float64) + oracle.moe_combine(y2, s2r, w64)
        bound = (oracle.moe_combine(1e-5 * ab2 + 1e-6, s2r, np.abs(w64)) +
                 1e-6 * (oracle.moe_combine(np.abs(y2), s2r, np.abs(w64)) + np.abs(base)) + 1e-7)
        got = out.cpu().numpy()
        assert np.all(np.abs(got - ref) <= bound), f"call {call}: worst excess {(np.abs(got - ref) - bound).max():.3e}"


def test_moe_ffn_wait_gives_up_cleanly():
    """A device-side bounded wait that runs out, made on purpose without any
    fault: the per-expert counters start far below zero, so no FC2 item's
    wait for its expert's FC1 items can succeed.  Every CTA gives up after
    its bound, the call reports DS4G_ERR_DEVICE through ds4g_check_device,
    the last CTA leaves the counters at zero, and the next call on the same
    context and buffers is correct."""
    fmt, T, k, E, d, I = MX, 4, 2, 8, 512, 512
    lg = synth.logits(T, E, 3, 1.5)
    idx, rw = oracle.route_topk(lg, k)
    offsets, r2s, s2r = oracle.moe_permute(idx, E)
    touched = [e for e in range(E) if offsets[e + 1] > offsets[e]]
    W1, g1 = _decode_weights(E, touched, 2 * I, d, fmt, 95)
    W2, g2 = _decode_weights(E, touched, d, I, fmt, 96)
    S = T * k
    a = oracle.quantize(_x_f32(S, d, 97), fmt)
    args = (to_dev(a), torch.from_numpy(offsets).to(dev()), E, T, to_dev(W1, g_per_expert=g1),
            to_dev(W2, g_per_expert=g2), d, I)
    hq = ds4g.Fp4Tensor.empty(S, I, fmt, dev())
    r2s_d, rw_d = torch.from_numpy(r2s).to(dev()), torch.from_numpy(rw.astype(np.float32)).to(dev())
    out = torch.zeros((T, d), dtype=torch.float32, device=dev())
    ctr = ds4g.ffn_counters(E, dev())
    ctr[:E] = -(1 << 20)                               # a completion count no FC1 item can bring to its target
    ds4g.ds4g_moe_ffn_fp4(*args, hq, r2s_d, rw_d, out, ctr)
    torch.cuda.synchronize()
    with pytest.raises(ds4g.Ds4gError) as ei:
        ds4g.ds4g_check_device()
    assert ei.value.status == 5                        # DS4G_ERR_DEVICE
    assert not ctr.any(), "the counters are left at zero after a wait gave up"
    ds4g.ds4g_check_device()                           # the error word was read and cleared
    out.zero_()
    ds4g.ds4g_moe_ffn_fp4(*args, hq, r2s_d, rw_d, out, ctr)
    ds4g.ds4g_check_device()
    y1, ab1 = _ref_gemm(a, offsets, W1, g1, 2 * I)
    h_ref, dh = _h_bound(y1, ab1, I)
    hq_host = from_dev(hq)
    check_requant(hq_host, h_ref, dh, fmt)
    y2, ab2 = _ref_gemm(hq_host, offsets, W2, g2, d)
    w64 = rw.astype(np.float32).astype(np.float64)
    ref = oracle.moe_combine(y2, s2r, w64)
    bound = (oracle.moe_combine(1e-5 * ab2 + 1e-6, s2r, np.abs(w64)) +
             1e-6 * oracle.moe_combine(np.abs(y2), s2r, np.abs(w64)) + 1e-7)
    assert np.all(np.abs(out.cpu().numpy() - ref) <= bound)


# ---- combine -----------------------------------------------------------------------

def test_combine():
    T, k, d, E = 33, 6, 7168, 256
    lg = synth.logits(T, E, 0)
    ridx, rw = oracle.route_topk(lg, k)
    _, _, s2r = oracle.moe_permute(ridx, E)
    y2 = synth.normal_f32((T * k, d), 0, 41, 3.0)
    w32 = rw.astype(np.float32)
    out = ds4g.ds4g_moe_combine(torch.from_numpy(y2).to(dev()), torch.from_numpy(s2r).to(dev()),
                                torch.from_numpy(w32).to(dev()))
    ref = oracle.moe_combine(y2.astype(np.float64), s2r, w32.astype(np.float64))
    absref = oracle.moe_combine(np.abs(y2.astype(np.float64)), s2r, np.abs(w32.astype(np.float64)))
    assert np.all(np.abs(out.cpu().numpy() - ref) <= 1e-6 * absref + 1e-7)


# ---- full layer --------------------------------------------------------------------

@pytest.mark.parametrize("fused,fused_combine,fused_dispatch", [(True, True, True), (False, False, False),
                                                               (True, False, True)])
def test_layer_tiny(fused, fused_combine, fused_dispatch):
    from synth import workloads
    from block_scaled_fp4_topk_b200.layer import MoeLayer
    from bench import synthetic_weights
    wl = workloads.WORKLOADS["tiny"]
    w1, w2 = synthetic_weights(wl.E, wl.d, wl.I, wl.fmt, device=dev())
    layer = MoeLayer(w1, w2, wl.E, wl.k, wl.d, wl.I, wl.fmt, fused=fused, fused_combine=fused_combine,
                     fused_dispatch=fused_dispatch)
    xb = workloads.host_x_bits(wl)
    lg = workloads.host_logits(wl)
    out = layer.forward(bf16_dev(xb), torch.from_numpy(lg).to(dev())).cpu().numpy()
    ds4g.ds4g_check_device()
    W1 = oracle.quantize(np.concatenate([workloads.host_w1(wl, e) for e in range(wl.E)]), MX)
    W2 = oracle.quantize(np.concatenate([workloads.host_w2(wl, e) for e in range(wl.E)]), MX)
    assert np.array_equal(from_dev(w1).data, W1.data) and np.array_equal(from_dev(w2).scales, W2.scales)
    res = oracle.moe_layer(synth.bf16_bits_to_f32(xb), lg, W1, W2, wl.k, MX)
    rel = np.linalg.norm(out - res["out"]) / np.linalg.norm(res["out"])
    assert rel <= 1e-2, rel
