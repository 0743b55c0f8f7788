"""Parity at the full problem sizes, in the configuration the bench times
(E = 256, top-6, d = 7168, I = 2048; MXFP4 decode T = 1 / 8, MXFP4 prefill
T = 2048 with the skewed router bias, NVFP4 prefill T = 16384), through the
library's C ABI with the same layer code the bench uses.

What is checked against the oracle, which runs its own chain from the same
seeded inputs:
  - routing indices (bit-exact) and weights, all tokens;
  - quantised activations, offsets, permutation and gathered rows (bit-exact);
  - FC1 + SwiGLU on sampled experts (the heaviest, a one-row expert, random
    ones): h within its propagated error bound, its FP4 codes valid;
  - FC2 on sampled rows whose FP4 input matches the oracle's byte for byte
    (rows where a code legitimately rounded the other way were validated in
    the FC1 check): per-element GEMM bound;
  - combine on sampled tokens; and for decode T = 1 the whole layer."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_helpers import assert_gemm_close, bf16_dev, check_requant, dev, from_dev
from synth import workloads

pytestmark = pytest.mark.gpu

ds4g = pytest.importorskip("block_scaled_fp4_topk_b200.ds4g")
from block_scaled_fp4_topk_b200.layer import MoeLayer  # noqa: E402

MX, NV = oracle.MX, oracle.NV
_LAYERS = {}


def _layer(fmt):
    if fmt not in _LAYERS:
        for k in list(_LAYERS):
            del _LAYERS[k]
        torch.cuda.empty_cache()
        wl = workloads.WORKLOADS["prefill" if fmt == MX else "prefill16k"]
        w1, w2 = MoeLayer.synthetic_weights(wl.E, wl.d, wl.I, fmt, device=dev())
        _LAYERS[fmt] = MoeLayer(w1, w2, wl.E, wl.k, wl.d, wl.I, fmt, g_h=workloads.G_H)
    return _LAYERS[fmt]


_WCACHE = {}


def _expert_weights(wl, e):
    key = (wl.fmt, e)
    if key not in _WCACHE:
        if len(_WCACHE) > 24:
            _WCACHE.clear()
        _WCACHE[key] = (oracle.quantize(workloads.host_w1(wl, e), wl.fmt),
                        oracle.quantize(workloads.host_w2(wl, e), wl.fmt))
    return _WCACHE[key]


def _h_bound(g, u, ag, au):
    dg, du = 1e-5 * ag + 1e-6, 1e-5 * au + 1e-6
    sig = 1.0 / (1.0 + np.exp(-g))
    h = g * sig * u
    fast = (4e-6 + 2.0 ** -23 * np.abs(g)) * np.abs(h)
    return h, np.abs(sig * (1 + g * (1 - sig))) * np.abs(u) * dg + np.abs(g * sig) * du + fast + 1e-30


def _run(name, rng_seed=0):
    wl = workloads.WORKLOADS[name]
    layer = _layer(wl.fmt)
    xb = workloads.host_x_bits(wl)
    lg = workloads.host_logits(wl)
    hdbg = torch.empty((wl.S, wl.I), dtype=torch.float32, device=dev())
    out = layer.forward(bf16_dev(xb), torch.from_numpy(lg).to(dev()), h_debug=hdbg)   # as the bench runs it
    ds4g.ds4g_check_device()
    b = dict(layer.buffers(wl.T, dev()))
    # FC2 rows as well (the layer fuses FC2 with the combine): the plain epilogue
    b["y2"] = ds4g.ds4g_grouped_gemm_fp4(b["hq"], b["offsets"], wl.E, wl.T, layer.w2, wl.d, ds4g.EPI_NONE)
    return wl, layer, xb, lg, b, hdbg, out


@pytest.mark.parametrize("name", ["decode_t1", "decode_t8", "prefill", "prefill16k"])
def test_fullsize_layer(name):
    wl, layer, xb, lg, b, hdbg, out = _run(name)
    rng = np.random.default_rng(123)
    x = synth.bf16_bits_to_f32(xb)

    # routing, quantisation, permutation: whole tensors, bit-exact
    idx, w = oracle.route_topk(lg, wl.k)
    assert np.array_equal(b["idx"].cpu().numpy(), idx)
    assert np.allclose(b["w"].cpu().numpy(), w, rtol=0, atol=2e-6)
    xq = oracle.quantize(x, wl.fmt)
    gxq = from_dev(b["xq"])
    assert np.array_equal(gxq.scales, xq.scales) and np.array_equal(gxq.data, xq.data)
    if wl.fmt == NV:
        assert np.float32(gxq.g) == np.float32(xq.g)
    offsets, r2s, s2r = oracle.moe_permute(idx, wl.E)
    assert np.array_equal(b["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(b["r2s"][:wl.S].cpu().numpy(), r2s)
    assert np.array_equal(b["s2r"][:wl.S].cpu().numpy(), s2r)
    a = oracle.gather_rows(xq, r2s, wl.k)
    ga = from_dev(b["a"])
    assert np.array_equal(ga.data, a.data) and np.array_equal(ga.scales, a.scales)

    # sampled experts: heaviest, a one-row one (if any), two random touched ones
    counts = np.diff(offsets)
    touched = np.nonzero(counts)[0]
    picks = {int(touched[np.argmax(counts[touched])])}
    ones = touched[counts[touched] == 1]
    if len(ones):
        picks.add(int(ones[0]))
    picks.update(int(e) for e in rng.choice(touched, size=min(2, len(touched)), replace=False))
    g_h = workloads.G_H if wl.fmt == NV else None
    hq_gpu = from_dev(b["hq"])
    y2_rows, y2_ref_rows, y2_ab = [], [], []
    for e in sorted(picks):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        rows = np.arange(r0, r1)
        if len(rows) > 6:
            rows = np.sort(np.concatenate([[r0, r1 - 1], rng.choice(np.arange(r0 + 1, r1 - 1), 4, replace=False)]))
        W1, W2 = _expert_weights(wl, e)
        cb = np.sort(rng.choice(wl.I // 32, size=4, replace=False))          # 32-column blocks of h
        cols = np.concatenate([np.arange(32 * c, 32 * c + 32) for c in cb])
        # FC1 on the sampled gate and up columns, in fp64
        gate, ag = oracle.expert_gemm_rows(a, rows, W1, (0, wl.I))
        up, au = oracle.expert_gemm_rows(a, rows, W1, (wl.I, 2 * wl.I))
        gate, up, ag, au = gate[:, cols], up[:, cols], ag[:, cols], au[:, cols]
        h_ref_full = oracle.swiglu(np.concatenate([gate, up], axis=1).astype(np.float32))   # oracle's fp32 h
        h_ref, dh = _h_bound(gate.astype(np.float32).astype(np.float64), up.astype(np.float32).astype(np.float64),
                             ag, au)
        h_gpu = hdbg[torch.from_numpy(rows).to(dev())].cpu().numpy()[:, cols].astype(np.float64)
        assert np.all(np.abs(h_gpu - h_ref) <= dh * 1.000001), f"expert {e}: h outside its bound"
        # codes of the sampled blocks
        blk = oracle.BLOCK[wl.fmt]
        sub = oracle.Fp4(hq_gpu.data[rows][:, np.concatenate([np.arange(16 * c, 16 * c + 16) for c in cb])],
                         hq_gpu.scales[rows][:, np.concatenate([np.arange(c * 32 // blk, (c + 1) * 32 // blk)
                                                                for c in cb])], hq_gpu.g, wl.fmt)
        check_requant(sub, h_ref_full.astype(np.float64), dh, wl.fmt, g=workloads.G_H, min_exact=0.98)

        # FC2 on rows whose FP4 input equals the oracle's byte for byte
        y1_rows, _ = oracle.expert_gemm_rows(a, rows, W1, (0, 2 * wl.I))
        h_full = oracle.swiglu(y1_rows.astype(np.float32))
        hq_ref = oracle.quantize(h_full, wl.fmt, g=g_h)
        same = np.all(hq_gpu.data[rows] == hq_ref.data, axis=1) & np.all(hq_gpu.scales[rows] == hq_ref.scales, axis=1)
        assert same.mean() >= 0.5, f"expert {e}: too few rows with identical FP4 h"
        n_cols = np.sort(rng.choice(wl.d, size=256, replace=False))
        hq_rows = oracle.Fp4(hq_ref.data, hq_ref.scales, hq_ref.g, wl.fmt)
        y2_ref, y2_abs = oracle.expert_gemm_rows(hq_rows, np.arange(len(rows)), W2, (0, wl.d))
        y2_gpu = b["y2"][torch.from_numpy(rows).to(dev())].cpu().numpy()
        for i in np.nonzero(same)[0]:
            assert_gemm_close(y2_gpu[i, n_cols], y2_ref[i, n_cols], y2_abs[i, n_cols], f"FC2 expert {e} row {rows[i]}")

    # combine on sampled tokens, from the oracle's own FC2 rows
    toks = rng.choice(wl.T, size=min(2, wl.T), replace=False)
    out_gpu = out.cpu().numpy() if wl.T <= 64 else out[torch.from_numpy(toks).to(dev())].cpu().numpy()
    for ti, t in enumerate(toks):
        acc = np.zeros(wl.d)
        bound = np.full(wl.d, 1e-7)
        exact_inputs = True
        for j in range(wl.k):
            r = int(s2r[t * wl.k + j])
            e = int(idx[t, j])
            W1, W2 = _expert_weights(wl, e)
            hrow = oracle.swiglu(oracle.expert_gemm_rows(a, np.array([r]), W1, (0, 2 * wl.I))[0].astype(np.float32))
            hq_ref = oracle.quantize(hrow, wl.fmt, g=g_h)
            exact_inputs &= bool(np.array_equal(hq_gpu.data[r], hq_ref.data[0]) and
                                 np.array_equal(hq_gpu.scales[r], hq_ref.scales[0]))
            y, yab = oracle.expert_gemm_rows(hq_ref, np.array([0]), W2, (0, wl.d))
            acc += w[t, j] * y[0].astype(np.float32)
            # FC2 bound of the row, carried by the routing weight, plus the
            # fp32 rounding of the weighted sum
            bound += abs(w[t, j]) * (1e-5 * yab[0] + 1e-6) + 1e-6 * abs(w[t, j] * y[0])
        got = out_gpu[t] if wl.T <= 64 else out_gpu[ti]
        if exact_inputs:
            assert np.all(np.abs(got - acc) <= bound), f"combine token {t}"


def test_fullsize_decode_t1_layer_l2():
    """the whole decode layer (one token, six experts) against the oracle's
    independent chain: relative L2 <= 1e-2"""
    wl, layer, xb, lg, b, hdbg, out = _run("decode_t1")
    x = synth.bf16_bits_to_f32(xb)
    idx, w = oracle.route_topk(lg, wl.k)
    xq = oracle.quantize(x, wl.fmt)
    ref = np.zeros(wl.d)
    for j in range(wl.k):
        W1, W2 = _expert_weights(wl, int(idx[0, j]))
        y1, _ = oracle.expert_gemm_rows(xq, np.array([0]), W1, (0, 2 * wl.I))
        hq = oracle.quantize(oracle.swiglu(y1.astype(np.float32)), wl.fmt)
        y2, _ = oracle.expert_gemm_rows(hq, np.array([0]), W2, (0, wl.d))
        ref += w[0, j] * y2[0].astype(np.float32)
    got = out.cpu().numpy()[0]
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= 1e-2, rel
