"""Parity at the full problem sizes, in the configuration the bench times
(E = 256, top-6, d = 7168, I = 2048; MXFP4 decode T = 1 / 4 / 8, MXFP4
prefill T = 2048 with the skewed router bias, NVFP4 prefill T = 16384),
through the library's C ABI with the same layer code the bench uses.

What is checked against the oracle, which runs its own chain from the same
seeded inputs:
  - routing indices (bit-exact) and weights, all tokens;
  - quantised activations, offsets, permutation and gathered rows (bit-exact);
  - FC1 + SwiGLU on sampled experts (the heaviest, a one-row expert, random
    ones): h within its propagated error bound, its FP4 codes valid;
  - FC2 on sampled rows whose FP4 input matches the oracle's byte for byte
    (rows where a code legitimately rounded the other way were validated in
    the FC1 check): per-element GEMM bound;
  - FC2 + combine on sampled tokens (all tokens at decode sizes; 32 at
    prefill sizes, among them tokens of the heaviest and of a one-row
    expert), from the GPU's own upstream tensors (its h codes and routing
    weights): per-element bound;
  - the whole layer on the same token sample against the oracle's own chain
    (routing, quantisation, FC1, SwiGLU, requantisation, FC2, combine):
    relative L2 <= 1e-2.
And the captured decode layer (split FC1 at T = 1, plain at T = 4; as two
calls, and at T = 1 / 4 / 8 with FC1 -> FC2 + combine as one launch)
replayed back to back with different inputs and routing on every replay,
each replay against the oracle's chain (offsets bit-exact, output relative
L2 <= 1e-2): routing-dependent ordering errors between the layer's kernels
only show when the routing changes between steps."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_helpers import assert_gemm_close, bf16_dev, check_requant, dev, from_dev, swiglu_eval_bound
from synth import workloads

pytestmark = pytest.mark.gpu

ds4g = pytest.importorskip("block_scaled_fp4_topk_b200.ds4g")
from block_scaled_fp4_topk_b200.layer import MoeLayer  # noqa: E402
from bench import synthetic_weights  # noqa: E402

MX, NV = oracle.MX, oracle.NV
_LAYERS = {}
L2_MAX = 1e-2


def _layer(fmt):
    if fmt not in _LAYERS:
        for k in list(_LAYERS):
            del _LAYERS[k]
        torch.cuda.empty_cache()
        wl = workloads.WORKLOADS["prefill" if fmt == MX else "prefill16k"]
        w1, w2 = synthetic_weights(wl.E, wl.d, wl.I, fmt, device=dev())
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
    # the GEMM's bound on g and u carried through silu(g) u, plus the fp32
    # evaluation of h from the GPU's own g and u (swiglu_eval_bound)
    return h, np.abs(sig * (1 + g * (1 - sig))) * np.abs(u) * dg + np.abs(g * sig) * du + swiglu_eval_bound(g, h)


def _chain(wl, xq, idx, w, toks, gpu=None):
    """For the tokens `toks`, the layer output by the oracle's own chain from
    the quantised activations xq and the routing (idx, w): FC1 of each token's
    k rows, SwiGLU on the fp32-rounded result, requantisation, FC2, and the
    weighted sum in fp64.  With gpu = (hq, s2r, w_gpu) (the GPU's h codes, its
    slot -> row map and its routing weights) also FC2 + combine from those
    upstream tensors and the per-element bound of that result.  Each expert's
    weights are quantised once, for all sample rows routed to it."""
    g_h = workloads.G_H if wl.fmt == NV else None
    n = len(toks)
    ref = np.zeros((n, wl.d))
    up = np.zeros((n, wl.d))
    bound = np.full((n, wl.d), 1e-7)
    sel = idx[toks]                                   # [n][k] experts
    for e in np.unique(sel):
        ii, jj = np.nonzero(sel == e)                 # sample token i, slot j
        W1, W2 = _expert_weights(wl, int(e))
        y1, _ = oracle.expert_gemm_rows(xq, toks[ii], W1, (0, 2 * wl.I))
        hq = oracle.quantize(oracle.swiglu(y1.astype(np.float32)), wl.fmt, g=g_h)
        y2, _ = oracle.expert_gemm_rows(hq, np.arange(len(ii)), W2, (0, wl.d))
        ref[ii] += w[toks[ii], jj][:, None] * y2.astype(np.float32)
        if gpu is not None:
            ghq, s2r, wg = gpu
            rows = s2r[toks[ii] * wl.k + jj]
            y2u, ab = oracle.expert_gemm_rows(ghq, rows, W2, (0, wl.d))
            wt = wg[toks[ii], jj].astype(np.float64)[:, None]
            up[ii] += wt * y2u
            # FC2 bound of each row carried by its routing weight, plus the
            # fp32 rounding of the weighted terms and of their sum
            bound[ii] += np.abs(wt) * (1e-5 * ab + 1e-6) + 1e-6 * np.abs(wt * y2u)
    return ref, up, bound


def _rel_l2(got, ref):
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def _run(name):
    wl = workloads.WORKLOADS[name]
    layer = _layer(wl.fmt)
    xb = workloads.host_x_bits(wl)
    lg = workloads.host_logits(wl)
    hdbg = torch.empty((wl.S, wl.I), dtype=torch.float32, device=dev())
    # the two-call FFN (h_debug asks for FC1's h; the bench's decode steps run
    # the one-launch FFN, checked in test_decode_one_launch_ffn_replays)
    out = layer.forward(bf16_dev(xb), torch.from_numpy(lg).to(dev()), h_debug=hdbg)
    ds4g.ds4g_check_device()
    b = dict(layer.buffers(wl.T, dev()))
    # FC2 rows as well (the layer fuses FC2 with the combine): the plain epilogue
    b["y2"] = ds4g.ds4g_grouped_gemm_fp4(b["hq"], b["offsets"], wl.E, wl.T, layer.w2, wl.d, ds4g.EPI_NONE)
    return wl, layer, xb, lg, b, hdbg, out


def _token_sample(wl, idx, offsets, r2s, rng, n=32):
    """all tokens up to n; else tokens of the heaviest expert, of a one-row
    expert (if any) and random ones, n in all"""
    if wl.T <= n:
        return np.arange(wl.T)
    counts = np.diff(offsets)
    heavy = int(np.argmax(counts))
    picks = set(int(s) // wl.k for s in r2s[offsets[heavy]:offsets[heavy] + 2])
    ones = np.nonzero(counts == 1)[0]
    for e in ones[:2]:
        picks.add(int(r2s[offsets[e]]) // wl.k)
    rest = np.setdiff1d(np.arange(wl.T), np.array(sorted(picks)))
    picks.update(int(t) for t in rng.choice(rest, size=n - len(picks), replace=False))
    return np.array(sorted(picks))


@pytest.mark.parametrize("name", ["decode_t1", "decode_t4", "decode_t8", "prefill", "prefill16k"])
def test_fullsize_layer(name):
    wl, layer, xb, lg, b, hdbg, out = _run(name)
    rng = np.random.default_rng(123)
    x = synth.bf16_bits_to_f32(xb)

    # routing, quantisation, permutation: whole tensors, bit-exact
    idx, w = oracle.route_topk(lg, wl.k)
    assert np.array_equal(b["idx"].cpu().numpy(), idx)
    w_gpu = b["w"].cpu().numpy()
    assert np.allclose(w_gpu, w, rtol=0, atol=2e-6)
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

    # the sampled tokens: FC2 + combine from the GPU's own h codes and routing
    # weights (per element), and the whole layer against the oracle's chain
    toks = _token_sample(wl, idx, offsets, r2s, rng)
    assert len(toks) >= min(wl.T, 32)
    ref, up, bound = _chain(wl, xq, idx, w, toks, gpu=(hq_gpu, s2r, w_gpu))
    got = out[torch.from_numpy(toks).to(dev())].cpu().numpy().astype(np.float64)
    err = np.abs(got - up)
    assert np.all(err <= bound), f"combine: worst excess {(err - bound).max():.3e} over {len(toks)} tokens"
    rel = _rel_l2(got, ref)
    assert rel <= L2_MAX, f"layer relative L2 {rel:.3e} over {len(toks)} tokens"


@pytest.mark.parametrize("name,replays", [("decode_t1", 4), ("decode_t4", 3)])
def test_decode_graph_replays_with_changing_routing(name, replays):
    """The decode layer captured once as two calls (MoeLayer.capture with
    one_launch=False: FC2 chained to FC1; FC1 split over CTA pairs at T = 1) and replayed back to back with new
    activations and router logits before every replay, no host sync in
    between; each replay's offsets bit-exact and its output within relative
    L2 1e-2 of the oracle's chain on that replay's inputs"""
    wl = workloads.WORKLOADS[name]
    base = _layer(MX)
    layer = MoeLayer(base.w1, base.w2, wl.E, wl.k, wl.d, wl.I, MX, g_h=workloads.G_H, one_launch=False)
    x = bf16_dev(workloads.host_x_bits(wl, 0))
    lg = torch.from_numpy(workloads.host_logits(wl, 0)).to(dev())
    graph, out = layer.capture(x, lg)
    b = layer.buffers(wl.T, dev())
    inputs, outs, offs = [], [], []
    for r in range(1, replays + 1):
        xb, lr = workloads.host_x_bits(wl, r), workloads.host_logits(wl, r)
        inputs.append((xb, lr))
        x.copy_(bf16_dev(xb))
        lg.copy_(torch.from_numpy(lr).to(dev()))
        graph.replay()
        outs.append(out.clone())
        offs.append(b["offsets"].clone())
    torch.cuda.synchronize()
    ds4g.ds4g_check_device()
    prev = None
    for r, ((xb, lr), o, of) in enumerate(zip(inputs, outs, offs)):
        idx, w = oracle.route_topk(lr, wl.k)
        offsets, _, _ = oracle.moe_permute(idx, wl.E)
        assert np.array_equal(of.cpu().numpy(), offsets), f"replay {r}: offsets"
        if prev is not None:
            assert not np.array_equal(offsets, prev), "the routing did not change between replays"
        prev = offsets
        xq = oracle.quantize(synth.bf16_bits_to_f32(xb), wl.fmt)
        ref, _, _ = _chain(wl, xq, idx, w, np.arange(wl.T))
        rel = _rel_l2(o.cpu().numpy().astype(np.float64), ref)
        assert rel <= L2_MAX, f"replay {r}: layer relative L2 {rel:.3e}"


@pytest.mark.parametrize("name,replays", [("decode_t1", 3), ("decode_t4", 2), ("decode_t8", 2)])
def test_decode_one_launch_ffn_replays(name, replays):
    """The decode layer with FC1 -> FC2 + combine as one launch
    (ds4g_moe_ffn_fp4), captured once and replayed with new activations and
    routing before every replay: each replay's offsets bit-exact and its
    output within relative L2 1e-2 of the oracle's chain; after the last one
    the combine per element from the GPU's own h codes and routing weights,
    and the per-expert counters back at zero"""
    wl = workloads.WORKLOADS[name]
    base = _layer(MX)
    layer = MoeLayer(base.w1, base.w2, wl.E, wl.k, wl.d, wl.I, MX, g_h=workloads.G_H, one_launch=True)
    assert layer.uses_one_launch(wl.T)
    x = bf16_dev(workloads.host_x_bits(wl, 0))
    lg = torch.from_numpy(workloads.host_logits(wl, 0)).to(dev())
    graph, out = layer.capture(x, lg)
    b = layer.buffers(wl.T, dev())
    inputs, outs, offs = [], [], []
    for r in range(1, replays + 1):
        xb, lr = workloads.host_x_bits(wl, 10 + r), workloads.host_logits(wl, 10 + r)
        inputs.append((xb, lr))
        x.copy_(bf16_dev(xb))
        lg.copy_(torch.from_numpy(lr).to(dev()))
        graph.replay()
        outs.append(out.clone())
        offs.append(b["offsets"].clone())
    torch.cuda.synchronize()
    ds4g.ds4g_check_device()
    assert not b["ctr"].any(), "counters not reset"
    for r, ((xb, lr), o, of) in enumerate(zip(inputs, outs, offs)):
        idx, w = oracle.route_topk(lr, wl.k)
        offsets, r2s, s2r = oracle.moe_permute(idx, wl.E)
        assert np.array_equal(of.cpu().numpy(), offsets), f"replay {r}: offsets"
        xq = oracle.quantize(synth.bf16_bits_to_f32(xb), wl.fmt)
        last = r == len(inputs) - 1
        gpu = (from_dev(b["hq"]), s2r, b["w"].cpu().numpy()) if last else None
        ref, up, bound = _chain(wl, xq, idx, w, np.arange(wl.T), gpu=gpu)
        got = o.cpu().numpy().astype(np.float64)
        rel = _rel_l2(got, ref)
        assert rel <= L2_MAX, f"replay {r}: layer relative L2 {rel:.3e}"
        if last:
            err = np.abs(got - up)
            assert np.all(err <= bound), f"combine: worst excess {(err - bound).max():.3e}"
