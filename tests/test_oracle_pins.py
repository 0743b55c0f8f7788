"""Pins of the CPU oracle against things other than itself: the hand-written
tables and cases under tests/golden/, closed forms, independent library
routines (torch's float8_e4m3fn, numpy's stable argsort and matmul, scipy's
expit) and brute force on tiny inputs.  CPU only."""
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def golden_e2m1():
    tab = {}
    for line in _read("e2m1_table.txt"):
        code, s, e, m, v = line.split()
        tab[int(code, 16)] = float(v)
    return tab


E2M1 = golden_e2m1()
E2M1_POS = np.array([E2M1[c] for c in range(8)])


def golden_decode(codes):
    codes = np.asarray(codes)
    mag = E2M1_POS[codes & 7]
    return np.where(codes & 8, -mag, mag)


def unpack(data):
    """packed bytes -> codes, element 2i = low nibble (golden nibble order)"""
    data = np.asarray(data, np.uint8)
    out = np.empty(data.shape[:-1] + (data.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = data & 0x0F
    out[..., 1::2] = data >> 4
    return out


def golden_dequant(t, with_g=True):
    codes = unpack(t.data).astype(np.int64)
    K = codes.shape[1]
    blk = oracle.BLOCK[t.fmt]
    sb = np.repeat(t.scales.astype(np.int64), blk, axis=1)[:, :K]
    if t.fmt == oracle.MX:
        sc = np.ldexp(1.0, sb - 127)
    else:
        sc = torch.from_numpy(sb.astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()
        if with_g:
            sc = sc * t.g
    return golden_decode(codes) * sc


# ---- codecs ----------------------------------------------------------------

def test_e2m1_table_exhaustive():
    for c in range(16):
        v = oracle.e2m1_decode(c)
        assert v == E2M1[c]
        assert np.signbit(v) == bool(c & 8)
        assert oracle.e2m1_encode(v) == c


def test_lut_claim():
    # any 16-entry lookup table decodes FP4 losslessly (sec. 5 of the PR #454 page)
    assert oracle.lut_decode_check() == 0


def test_e2m1_rounding_cases():
    for line in _read("e2m1_rounding_cases.txt"):
        x, code = line.split()
        assert oracle.e2m1_encode(float(x)) == int(code, 16), line


def test_e2m1_encode_is_nearest_bruteforce():
    rng = np.random.default_rng(1)
    for y in rng.uniform(-8, 8, 2000):
        c = oracle.e2m1_encode(y)
        d = abs(abs(y) - E2M1_POS)
        assert d[c & 7] == d.min()


def test_nibble_order():
    for line in _read("nibble_order.txt"):
        b, lo, hi = (int(v, 16) for v in line.split())
        t = oracle.Fp4(np.array([[b] * 16], np.uint8), np.array([[127]], np.uint8), 1.0, oracle.MX)
        deq = oracle.dequantize(t)
        assert deq[0, 0] == E2M1[lo] and deq[0, 1] == E2M1[hi]


def test_ue8m0_closed_form_and_roundtrip():
    for b in range(255):
        assert oracle.ue8m0_decode(b) == np.ldexp(1.0, b - 127)
    assert np.isnan(oracle.ue8m0_decode(255))


def test_ue4m3_against_torch_float8():
    vals = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for b in range(127):
        assert oracle.ue4m3_decode(b) == vals[b]
        assert oracle.ue4m3_encode(vals[b]) == b
    assert oracle.ue4m3_decode(0x7E) == 448.0
    assert np.isnan(oracle.ue4m3_decode(0x7F))
    # RNE encode of arbitrary fp32 values in range agrees with torch's conversion
    rng = np.random.default_rng(2)
    r = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(-16, 6, 3000))]).astype(np.float32)
    r = r[r <= 448]
    ref = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.ue4m3_encode(float(v)) for v in r])
    assert np.array_equal(got, ref)
    assert oracle.ue4m3_encode(1000.0) == 0x7E


# ---- quantisation ----------------------------------------------------------

def test_mx_block_cases():
    for line in _read("mx_block_cases.txt"):
        vals, sbyte, codes = (p.strip() for p in line.split(";"))
        v = np.zeros((1, 32), np.float32)
        listed = np.array([float(t) for t in vals.split()], np.float32)
        v[0, :len(listed)] = listed
        q = oracle.quantize(v, oracle.MX)
        assert int(q.scales[0, 0]) == int(sbyte), line
        got = unpack(q.data)[0, :len(listed)]
        assert [int(c) for c in got] == [int(c, 16) for c in codes.split()], line


def _mx_ref_block(v):
    """independent restatement with numpy: X from the float's exponent via
    np.frexp, codes by nearest-even search over the golden table"""
    amax = np.abs(v).max()
    X = -127 if amax == 0 else int(np.clip(np.frexp(amax)[1] - 1 - 2, -127, 127))
    y = np.ldexp(v.astype(np.float64), -X)
    a = np.abs(y)[:, None]
    d = np.abs(a - E2M1_POS[None, :])
    best = np.argmin(d, axis=1)
    # resolve exact ties to even code
    for i in range(len(best)):
        m = d[i].min()
        cands = [c for c in range(8) if d[i, c] == m]
        best[i] = [c for c in cands if c % 2 == 0][0] if len(cands) > 1 else cands[0]
    return X + 127, best | np.where(np.signbit(y), 8, 0)


def test_mx_quantize_matches_independent_restatement():
    x = synth.normal_f32((8, 256), seed=0, stream=99, sigma=1.0)
    x[0, :32] = 0.0
    x[1, 32:64] *= 1e-30
    q = oracle.quantize(x, oracle.MX)
    codes = unpack(q.data)
    for r in range(8):
        for b in range(8):
            sb, c = _mx_ref_block(x[r, b * 32:(b + 1) * 32])
            assert q.scales[r, b] == sb
            assert np.array_equal(codes[r, b * 32:(b + 1) * 32], c)


def test_quantize_laws_mx_nv():
    x = synth.normal_f32((16, 512), seed=0, stream=98, sigma=3.0)
    for fmt in (oracle.MX, oracle.NV):
        q = oracle.quantize(x, fmt)
        deq = golden_dequant(q)
        assert np.array_equal(deq, oracle.dequantize(q))
        # idempotence: re-quantising the dequantised values changes nothing
        q2 = oracle.quantize(deq.astype(np.float32), fmt, g=q.g if fmt == oracle.NV else None)
        assert np.array_equal(golden_dequant(q2), deq)
        # error bound: half a grid step of the block scale (or saturation)
        blk = oracle.BLOCK[fmt]
        codes = unpack(q.data)
        if fmt == oracle.MX:
            sc = np.ldexp(1.0, np.repeat(q.scales.astype(np.int64), blk, axis=1) - 127)
        else:
            sc = torch.from_numpy(np.repeat(q.scales, blk, axis=1)).view(torch.float8_e4m3fn).double().numpy() * q.g
        step = np.where((codes & 7) >= 6, 2.0, np.where((codes & 7) >= 4, 1.0, 0.5)) * sc
        err = np.abs(x.astype(np.float64) - deq)
        sat = (codes & 7) == 7
        assert np.all((err <= 0.5 * step * (1 + 1e-6)) | sat)
        assert np.all(np.abs(x[sat]) >= 5.0 * sc[sat] * (1 - 1e-6))


def test_nv_scale_matches_torch_e4m3():
    x = synth.normal_f32((4, 256), seed=0, stream=97, sigma=1.0)
    q = oracle.quantize(x, oracle.NV)
    amax_t = np.abs(x).max()
    assert q.g == np.float32(amax_t) / np.float32(2688.0)
    six_g = np.float32(6.0) * np.float32(q.g)
    amax_b = np.abs(x.reshape(4, 16, 16)).max(axis=2)
    r = (amax_b / six_g).astype(np.float32)
    ref = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q.scales, ref)


# ---- GEMM ------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [oracle.MX, oracle.NV])
@pytest.mark.parametrize("K", [64, 128])
def test_gemm_bruteforce_tiny(fmt, K):
    E, N = 3, 8
    a = synth.normal_f32((7, K), seed=0, stream=96, sigma=1.0)
    w = synth.normal_f32((E * N, K), seed=0, stream=95, sigma=0.5)
    aq, wq = oracle.quantize(a, fmt), oracle.quantize(w, fmt)
    offsets = np.array([0, 2, 2, 7], np.int32)          # expert 1 is empty
    out, ab = oracle.grouped_gemm(aq, offsets, wq, N)
    # operands without the NV tensor scales: every product and the K <= 128
    # sums are exact in fp64, so the unscaled results must match bit for bit
    A, W = golden_dequant(aq, with_g=False), golden_dequant(wq, with_g=False)
    gg = aq.g * wq.g if fmt == oracle.NV else 1.0
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            ref = W[e * N:(e + 1) * N] @ A[r]
            assert np.array_equal(out[r], ref * gg)
            assert np.array_equal(ab[r], (np.abs(W[e * N:(e + 1) * N]) @ np.abs(A[r])) * gg)


def test_gemm_unit_scales_integer():
    # all scale bytes 127: every operand is an E2M1 value, 4 * sum is an integer
    rng = np.random.default_rng(3)
    a = oracle.Fp4(rng.integers(0, 256, (4, 32), dtype=np.uint8), np.full((4, 2), 127, np.uint8), 1.0, oracle.MX)
    w = oracle.Fp4(rng.integers(0, 256, (6, 32), dtype=np.uint8), np.full((6, 2), 127, np.uint8), 1.0, oracle.MX)
    out, _ = oracle.grouped_gemm(a, np.array([0, 4], np.int32), w, 6)
    assert np.all(4 * out == np.round(4 * out))
    ci = golden_decode(unpack(a.data).astype(np.int64)) * 2
    wi = golden_decode(unpack(w.data).astype(np.int64)) * 2
    assert np.array_equal(4 * out, (ci.astype(np.int64) @ wi.astype(np.int64).T).astype(np.float64))


def test_expert_gemm_rows_matches_grouped():
    K, N, E = 128, 16, 2
    a = oracle.quantize(synth.normal_f32((5, K), 0, 94), oracle.MX)
    w = oracle.quantize(synth.normal_f32((E * N, K), 0, 93, 0.02), oracle.MX)
    offsets = np.array([0, 3, 5], np.int32)
    full, _ = oracle.grouped_gemm(a, offsets, w, N)
    w1 = oracle.Fp4(w.data[N:], w.scales[N:], 1.0, oracle.MX)
    sub, _ = oracle.expert_gemm_rows(a, np.array([3, 4]), w1, (4, 12))
    assert np.array_equal(sub, full[3:5, 4:12])


# ---- routing / permutation --------------------------------------------------

def test_topk_full_sort_and_softmax():
    lg = synth.logits(20, 8, seed=0)
    lg[3, 2] = lg[3, 5]                      # a tie: lower index first
    idx, w = oracle.route_topk(lg, 8)
    for t in range(20):
        assert np.array_equal(idx[t], np.argsort(-lg[t].astype(np.float64), kind="stable"))
    sel = np.take_along_axis(lg.astype(np.float64), idx, axis=1)
    ref = np.exp(sel - sel.max(axis=1, keepdims=True))
    ref /= ref.sum(axis=1, keepdims=True)
    assert np.allclose(w, ref, rtol=1e-15, atol=0)
    idx2, w2 = oracle.route_topk(lg, 2)
    assert np.array_equal(idx2, idx[:, :2])
    assert np.allclose(w2.sum(axis=1), 1.0, atol=1e-15)
    assert np.all(np.diff(w2, axis=1) <= 0)


def test_topk_non_finite_logits():
    """A NaN logit ranks as -inf; a pick equal to the token's maximum has
    softmax factor 1, the limit of the softmax when the maximum is +inf or
    every pick is -inf.  Ranking is checked against a stable sort of that key,
    the weights against the limits in closed form."""
    E, k = 8, 3
    lg = synth.logits(7, E, seed=1)
    lg[0, :] = -np.inf                       # all -inf: experts 0..k-1, equal weights
    lg[1, 4] = np.inf                        # one +inf takes all the weight
    lg[2, [1, 6]] = np.inf                   # two +inf: half each, lower index first
    lg[3, :] = np.nan
    lg[3, 5] = 0.0                           # the one number first, then NaNs in index order
    lg[4, [0, 2]] = np.nan                   # NaNs among numbers are never picked
    lg[5, :] = np.nan                        # all NaN: as all -inf
    lg[6, [3, 7]] = -np.inf                  # -inf among numbers
    idx, w = oracle.route_topk(lg, k)
    key = np.where(np.isnan(lg), -np.inf, lg.astype(np.float64))
    for t in range(lg.shape[0]):
        assert np.array_equal(idx[t], np.argsort(-key[t], kind="stable")[:k])
    assert np.array_equal(idx[0], [0, 1, 2]) and np.array_equal(idx[5], [0, 1, 2])
    assert np.allclose(w[0], 1.0 / k, rtol=1e-15) and np.allclose(w[5], 1.0 / k, rtol=1e-15)
    assert idx[1, 0] == 4 and np.array_equal(w[1], [1.0, 0.0, 0.0])
    assert np.array_equal(idx[2, :2], [1, 6]) and np.array_equal(w[2], [0.5, 0.5, 0.0])
    assert idx[3, 0] == 5 and np.array_equal(idx[3, 1:], [0, 1]) and np.array_equal(w[3], [1.0, 0.0, 0.0])
    for t in (4, 6):
        sel = key[t, idx[t]]
        assert np.all(np.isfinite(sel))
        ref = np.exp(sel - sel.max())
        assert np.allclose(w[t], ref / ref.sum(), rtol=1e-15, atol=0)


def test_permute_invariants():
    T, k, E = 37, 3, 16
    lg = synth.logits(T, E, seed=0, bias_sigma=1.5)
    idx, _ = oracle.route_topk(lg, k)
    offsets, r2s, s2r = oracle.moe_permute(idx, E)
    S = T * k
    counts = np.bincount(idx.ravel(), minlength=E)
    assert offsets[0] == 0 and offsets[-1] == S
    assert np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(r2s), np.arange(S))
    assert np.array_equal(s2r[r2s], np.arange(S))
    assert np.array_equal(r2s, np.argsort(idx.ravel(), kind="stable"))
    for e in range(E):
        seg = r2s[offsets[e]:offsets[e + 1]]
        assert np.all(idx.ravel()[seg] == e)
        assert np.all(np.diff(seg) > 0)


def test_gather_commutes_with_quantise():
    T, k, E, K = 9, 2, 4, 64
    x = synth.normal_f32((T, K), 0, 92)
    idx, _ = oracle.route_topk(synth.logits(T, E, 0), k)
    _, r2s, _ = oracle.moe_permute(idx, E)
    for fmt in (oracle.MX,):
        a = oracle.gather_rows(oracle.quantize(x, fmt), r2s, k)
        b = oracle.quantize(x[r2s // k], fmt)
        assert np.array_equal(a.data, b.data) and np.array_equal(a.scales, b.scales)


# ---- SwiGLU / combine / layer ------------------------------------------------

def test_swiglu_against_expit():
    y1 = synth.normal_f32((6, 64), 0, 91, 3.0)
    h = oracle.swiglu(y1)
    g, u = y1[:, :32].astype(np.float64), y1[:, 32:].astype(np.float64)
    assert np.array_equal(h, (g * expit(g) * u).astype(np.float32)) or np.allclose(h, g * expit(g) * u, rtol=2e-7)
    z = np.zeros((1, 4), np.float32)
    z[0, 2:] = 5.0
    assert oracle.swiglu(z)[0, 0] == 0.0


def test_combine_identity_and_linearity():
    T, k, d = 5, 2, 8
    y2 = synth.normal_f32((T * k, d), 0, 90).astype(np.float64)
    s2r = np.arange(T * k, dtype=np.int32)[::-1].copy()
    w = np.zeros((T, k))
    w[:, 0] = 1.0
    out = oracle.moe_combine(y2, s2r, w)
    assert np.array_equal(out, y2[s2r.reshape(T, k)[:, 0]])
    w = np.full((T, k), 0.5)
    out = oracle.moe_combine(y2, s2r, w)
    assert np.allclose(out, 0.5 * y2[s2r.reshape(T, k)].sum(axis=1), rtol=1e-15)


def test_layer_reduces_to_dense_chain():
    # E = 1, k = 1: routing is trivial and the layer is GEMM -> SwiGLU -> GEMM
    T, d, I = 4, 64, 32
    x = synth.bf16_bits_to_f32(synth.normal_bf16_bits((T, d), 0, synth.STREAM_X))
    lg = synth.logits(T, 1, 0)
    w1 = oracle.quantize(synth.normal_f32((2 * I, d), 0, synth.STREAM_W1, 0.02), oracle.MX)
    w2 = oracle.quantize(synth.normal_f32((d, I), 0, synth.STREAM_W2, 0.02), oracle.MX)
    res = oracle.moe_layer(x, lg, w1, w2, 1, oracle.MX)
    assert np.all(res["w"] == 1.0)
    A = golden_dequant(oracle.quantize(x, oracle.MX))
    y1 = (A @ golden_dequant(w1).T).astype(np.float32)
    h = oracle.swiglu(y1)
    Hq = golden_dequant(oracle.quantize(h, oracle.MX))
    y2 = (Hq @ golden_dequant(w2).T).astype(np.float32)
    assert np.allclose(res["out"], y2.astype(np.float64), rtol=1e-6, atol=1e-9)


# ---- FP8 (E4M3) activations: the MXFP8 format of the FP8 x FP4 variant ------

def test_e4m3_against_torch_float8():
    """all 256 codes decode as torch's float8_e4m3fn; every finite code
    re-encodes to itself (sign of zero kept); the RNE encode of in-range fp32
    values agrees with torch's conversion; beyond 448 the encode saturates"""
    codes = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if np.isnan(tv[c]):
            assert np.isnan(v) and c in (0x7F, 0xFF)
            continue
        assert v == tv[c] and np.signbit(v) == np.signbit(tv[c])
        assert oracle.e4m3_encode(v) == c
    rng = np.random.default_rng(5)
    r = np.concatenate([rng.uniform(-448, 448, 4000), rng.choice([-1, 1], 4000) * np.exp(rng.uniform(-14, 6, 4000)),
                        rng.normal(0, 1e-3, 1000)]).astype(np.float32)
    ref = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in r])
    assert np.array_equal(got, ref)
    # saturation: 464 is halfway between 448 and the NaN code's 480, so the
    # nearest finite value is 448 either way
    assert oracle.e4m3_encode(464.0) == 0x7E and oracle.e4m3_encode(1e6) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE and oracle.e4m3_encode(-0.0) == 0x80


def test_mx8_block_cases():
    for line in _read("mx8_block_cases.txt"):
        vals, sbyte, codes = (p.strip() for p in line.split(";"))
        v = np.zeros((1, 32), np.float32)
        listed = np.array([float(t) for t in vals.split()], np.float32)
        v[0, :len(listed)] = listed
        q = oracle.quantize(v, oracle.MX8)
        assert q.data.shape == (1, 32) and q.scales.shape == (1, 1)
        assert int(q.scales[0, 0]) == int(sbyte), line
        assert [int(c) for c in q.data[0, :len(listed)]] == [int(c, 16) for c in codes.split()], line


def test_mx8_quantize_matches_independent_restatement():
    """numpy restatement: X from np.frexp, codes from torch's E4M3 conversion
    of the scaled values clipped to the largest finite magnitude"""
    x = synth.normal_f32((8, 256), seed=0, stream=93, sigma=2.0)
    x[0, :32] = 0.0
    x[1, 32:64] *= 1e-30
    x[2, 64] = 1e30
    q = oracle.quantize(x, oracle.MX8)
    for r in range(8):
        for b in range(8):
            v = x[r, b * 32:(b + 1) * 32]
            amax = np.abs(v).max()
            X = -127 if amax == 0 else int(np.clip(np.frexp(amax)[1] - 1 - 8, -127, 127))
            assert q.scales[r, b] == X + 127
            y = np.clip(np.ldexp(v.astype(np.float64), -X), -448, 448).astype(np.float32)
            ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q.data[r, b * 32:(b + 1) * 32], ref)


def test_quantize_laws_mx8():
    x = synth.normal_f32((16, 512), seed=0, stream=92, sigma=3.0)
    q = oracle.quantize(x, oracle.MX8)
    sc = np.ldexp(1.0, np.repeat(q.scales.astype(np.int64), 32, axis=1) - 127)
    deq = torch.from_numpy(q.data).view(torch.float8_e4m3fn).double().numpy() * sc
    assert np.array_equal(deq, oracle.dequantize(q))
    q2 = oracle.quantize(deq.astype(np.float32), oracle.MX8)
    assert np.array_equal(oracle.dequantize(q2), deq)
    # error within half an E4M3 step (3 mantissa bits: step 2^(e-10) of the
    # scaled value, or the subnormal step 2^-9) unless saturated
    y = np.abs(x.astype(np.float64)) / sc
    e = np.floor(np.log2(np.maximum(y, 2.0 ** -6)))
    step = np.ldexp(1.0, (e - 3).astype(np.int64)) * sc
    err = np.abs(x - deq)
    sat = (q.data & 0x7F) == 0x7E
    assert np.all((err <= 0.5 * step * (1 + 1e-9)) | sat)


@pytest.mark.parametrize("K", [64, 128])
def test_gemm_mixed_fp8_fp4_bruteforce_tiny(K):
    """FP8 (MXFP8) activations x FP4 (MXFP4) weights: each product of an E4M3
    and an E2M1 value with power-of-two scales is exact in fp64, so the
    result equals numpy's matmul of the dequantised operands bit for bit"""
    N = 8
    a = synth.normal_f32((5, K), seed=0, stream=91, sigma=1.0)
    w = synth.normal_f32((N, K), seed=0, stream=90, sigma=0.5)
    aq, wq = oracle.quantize(a, oracle.MX8), oracle.quantize(w, oracle.MX)
    out, ab = oracle.expert_gemm_rows(aq, np.arange(5), wq, (0, N))
    A = torch.from_numpy(aq.data).view(torch.float8_e4m3fn).double().numpy() * \
        np.ldexp(1.0, np.repeat(aq.scales.astype(np.int64), 32, axis=1) - 127)
    W = golden_dequant(wq, with_g=False)
    assert np.array_equal(out, A @ W.T)
    assert np.array_equal(ab, np.abs(A) @ np.abs(W).T)


def test_gather_mx8_rows():
    x = synth.normal_f32((5, 128), seed=0, stream=89, sigma=1.0)
    q = oracle.quantize(x, oracle.MX8)
    r2s = np.array([4, 0, 9, 2, 7, 5], np.int32)        # k = 2: token = slot // 2
    g = oracle.gather_rows(q, r2s, 2)
    assert np.array_equal(g.data, q.data[r2s // 2]) and np.array_equal(g.scales, q.scales[r2s // 2])


def test_encoders_saturate_far_beyond_the_range():
    """the nearest representable value to anything beyond the largest finite
    one is that value, also where the distances themselves round (|y| near
    1e30 and beyond)"""
    for y in (6.0, 7.0, 1e10, 1e30, 1e300):
        assert oracle.e2m1_encode(y) == 0x7 and oracle.e2m1_encode(-y) == 0xF
    for y in (448.0, 1e10, 1e30, 1e300):
        assert oracle.e4m3_encode(y) == 0x7E and oracle.e4m3_encode(-y) == 0xFE
        assert oracle.ue4m3_encode(y) == 0x7E


def test_grouped_gemm_fp8_weights_bruteforce_tiny():
    """MXFP8 activations x MXFP8 weights (the shared expert's FP8 weights),
    grouped over experts: numpy's matmul of the dequantised operands, exact"""
    E, N, K = 3, 8, 128
    a = synth.normal_f32((7, K), seed=0, stream=88, sigma=1.0)
    w = synth.normal_f32((E * N, K), seed=0, stream=87, sigma=0.5)
    aq, wq = oracle.quantize(a, oracle.MX8), oracle.quantize(w, oracle.MX8)
    offsets = np.array([0, 2, 2, 7], np.int32)
    out, ab = oracle.grouped_gemm(aq, offsets, wq, N)

    def deq(t):
        return torch.from_numpy(t.data).view(torch.float8_e4m3fn).double().numpy() * \
            np.ldexp(1.0, np.repeat(t.scales.astype(np.int64), 32, axis=1) - 127)
    A, W = deq(aq), deq(wq)
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            assert np.array_equal(out[r], W[e * N:(e + 1) * N] @ A[r])
            assert np.array_equal(ab[r], np.abs(W[e * N:(e + 1) * N]) @ np.abs(A[r]))
