"""Expert parallelism's device side on one GPU (a one-rank NCCL group: the
exchanges move rows to the rank itself, every kernel of the path runs):
ds4g_segment_ids against numpy, and EpMoeLayer (MXFP4 and NVFP4) against
the oracle's chain of the same layer (relative L2 <= 1e-2).  The multi-rank exchange logic is
covered on CPU (tests/test_ep_cpu.py); this run has one GPU."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_helpers import bf16_dev, dev
from synth import workloads

pytestmark = pytest.mark.gpu

ds4g = pytest.importorskip("block_scaled_fp4_topk_b200.ds4g")


@pytest.mark.parametrize("counts,modulo", [([3, 0, 5, 1, 0, 2], 3), ([0, 0, 7], 1), ([4, 4, 4, 4], 2), ([], 1)])
def test_segment_ids(counts, modulo):
    bounds = np.concatenate([[5], 5 + np.cumsum(counts)]).astype(np.int32)     # offsets need not start at 0
    nseg = max(len(counts), 1)
    if not counts:
        bounds = np.array([5, 5], np.int32)
    rows = int(bounds[-1] - bounds[0])
    got = ds4g.ds4g_segment_ids(torch.from_numpy(bounds).to(dev()), nseg, modulo, rows).cpu().numpy()
    ref = np.repeat(np.arange(nseg) % modulo, np.diff(bounds))
    assert np.array_equal(got, ref)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_layer(wl, x, lg, fmt):
    """the oracle's chain of the layer with per-expert weights (NVFP4: each
    expert's tensor scale; h requantised with the static tensor scale of h)"""
    idx, w = oracle.route_topk(lg, wl.k)
    xq = oracle.quantize(x, fmt)
    offsets, r2s, s2r = oracle.moe_permute(idx, wl.E)
    a = oracle.gather_rows(xq, r2s, wl.k)
    y2 = np.zeros((a.data.shape[0], wl.d))
    g_h = workloads.G_H if fmt == oracle.NV else None
    for e in range(wl.E):
        rows = np.arange(offsets[e], offsets[e + 1])
        if not len(rows):
            continue
        W1 = oracle.quantize(workloads.host_w1(wl, e), fmt)
        W2 = oracle.quantize(workloads.host_w2(wl, e), fmt)
        y1 = oracle.expert_gemm_rows(a, rows, W1, (0, 2 * wl.I))[0]
        hq = oracle.quantize(oracle.swiglu(y1.astype(np.float32)), fmt, g=g_h)
        y2[rows] = oracle.expert_gemm_rows(hq, np.arange(len(rows)), W2, (0, wl.d))[0]
    return oracle.moe_combine(y2, s2r, w)


@pytest.mark.parametrize("fmt", [oracle.MX, oracle.NV])
def test_ep_layer_one_rank(fmt):
    import torch.distributed as dist
    from block_scaled_fp4_topk_b200.ep import EpMoeLayer
    from bench import synthetic_weights
    wl = workloads.Workload("ep_gpu", T=64, E=8, k=2, d=512, I=512, fmt=fmt, bias_sigma=1.5)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1)
    try:
        w1, w2 = synthetic_weights(wl.E, wl.d, wl.I, fmt, device=dev())
        layer = EpMoeLayer(w1, w2, wl.E, wl.k, wl.d, wl.I, g_h=workloads.G_H)
        xb, lg = workloads.host_x_bits(wl), workloads.host_logits(wl)
        out = layer.forward(bf16_dev(xb), torch.from_numpy(lg).to(dev())).cpu().numpy().astype(np.float64)
        ds4g.ds4g_check_device()
    finally:
        dist.destroy_process_group()
    ref = _oracle_layer(wl, synth.bf16_bits_to_f32(xb), lg, fmt)
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel <= 1e-2, rel
