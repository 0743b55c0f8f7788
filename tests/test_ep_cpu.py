"""Expert parallelism's host side on CPU: two gloo ranks, each with its own
tokens and half of the experts, run the plan and the exchanges of
block_scaled_fp4_topk_b200.ep (row counts, quantised rows, FC2 rows back;
for NVFP4 also the shared activation tensor scale) with the oracle doing each
step's arithmetic in place of the library's kernels.  Every rank's output
must equal the single-rank oracle layer on its own tokens (quantised with the
same tensor scale) bit for bit: the exchange only moves rows, and every row
meets the same arithmetic.  Also: the plan's arithmetic on hand-written
counts."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

E, K_TOP, D, I, T = 8, 2, 256, 128, 24


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _weights(e, fmt):
    import oracle
    from synth import workloads
    wl = workloads.Workload("ep_cpu", T=T, E=E, k=K_TOP, d=D, I=I, fmt=fmt, bias_sigma=1.5)
    return oracle.quantize(workloads.host_w1(wl, e), fmt), oracle.quantize(workloads.host_w2(wl, e), fmt)


def _h_q(y1, fmt):
    """h = SwiGLU(y1) requantised (NVFP4: with the static tensor scale of h)"""
    import oracle
    from synth import workloads
    return oracle.quantize(oracle.swiglu(y1.astype(np.float32)), fmt, g=workloads.G_H if fmt == oracle.NV else None)


def _tokens(rank):
    import synth
    from synth import workloads
    wl = workloads.Workload("ep_cpu", T=T, E=E, k=K_TOP, d=D, I=I, fmt=0, bias_sigma=1.5)
    return synth.bf16_bits_to_f32(workloads.host_x_bits(wl, rank)), workloads.host_logits(wl, rank)


def _expert_rows(a, rows, e, which, fmt):
    import oracle
    W1, W2 = _weights(e, fmt)
    if which == 1:
        return oracle.expert_gemm_rows(a, rows, W1, (0, 2 * I))[0]
    return oracle.expert_gemm_rows(a, rows, W2, (0, D))[0]


def _local_layer(x, lg, fmt, g):
    """the single-rank oracle layer on these tokens, all experts (NVFP4: the
    activations quantised with tensor scale g)"""
    import oracle
    idx, w = oracle.route_topk(lg, K_TOP)
    xq = oracle.quantize(x, fmt, g=g)
    offsets, r2s, s2r = oracle.moe_permute(idx, E)
    a = oracle.gather_rows(xq, r2s, K_TOP)
    y2 = np.zeros((a.data.shape[0], D))
    for e in range(E):
        rows = np.arange(offsets[e], offsets[e + 1])
        if len(rows):
            y1 = _expert_rows(a, rows, e, 1, fmt)
            y2[rows] = _expert_rows(_h_q(y1, fmt), np.arange(len(rows)), e, 2, fmt)
    return oracle.moe_combine(y2, s2r, w)


def _rank(rank, world, port, q, fmt):
    try:
        _rank_body(rank, world, port, q, fmt)
    except BaseException as exc:          # report at once instead of leaving the parent waiting
        q.put((rank, False, float("nan"), repr(exc), None))
        raise


def _rank_body(rank, world, port, q, fmt):
    import torch
    import torch.distributed as dist
    import oracle
    from block_scaled_fp4_topk_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    G, El = world, ep.experts_per_rank(E, world)
    x, lg = _tokens(rank)
    # NVFP4: one activation tensor scale for all ranks, the largest of theirs
    g = None
    if fmt == oracle.NV:
        g_local = torch.tensor([oracle.quantize(x, oracle.NV).g], dtype=torch.float32)
        g = float(ep.shared_tensor_scale(g_local).item())
    # dispatch on this rank's tokens, all E experts
    idx, w = oracle.route_topk(lg, K_TOP)
    xq = oracle.quantize(x, fmt, g=g)
    offsets, r2s, s2r = oracle.moe_permute(idx, E)
    a = oracle.gather_rows(xq, r2s, K_TOP)
    # the plan and the exchanges of the library's expert-parallel layer
    sc = ep.send_counts(offsets, G)
    rcnt = ep.exchange(torch.from_numpy(ep.expert_counts(offsets)), [El] * G, [El] * G).numpy()
    rc, bounds = ep.recv_layout(rcnt, G)
    rd = ep.exchange(torch.from_numpy(a.data), sc, rc).numpy()
    rs = ep.exchange(torch.from_numpy(a.scales), sc, rc).numpy()
    R = int(bounds[-1])
    # receiver: local experts of the received rows, their expert-contiguous
    # order, FC1, SwiGLU, requantisation, FC2, rows back in received order
    ids = np.repeat(np.arange(G * El) % El, np.diff(bounds)).astype(np.int32)
    offs_l, r2s_l, s2r_l = oracle.moe_permute(ids.reshape(R, 1), El)
    a_l = oracle.gather_rows(oracle.Fp4(rd, rs, 1.0 if g is None else g, fmt), r2s_l, 1)
    y2_l = np.zeros((R, D))
    for le in range(El):
        rows = np.arange(offs_l[le], offs_l[le + 1])
        if len(rows):
            e = rank * El + le
            y1 = _expert_rows(a_l, rows, e, 1, fmt)
            y2_l[rows] = _expert_rows(_h_q(y1, fmt), np.arange(len(rows)), e, 2, fmt)
    y2_recv = y2_l[s2r_l]
    y2_back = ep.exchange(torch.from_numpy(y2_recv), rc, sc).numpy()
    out = oracle.moe_combine(y2_back, s2r, w)
    ref = _local_layer(x, lg, fmt, g)
    q.put((rank, bool(np.array_equal(out, ref)), float(np.abs(out - ref).max()), sc, rc))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt", [0, 1])
def test_two_rank_expert_parallel_exchange_matches_local_layer(fmt):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, fmt)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
    for rank, same, err, sc, rc in res:
        assert same, f"rank {rank}: expert-parallel output differs from the local layer ({err}, {sc})"
    assert all(p.exitcode == 0 for p in procs)
    # what rank 0 sends to rank 1 is what rank 1 receives from rank 0, and back
    assert res[0][3][1] == res[1][4][0] and res[1][3][0] == res[0][4][1]
    assert sum(res[0][3]) == T * K_TOP and sum(res[1][3]) == T * K_TOP


def test_plan_on_hand_written_counts():
    from block_scaled_fp4_topk_b200 import ep
    offsets = [0, 3, 3, 7, 9, 9, 9, 12, 12]          # 8 experts, 12 rows
    assert ep.send_counts(offsets, 2) == [9, 3]      # experts 0-3 / 4-7
    assert ep.send_counts(offsets, 4) == [3, 6, 0, 3]
    assert list(ep.expert_counts(offsets)) == [3, 0, 4, 2, 0, 0, 3, 0]
    # received from 2 sources, 2 local experts each: counts [src0 e0, src0 e1, src1 e0, src1 e1]
    per_source, bounds = ep.recv_layout([1, 2, 0, 4], 2)
    assert per_source == [3, 4] and list(bounds) == [0, 1, 3, 3, 7]
    try:
        ep.experts_per_rank(8, 3)
        raise AssertionError("8 experts over 3 ranks must be refused")
    except ValueError:
        pass
