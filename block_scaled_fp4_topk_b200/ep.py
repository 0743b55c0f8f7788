"""Expert parallelism across GPUs: one MoE layer whose E experts are split
over G ranks (rank r holds experts [r E/G, (r + 1) E/G)), each rank with its
own tokens.  The dispatch of the pages' MoE layer ("Moore Threads full-link
adaptation of DeepSeek-V4": MoE dispatch / combine across devices;
"DGX Spark native FP4 matrix instructions ...", sec. 6: several GPUs), as:

  1. routing, quantisation and the expert-contiguous permutation of the
     rank's own tokens (one library call).  Experts of one rank are
     contiguous, so the permuted rows are already grouped by destination;
  2. an exchange of the per-expert row counts, then of the quantised rows
     (codes and scales), over NCCL (all_to_all_single);
  3. on the receiving rank: each row's local expert from the counts
     (ds4g_segment_ids), the expert-contiguous order of all received rows
     (ds4g_moe_permute with one slot per row), FC1 with the fused SwiGLU +
     requantisation and FC2 over the rank's experts, and the FC2 rows put back
     in received order (ds4g_moe_combine with one slot per row, weight 1);
  4. the FC2 rows sent back to their source ranks (all_to_all_single, the
     splits reversed), which combine them with their routing weights.

The data plane is NCCL; the row counts travel to the host once per step
(the splits of the exchanges).  MXFP4 or NVFP4 weights and activations.  With
NVFP4 every rank quantises its activations with one shared tensor scale, the
largest of the ranks' own (an all-reduce of one float before the dispatch),
so that an expert's rows from all ranks share their scale, as its GEMMs need.

The host-side pieces (the plan of the exchanges and the exchange itself) are
plain functions so that multi-rank tests can run them on CPU tensors.
"""
import numpy as np
import torch
import torch.distributed as dist

from . import ds4g
from .ds4g import EPI_NONE, EPI_SWIGLU_REQUANT, MXFP4, NVFP4, Fp4Tensor


def experts_per_rank(E, G):
    if E % G != 0:
        raise ValueError(f"{E} experts do not split over {G} ranks")
    return E // G


def send_counts(offsets, G):
    """rows of this rank's permuted batch bound for each rank, from the
    expert offsets [E + 1] (host): experts of rank d are [d E/G, (d+1) E/G)"""
    offsets = np.asarray(offsets, np.int64)
    El = experts_per_rank(len(offsets) - 1, G)
    return [int(offsets[(d + 1) * El] - offsets[d * El]) for d in range(G)]


def expert_counts(offsets):
    """rows per expert [E] (int64), grouped by destination rank already"""
    return np.diff(np.asarray(offsets, np.int64))


def recv_layout(recv_expert_counts, G):
    """from the counts received from each source rank for each local expert
    ([G * El], source-major): rows from each source and the group boundaries
    [G * El + 1] of the received rows (source-major, then expert)"""
    c = np.asarray(recv_expert_counts, np.int64).reshape(G, -1)
    per_source = [int(x) for x in c.sum(axis=1)]
    bounds = np.concatenate([[0], np.cumsum(c.reshape(-1))]).astype(np.int64)
    return per_source, bounds


def shared_tensor_scale(g_local, group=None):
    """the NVFP4 activation tensor scale every rank quantises with: the
    largest of the ranks' own (fp32 [1], in place)"""
    dist.all_reduce(g_local, op=dist.ReduceOp.MAX, group=group)
    return g_local


def exchange(send, send_splits, recv_splits, group=None):
    """all_to_all of the rows of `send` (first dimension split by
    send_splits, one part per rank) into a new tensor of sum(recv_splits)
    rows, parts in rank order"""
    recv = torch.empty((int(sum(recv_splits)),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(recv, send.contiguous(), list(map(int, recv_splits)), list(map(int, send_splits)),
                           group=group)
    return recv


class EpMoeLayer:
    """One MoE layer with its experts split over the ranks of `group`
    (NCCL).  w1_local [El*2I][d], w2_local [El*d][I]: MXFP4 or NVFP4 weights
    of this rank's experts, El = E / world_size (NVFP4: w.g holds the El
    experts' tensor scales); g_h: the static NVFP4 tensor scale of h."""

    def __init__(self, w1_local, w2_local, E, k, d, I, group=None, g_h=1.0):
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.El = experts_per_rank(E, self.G)
        self.w1, self.w2 = w1_local, w2_local
        self.E, self.k, self.d, self.I = E, k, d, I
        self.fmt = w1_local.fmt
        if self.fmt not in (MXFP4, NVFP4) or w2_local.fmt != self.fmt:
            raise ValueError("expert parallelism takes MXFP4 or NVFP4 weights, both GEMMs the same")
        self.g_h = None
        if self.fmt == NVFP4:
            self.g_h = torch.tensor([g_h], dtype=torch.float32, device=w1_local.data.device)

    def forward(self, x, logits):
        """x bf16 [T][d], logits fp32 [T][E] (this rank's tokens, device) ->
        fp32 [T][d]"""
        dev = x.device
        T = x.shape[0]
        G, El, fmt = self.G, self.El, self.fmt
        g = None
        if fmt == NVFP4:
            # one activation tensor scale for all ranks (this rank's own from
            # a quantisation pass, then the largest over the ranks)
            g = shared_tensor_scale(ds4g.ds4g_quantize_mx(x, NVFP4).g.clone(), self.group)
        idx, w, xq, offsets, r2s, s2r, a = ds4g.ds4g_moe_dispatch(logits, x, self.k, fmt, g_in=g)
        S = T * self.k
        offs_h = offsets.cpu().numpy()
        sc = send_counts(offs_h, G)
        cnt = torch.from_numpy(expert_counts(offs_h)).to(dev)
        rcnt = exchange(cnt, [El] * G, [El] * G, self.group).cpu().numpy()
        rc, bounds = recv_layout(rcnt, G)
        R = int(bounds[-1])
        # the quantised rows (codes and scales) to their experts' ranks
        rd = exchange(a.data[:S], sc, rc, self.group)
        rs = exchange(a.scales[:S], sc, rc, self.group)
        recv = Fp4Tensor(rd, rs, g, fmt)
        # each received row's local expert, then the expert-contiguous order
        bnd = torch.from_numpy(bounds.astype(np.int32)).to(dev)
        ids = ds4g.ds4g_segment_ids(bnd, G * El, El, R)
        offs_l, r2s_l, s2r_l, a_l = ds4g.ds4g_moe_permute(ids.view(R, 1), El, recv)
        hq = Fp4Tensor.empty(R, self.I, fmt, dev)
        if fmt == NVFP4:
            hq.g = self.g_h
        ds4g.ds4g_grouped_gemm_fp4(a_l, offs_l, El, R, self.w1, 2 * self.I, EPI_SWIGLU_REQUANT, out_q=hq)
        y2 = ds4g.ds4g_grouped_gemm_fp4(hq, offs_l, El, R, self.w2, self.d, EPI_NONE)
        # FC2 rows back in received order, then to their source ranks
        ones = torch.ones((R, 1), dtype=torch.float32, device=dev)
        y2_recv = ds4g.ds4g_moe_combine(y2, s2r_l, ones)
        y2_back = exchange(y2_recv, rc, sc, self.group)
        return ds4g.ds4g_moe_combine(y2_back, s2r[:S], w)
