"""One routed-expert MoE FFN layer with block-scaled FP4 expert weights,
run as the sequence of libds4g calls (route -> quantise -> permute -> FC1
with fused SwiGLU + requantisation -> FC2 with the weighted combine fused;
the unfused SwiGLU and combine steps are available as options) on one stream.

All arithmetic happens in the library's kernels; this module only owns the
device buffers and issues the calls.
"""
import torch

from . import ds4g
from .ds4g import EPI_NONE, EPI_SWIGLU_REQUANT, MXFP4, MXFP8, NVFP4, Fp4Tensor


class MoeLayer:
    def __init__(self, w1, w2, E, k, d, I, fmt, g_h=None, fused=True, fused_combine=True, fused_dispatch=True,
                 chained=True, act_fmt=None, shared=None, one_launch=True):
        """w1: Fp4Tensor [E*2I][d] (gate rows then up rows per expert),
        w2: Fp4Tensor [E*d][I]; NVFP4 weights carry one tensor scale per
        expert (w.g has E floats); g_h: the static NVFP4 tensor scale of h.
        chained: the output is zeroed before the dispatch and FC2 + combine
        is launched to overlap the end of FC1 (decode sizes).
        act_fmt: the format of the activations and of h, fmt by default;
        MXFP8 with MXFP4 weights is the FP8 x FP4 variant (its activations
        take the separate routing / quantisation / permutation calls).
        shared: (ws1 [2I_s][d], ws2 [d][I_s]) MXFP8 weights of a shared expert
        that every token also goes through (FP8 activations only); its output
        is added to the routed experts' sum with weight 1.
        one_launch: at decode sizes (at most 16 tokens, shapes the decode
        kernel tiles) FC1 + SwiGLU/requant and FC2 + combine run as one
        launch (ds4g_moe_ffn_fp4); other sizes, and one_launch=False, take
        the two calls (FC2 chained to FC1)."""
        self.w1, self.w2 = w1, w2
        self.E, self.k, self.d, self.I, self.fmt = E, k, d, I, fmt
        self.act_fmt = fmt if act_fmt is None else act_fmt
        if self.act_fmt == MXFP8 and fmt != MXFP4:
            raise ValueError("FP8 activations multiply MXFP4 weights")
        self.fused = fused or self.act_fmt == MXFP8        # h is requantised in FC1's epilogue
        self.fused_combine = fused_combine
        self.fused_dispatch = fused_dispatch and self.act_fmt != MXFP8
        self.shared = shared
        if shared is not None:
            if self.act_fmt != MXFP8 or shared[0].fmt != MXFP8 or shared[1].fmt != MXFP8:
                raise ValueError("the shared expert takes MXFP8 weights and FP8 activations")
            self.I_s = shared[0].rows // 2
        self.chained = chained and fused_combine
        self.one_launch = one_launch and self.fused and self.chained and self.act_fmt == fmt and fmt in (MXFP4, NVFP4)
        self.g_h = None
        if fmt == NVFP4:
            dev = w1.data.device
            self.g_h = torch.tensor([g_h if g_h is not None else 1.0], dtype=torch.float32, device=dev)
        self._bufs = {}

    def buffers(self, T, device):
        key = (T, str(device))
        b = self._bufs.get(key)
        if b is None:
            S = T * self.k
            b = dict(
                idx=torch.empty((T, self.k), dtype=torch.int32, device=device),
                w=torch.empty((T, self.k), dtype=torch.float32, device=device),
                xq=Fp4Tensor.empty(T, self.d, self.act_fmt, device),
                offsets=torch.empty(self.E + 1, dtype=torch.int32, device=device),
                r2s=torch.empty(max(S, 1), dtype=torch.int32, device=device),
                s2r=torch.empty(max(S, 1), dtype=torch.int32, device=device),
                a=Fp4Tensor.empty(S, self.d, self.act_fmt, device),
                hq=Fp4Tensor.empty(S, self.I, self.act_fmt, device),
                out=torch.empty((T, self.d), dtype=torch.float32, device=device),
                pws=ds4g.permute_workspace(T, self.k, self.E, device),
                dws=ds4g.dispatch_workspace(T, self.k, self.E, self.fmt, False, device),
                qws=torch.empty(16, dtype=torch.uint8, device=device),
                ctr=ds4g.ffn_counters(self.E, device),
            )
            if self.fmt == NVFP4:
                b["hq"].g = self.g_h
            if self.shared is not None:
                b["s_off"] = torch.tensor([0, T], dtype=torch.int32, device=device)
                b["s_hq"] = Fp4Tensor.empty(T, self.I_s, MXFP8, device)
                b["s_rows"] = torch.arange(max(T, 1), dtype=torch.int32, device=device)
                b["s_w"] = torch.ones((T, 1), dtype=torch.float32, device=device)
            if not self.fused:
                b["y1"] = torch.empty((S, 2 * self.I), dtype=torch.float32, device=device)
            if not self.fused_combine:
                b["y2"] = torch.empty((S, self.d), dtype=torch.float32, device=device)
            self._bufs[key] = b
        return b

    def uses_one_launch(self, T):
        """whether the FFN of a T-token step runs as one launch"""
        return self.one_launch and T <= 16 and ds4g.ffn_supported(self.fmt, self.d, self.I, self.E)

    def forward(self, x, logits, h_debug=None, out=None):
        """x: bf16 [T][d] (device), logits: fp32 [T][E] (device) -> fp32 [T][d]
        (written into `out` when given, else into the layer's own buffer)"""
        T = x.shape[0]
        b = self.buffers(T, x.device)
        self.dispatch(x, logits, b, out)
        if h_debug is None and self.uses_one_launch(T):
            return self.ffn(b, T, out)
        self.fc1(b, T, h_debug)
        return self.fc2(b, T, out)

    def ffn(self, b, T, out=None):
        """FC1 + SwiGLU/requant and FC2 + combine into out (zeroed before the
        dispatch) as one launch"""
        out = b["out"] if out is None else out
        ds4g.ds4g_moe_ffn_fp4(b["a"], b["offsets"], self.E, T, self.w1, self.w2, self.d, self.I, b["hq"], b["r2s"],
                              b["w"], out, b["ctr"])
        return out

    def dispatch(self, x, logits, b, out=None):
        """routing, activation quantisation and the expert-contiguous
        permutation (one library call; self.fused_dispatch=False issues the
        three separate calls); chained: the output is zeroed first"""
        if self.chained:
            ds4g.ds4g_zero_fill(b["out"] if out is None else out)
        if self.fused_dispatch:
            ds4g.ds4g_moe_dispatch(logits, x, self.k, self.fmt, idx=b["idx"], w=b["w"], x_q=b["xq"],
                                   offsets=b["offsets"], row_to_slot=b["r2s"], slot_to_row=b["s2r"], a_perm=b["a"],
                                   workspace=b["dws"])
            return
        ds4g.ds4g_route_topk(logits, self.k, idx=b["idx"], w=b["w"])
        ds4g.ds4g_quantize_mx(x, self.act_fmt, out=b["xq"], workspace=b["qws"])
        ds4g.ds4g_moe_permute(b["idx"], self.E, b["xq"], offsets=b["offsets"], row_to_slot=b["r2s"],
                              slot_to_row=b["s2r"], a_perm=b["a"], workspace=b["pws"])

    def fc1(self, b, T, h_debug=None):
        """grouped FC1 with SwiGLU and the FP4 requantisation of h"""
        if self.fused:
            ds4g.ds4g_grouped_gemm_fp4(b["a"], b["offsets"], self.E, T, self.w1, 2 * self.I, EPI_SWIGLU_REQUANT,
                                       out_q=b["hq"], h_debug=h_debug)
        else:
            ds4g.ds4g_grouped_gemm_fp4(b["a"], b["offsets"], self.E, T, self.w1, 2 * self.I, EPI_NONE, out=b["y1"])
            ds4g.ds4g_swiglu_requant(b["y1"], self.fmt, h_q=b["hq"], h_debug=h_debug)

    def shared_expert(self, b, T, out):
        """the shared expert on every token's FP8 activations: FC1 with the
        fused SwiGLU + FP8 requantisation, then FC2 adding each token's row
        into out (the combine epilogue with one slot per token, weight 1)"""
        ws1, ws2 = self.shared
        ds4g.ds4g_grouped_gemm_fp4(b["xq"], b["s_off"], 1, T, ws1, 2 * self.I_s, EPI_SWIGLU_REQUANT, out_q=b["s_hq"])
        ds4g.ds4g_grouped_gemm_fp4_combine_chained(b["s_hq"], b["s_off"], 1, T, ws2, self.d, b["s_rows"], b["s_w"],
                                                   out)

    def fc2(self, b, T, out=None):
        """grouped FC2 and the routing-weighted combine into out [T][d]"""
        out = b["out"] if out is None else out
        if self.chained:
            ds4g.ds4g_grouped_gemm_fp4_combine_chained(b["hq"], b["offsets"], self.E, T, self.w2, self.d, b["r2s"],
                                                       b["w"], out)
        elif self.fused_combine:
            ds4g.ds4g_grouped_gemm_fp4_combine(b["hq"], b["offsets"], self.E, T, self.w2, self.d, b["r2s"],
                                               b["w"], out=out)
        else:
            ds4g.ds4g_grouped_gemm_fp4(b["hq"], b["offsets"], self.E, T, self.w2, self.d, EPI_NONE, out=b["y2"])
            ds4g.ds4g_moe_combine(b["y2"], b["s2r"][:T * self.k], b["w"], out=out)
        if self.shared is not None:
            self.shared_expert(b, T, out)
        return out

    def _warm(self, x, logits):
        side = torch.cuda.Stream(device=x.device)
        side.wait_stream(torch.cuda.current_stream(x.device))
        with torch.cuda.stream(side):
            self.forward(x, logits)            # first call sets kernel attributes, buffers
        torch.cuda.current_stream(x.device).wait_stream(side)

    def capture(self, x, logits, out=None):
        """Records forward(x, logits) on these (static) input buffers as a CUDA
        graph; returns (graph, out).  Replaying the graph re-runs the whole
        layer on whatever x / logits hold at that time, writing `out` when
        given (else the layer's own output buffer)."""
        self._warm(x, logits)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            out = self.forward(x, logits, out=out)
        return graph, out

    def capture_stages(self, x, logits):
        """The same layer as three graphs replayed in order, so that each
        stage can be bracketed by events: dispatch, FC1, FC2 + combine;
        returns ([(name, graph), ...], out)."""
        self._warm(x, logits)
        T = x.shape[0]
        b = self.buffers(T, x.device)
        if self.uses_one_launch(T):
            names = ["dispatch", "ffn"]
            graphs = [torch.cuda.CUDAGraph() for _ in names]
            with torch.cuda.graph(graphs[0]):
                self.dispatch(x, logits, b)
            with torch.cuda.graph(graphs[1]):
                out = self.ffn(b, T)
            return list(zip(names, graphs)), out
        names = ["dispatch", "fc1_swiglu", "fc2_combine"]
        graphs = [torch.cuda.CUDAGraph() for _ in names]
        with torch.cuda.graph(graphs[0]):
            self.dispatch(x, logits, b)
        with torch.cuda.graph(graphs[1]):
            self.fc1(b, T)
        with torch.cuda.graph(graphs[2]):
            out = self.fc2(b, T)
        return list(zip(names, graphs)), out
