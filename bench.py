"""Benchmark of one routed-expert MoE FFN layer with block-scaled FP4 expert
weights on B200 (sm_100a), through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole layer (route -> quantise -> permute -> FC1 + SwiGLU +
requantise -> FC2 + weighted combine) over one batch of T synthetic tokens.
Default workload: the largest layer, prefill T = 16384 (E = 256, top-6,
d = 7168, I = 2048, NVFP4, skewed router bias).  Without --steps the number
of timed steps is chosen so that the timed region lasts about a second.
Under torchrun every rank runs its own replica on its own GPU (independent
token shards, no data-path collective; weak scaling); the timed region is
bracketed by barriers and reported as the max over ranks.  Prints one JSON
line (rank 0).

--workload dense_m1 / dense_m64 times the single dense FP4 GEMM of that size
(M = 1 / 64, N = 4096, K = 7168, MXFP4: activation quantisation + GEMM per
call) instead of a layer, with consecutive calls cycling through enough
weight copies that none finds its weights in L2.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

L2_BYTES = 126 * 1000 * 1000
# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu
# capture of the kernel as it is now; workloads without one report null.
# prefill16k: the 64-expert stand-in's FC1 launch (990.7 MB against 969.7 MB
# algorithmic, 1.022x) scaled to the full launch by its algorithmic bytes
# (3350.2 MB).  prefill: its full-size capture (1.033x) predates the prefill
# GEMM's second scale transposer, so it reports null.
FC1_TRAFFIC = {"prefill16k": (3422842407, "profiles/k_gemm_tc_fc1_prof_prefill16k_nvfp4.md (stand-in, scaled)"),
               "prefill": (None, "none of the current kernel; profiles/dram_traffic_k_gemm_tc_prefill_T2048_mxfp4.md "
                                 "(1.033x, the kernel before its second scale transposer)"),
               # the one-launch decode FFN: the decode stand-in's traffic ratio (1.00882) x the algorithmic bytes
               "decode_t8": (1039043879, "profiles/k_gemv_tc_ffn_prof_decode_t8_mxfp4.md (stand-in ratio, scaled)"),
               "decode_t4": (566727518, "profiles/k_gemv_tc_ffn_prof_decode_t8_mxfp4.md (stand-in ratio, scaled)"),
               "decode_t1": (141681879, "profiles/k_gemv_tc_ffn_prof_decode_t8_mxfp4.md (stand-in ratio, scaled)")}

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default: about 1 s of steps)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill16k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    return ap.parse_args()


def workload_desc(wl):
    fmt = "MXFP4" if wl.fmt == 0 else "NVFP4"
    if getattr(wl, "afmt", wl.fmt) == 2:
        fmt = "MXFP8 activations x MXFP4 weights"
    if wl.dense:
        return f"dense FP4 GEMM M={wl.T} N={wl.I} K={wl.d} {fmt}"
    bias = f", router bias N(0,{wl.bias_sigma})" if wl.bias_sigma else ""
    return f"MoE layer T={wl.T} E={wl.E} top-{wl.k} d={wl.d} I={wl.I} {fmt}{bias}"


# ---------------------------------------------------------------------------
# synthetic expert weights on the device (bench, tests and the smoke check)
# ---------------------------------------------------------------------------
def synthetic_weights(E, d, I, fmt, seed=0, device="cuda", rows_w1=None, chunk=8, e0=0):
    """Expert weights drawn on the device by the seeded generator
    (W1[e] ~ N(0, 0.02) [2I][d], W2[e] ~ N(0, 0.02) [d][I]) and quantised
    with the library's own quantiser, offline (not part of a step).  NVFP4
    weights get one tensor scale per expert.  Experts e0 .. e0 + E - 1 of the
    model (an expert-parallel rank's share).  Returns (w1, w2) Fp4Tensors."""
    import torch
    import synth
    from synth.workloads import W_SIGMA
    from block_scaled_fp4_topk_b200 import ds4g
    from block_scaled_fp4_topk_b200.ds4g import NVFP4, Fp4Tensor
    r1 = rows_w1 if rows_w1 is not None else 2 * I
    st = torch.cuda.current_stream().cuda_stream
    w1 = Fp4Tensor.empty(E * r1, d, fmt, device)
    w2 = Fp4Tensor.empty(E * d, I, fmt, device)
    if fmt == NVFP4:
        w1.g = torch.empty(E, dtype=torch.float32, device=device)
        w2.g = torch.empty(E, dtype=torch.float32, device=device)
    ws = torch.empty(16, dtype=torch.uint8, device=device)
    for dst, rows, cols, base in ((w1, r1, d, synth.STREAM_W1), (w2, d, I, synth.STREAM_W2)):
        buf = torch.empty((chunk * rows, cols), dtype=torch.float32, device=device)
        for c0 in range(0, E, chunk):
            n = min(chunk, E - c0)
            for j in range(n):
                synth.cuda_fill_normal_f32(buf[j * rows:(j + 1) * rows].data_ptr(), rows * cols, seed,
                                           base + e0 + c0 + j, W_SIGMA, 0, st)
            if fmt == NVFP4:
                for j in range(n):
                    e = c0 + j
                    part = Fp4Tensor(dst.data[e * rows:(e + 1) * rows], dst.scales[e * rows:(e + 1) * rows],
                                     dst.g[e:e + 1], fmt)
                    ds4g.ds4g_quantize_mx(buf[j * rows:(j + 1) * rows], fmt, out=part, workspace=ws)
            else:
                part = dst.view_rows(c0 * rows, (c0 + n) * rows)
                ds4g.ds4g_quantize_mx(buf[:n * rows], fmt, out=part)
        del buf
    return w1, w2


def synthetic_shared_weights(d, I, seed=0, device="cuda"):
    """The shared expert's weights drawn on the device by the seeded generator
    (FC1 [2I][d], FC2 [d][I], ~ N(0, 0.02)) and quantised by the library to
    MXFP8 (E4M3 + UE8M0 per 32).  Returns (ws1, ws2) Fp4Tensors."""
    import torch
    import synth
    from synth.workloads import W_SIGMA
    from block_scaled_fp4_topk_b200 import ds4g
    st = torch.cuda.current_stream().cuda_stream
    out = []
    for rows, cols, stream in ((2 * I, d, synth.STREAM_WS1), (d, I, synth.STREAM_WS2)):
        buf = torch.empty((rows, cols), dtype=torch.float32, device=device)
        synth.cuda_fill_normal_f32(buf.data_ptr(), rows * cols, seed, stream, W_SIGMA, 0, st)
        out.append(ds4g.ds4g_quantize_mx(buf, ds4g.MXFP8))
        del buf
    return tuple(out)


# ---------------------------------------------------------------------------
# oracle timing on the host cores (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------
_WCACHE = {}


def oracle_sample(wl, ntok, seed=0):
    """Times the oracle on the first `ntok` tokens of the workload: routing,
    quantisation, permutation, FC1, SwiGLU, requantisation, FC2 and combine,
    over the experts those tokens touch (weights quantised beforehand, not
    timed).  Returns (seconds, tokens)."""
    import oracle
    import synth
    from synth import workloads
    lg = workloads.host_logits(wl, seed)[:ntok]
    xb = workloads.host_x_bits(wl, seed)[:ntok]
    x = synth.bf16_bits_to_f32(xb)
    idx, _ = oracle.route_topk(lg, wl.k)
    touched = np.unique(idx)
    remap = np.full(wl.E, -1, np.int64)
    remap[touched] = np.arange(len(touched))
    fmt = wl.fmt
    w1s, w2s = [], []
    for e in touched:
        key = (wl.name, int(e), seed)
        if key not in _WCACHE:
            _WCACHE[key] = (oracle.quantize(workloads.host_w1(wl, int(e), seed), fmt),
                            oracle.quantize(workloads.host_w2(wl, int(e), seed), fmt))
        w1s.append(_WCACHE[key][0])
        w2s.append(_WCACHE[key][1])
    g_h = workloads.G_H if fmt == oracle.NV else None
    afmt = wl.afmt                  # the activations' (and h's) format
    t0 = time.perf_counter()
    idx, w = oracle.route_topk(lg, wl.k)
    cidx = remap[idx].astype(np.int32)
    E2 = len(touched)
    xq = oracle.quantize(x, afmt)
    offsets, r2s, s2r = oracle.moe_permute(cidx, E2)
    a = oracle.gather_rows(xq, r2s, wl.k)
    y1 = np.empty((a.data.shape[0], 2 * wl.I))
    for j in range(E2):
        r0, r1 = offsets[j], offsets[j + 1]
        if r1 > r0:
            y1[r0:r1], _ = oracle.expert_gemm_rows(a, np.arange(r0, r1), w1s[j], (0, 2 * wl.I))
    h = oracle.swiglu(y1.astype(np.float32))
    hq = oracle.quantize(h, afmt, g=g_h)
    y2 = np.empty((a.data.shape[0], wl.d))
    for j in range(E2):
        r0, r1 = offsets[j], offsets[j + 1]
        if r1 > r0:
            y2[r0:r1], _ = oracle.expert_gemm_rows(hq, np.arange(r0, r1), w2s[j], (0, wl.d))
    oracle.moe_combine(y2.astype(np.float32).astype(np.float64), s2r, w)
    return time.perf_counter() - t0, ntok


def cpu_cores():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)


def cpu_baseline(wl, budget_s):
    # grow the token sample until one run takes a meaningful share of the budget
    ntok, dt = 1, 0.0
    while True:
        dt, n = oracle_sample(wl, ntok)
        if dt > budget_s / 4 or ntok >= wl.T:
            break
        ntok = min(wl.T, max(ntok * 2, int(ntok * budget_s / 4 / max(dt, 1e-3))))
    return {"value": n / dt, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"first {n} of {wl.T} tokens of the same workload (full layer over the experts they touch; "
                      f"weights quantised beforehand, untimed), {dt:.2f} s"}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                if out:
                    self.samples.append([v.strip() for v in out.split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        smax = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for s in self.samples:
            for i, nm in enumerate(names):
                if len(s) > 5 + i and s[5 + i].lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
def algorithmic(wl, offsets):
    """bytes and flops of one layer and of its FC1 call, from the routing"""
    counts = np.diff(offsets)
    touched = int((counts > 0).sum())
    S = wl.S
    blk = 32 if wl.fmt == 0 else 16
    wrow1 = wl.d // 2 + wl.d // blk           # packed bytes + scale bytes of one K=d weight row
    wrow2 = wl.I // 2 + wl.I // blk
    fp8 = getattr(wl, "afmt", wl.fmt) == 2    # FP8 activations: one byte per element, UE8M0 per 32
    row1 = wl.d + wl.d // 32 if fp8 else wrow1   # one activation row (K = d) and one h row (K = I)
    row2 = wl.I + wl.I // 32 if fp8 else wrow2
    w1_bytes = touched * 2 * wl.I * wrow1
    w2_bytes = touched * wl.d * wrow2
    fc1_bytes = w1_bytes + S * row1 + S * row2
    fc1_flops = 2.0 * S * 2 * wl.I * wl.d
    fc2_flops = 2.0 * S * wl.d * wl.I
    # the one-launch decode FFN: FC1's bytes, then W2, h and the output rows
    # (zeroed before the dispatch, the sums added into them)
    ffn_bytes = fc1_bytes + w2_bytes + S * row2 + wl.T * wl.d * 4
    # route (logits), quantise (x -> xq), permute (xq rows -> a), FC1 (a, W1
    # -> hq), FC2 + combine (hq, W2 -> out, zeroed then accumulated)
    layer_bytes = (wl.T * wl.E * 4 + wl.T * wl.d * 2 + wl.T * row1 + 2 * S * row1 + fc1_bytes
                   + w2_bytes + S * row2 + 2 * wl.T * wl.d * 4)
    return dict(touched=touched, fc1_bytes=fc1_bytes, fc1_flops=fc1_flops, ffn_bytes=ffn_bytes,
                ffn_flops=fc1_flops + fc2_flops, layer_flops=fc1_flops + fc2_flops,
                layer_bytes=layer_bytes, working_set=layer_bytes, max_rows=int(counts.max()))


def max_over_ranks(ms, world, device):
    """the slowest rank's elapsed time (barrier-bracketed regions)"""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tokens_per_s(T, steps, ms, world):
    """whole-job throughput: every rank processed T tokens per step"""
    return world * T * steps / (ms / 1e3)


TIMED_SECONDS = 1.0


def calibrate_steps(step, st, world, device, lo=20, hi=20000):
    """number of steps that fill about TIMED_SECONDS, from a few timed steps
    after the warm-up (the slowest rank's estimate, so all ranks agree)"""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 4
    e0.record(st)
    for i in range(n):
        step(i)
    e1.record(st)
    torch.cuda.synchronize()
    per = max_over_ranks(e0.elapsed_time(e1) / n, world, device) / 1e3
    return int(min(hi, max(lo, round(TIMED_SECONDS / max(per, 1e-9)))))


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from synth import workloads
    import synth
    from block_scaled_fp4_topk_b200 import ds4g
    from block_scaled_fp4_topk_b200.layer import MoeLayer

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workloads.WORKLOADS[args.workload]
    if wl.dense:
        return run_dense(args, rank, world, dev, wl)
    st = torch.cuda.current_stream()
    w1, w2 = synthetic_weights(wl.E, wl.d, wl.I, wl.fmt, device=dev)
    layer = MoeLayer(w1, w2, wl.E, wl.k, wl.d, wl.I, wl.fmt, g_h=workloads.G_H, act_fmt=wl.afmt)
    one = layer.uses_one_launch(wl.T)
    # inputs resident in HBM (bf16 activations, fp32 logits), each rank its own token shard
    x = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device=dev)
    lg = torch.empty((wl.T, wl.E), dtype=torch.float32, device=dev)
    seed = rank
    synth.cuda_fill_normal_bf16(x.data_ptr(), x.numel(), seed, synth.STREAM_X, 1.0, 0, st.cuda_stream)
    synth.cuda_fill_logits(lg.data_ptr(), wl.T, wl.E, seed, wl.bias_sigma, st.cuda_stream)
    torch.cuda.synchronize()

    # the layer step as one CUDA graph (all its library calls, no host work)
    graph, gout = layer.capture(x, lg)
    b = layer.buffers(wl.T, dev)
    torch.cuda.synchronize()
    ds4g.ds4g_check_device()
    offsets = b["offsets"].cpu().numpy()
    alg = algorithmic(wl, offsets)
    # dispatch: one kernel up to 512 slots, else routing, counts, scan, ranks
    # and quantise-and-scatter (NVFP4: amax and g before them); then FC1 +
    # SwiGLU/requant and FC2 + combine
    if wl.afmt == 2:      # FP8 activations: routing, quantisation, permutation (1 or 4 kernels) as separate calls
        launches_per_step = 2 + (1 if wl.S <= 512 else 4) + 2
    else:
        launches_per_step = (1 if wl.S <= 512 else (5 if wl.fmt == 0 else 7)) + (1 if one else 2)
    # A step whose working set is under 3x L2 (decode) would find its weights
    # in L2 when the same layer ran just before.  Consecutive steps then run
    # R layers of the same shape with their own weights, as consecutive
    # layers of a model do, so that a weight is touched again only after
    # R x the working set (> 3x L2).  R is even: replica r uses the e2e
    # buffer pair r & 1 below.
    R = 1
    if alg["working_set"] < 3 * L2_BYTES:
        R = -(-3 * L2_BYTES // alg["working_set"]) + 1
        R += R & 1
    layers, graphs, gouts = [layer], [graph], [gout]
    for r in range(1, R):
        w1r, w2r = synthetic_weights(wl.E, wl.d, wl.I, wl.fmt, seed=r, device=dev)
        layers.append(MoeLayer(w1r, w2r, wl.E, wl.k, wl.d, wl.I, wl.fmt, g_h=workloads.G_H, act_fmt=wl.afmt))
        gr, go = layers[r].capture(x, lg)
        graphs.append(gr)
        gouts.append(go)
    # and as three graphs (dispatch, FC1, FC2 + combine) so that FC1, the
    # dominant kernel, can be bracketed by CUDA events on its stream
    stages = [lr.capture_stages(x, lg)[0] for lr in layers]
    for _ in range(args.warmup):
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    ds4g.ds4g_check_device()
    if args.steps is None:
        args.steps = calibrate_steps(lambda i: graphs[i % R].replay(), st, world, dev)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                      int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for i in range(args.steps):
            graphs[i % R].replay()
        e1.record(st)
        torch.cuda.synchronize()
        ms_total = e0.elapsed_time(e1)
    if world > 1:
        dist.barrier()
    ds4g.ds4g_check_device()
    ms_total = max_over_ranks(ms_total, world, dev)

    # FC1, the dominant kernel, timed over the same number of whole steps:
    # the layer replayed as its stage graphs (dispatch, FC1, FC2 + combine)
    # with events on the launching stream between them
    names = [n for n, _ in stages[0]]
    ns = len(names)
    st_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(ns + 1)] for _ in range(args.steps)]
    for i in range(args.steps):
        st_ev[i][0].record(st)
        for g in range(ns):
            stages[i % R][g][1].replay()
            st_ev[i][g + 1].record(st)
    torch.cuda.synchronize()
    ds4g.ds4g_check_device()
    stage_ms = {names[g]: float(np.mean([ev[g].elapsed_time(ev[g + 1]) for ev in st_ev])) for g in range(ns)}
    # the dominant kernel: FC1, or the one-launch FFN at decode sizes
    fc1_ms = stage_ms["ffn"] if one else stage_ms["fc1_swiglu"]

    # end to end through the public API: every step copies its inputs from
    # pinned host memory to the device, runs the layer and copies its result
    # back to pinned host memory.  The copies run on their own streams (one
    # per direction) against two sets of device inputs and outputs, so that
    # step i's result read-back and step i+1's input upload overlap step i's
    # and i+1's compute, as a serving loop would run them.
    xh = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, pin_memory=True)
    lh = torch.empty((wl.T, wl.E), dtype=torch.float32, pin_memory=True)
    xh.copy_(x)
    lh.copy_(lg)
    oh = [torch.empty((wl.T, wl.d), dtype=torch.float32, pin_memory=True) for _ in range(2)]
    xs = [x, x.clone()]
    lgs = [lg, lg.clone()]
    outs = [torch.empty((wl.T, wl.d), dtype=torch.float32, device=dev) for _ in range(2)]
    egraphs = [[lr.capture(xs[s], lgs[s], out=outs[s])[0] for s in range(2)] for lr in layers]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()                                       # noqa: E731
    h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_step(i):
        s = i & 1
        with torch.cuda.stream(up):
            up.wait_event(comp_done[s])            # step i-2 has read xs[s], lgs[s]
            xs[s].copy_(xh, non_blocking=True)
            lgs[s].copy_(lh, non_blocking=True)
            h2d_done[s].record(up)
        st.wait_event(h2d_done[s])
        st.wait_event(d2h_done[s])                 # step i-2's result has left outs[s]
        egraphs[i % R][s].replay()
        comp_done[s].record(st)
        with torch.cuda.stream(down):
            down.wait_event(comp_done[s])
            oh[s].copy_(outs[s], non_blocking=True)
            d2h_done[s].record(down)

    for s in range(2):
        comp_done[s].record(st)
        d2h_done[s].record(st)
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(st)
    up.wait_event(a0)
    down.wait_event(a0)
    for i in range(args.steps):
        e2e_step(i)
    st.wait_event(d2h_done[(args.steps - 1) & 1])
    st.wait_event(d2h_done[args.steps & 1])
    a1.record(st)
    torch.cuda.synchronize()
    e2e_ms = a0.elapsed_time(a1)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    # the result read back in the last step is that step's layer output
    last_r = (args.steps - 1) % R
    graphs[last_r].replay()
    ref = gouts[last_r].cpu()
    last = oh[(args.steps - 1) & 1]
    if not torch.allclose(last, ref, rtol=1e-5, atol=1e-5 * float(ref.abs().max())):
        raise RuntimeError("end-to-end read-back differs from the layer's output")
    del egraphs

    if rank != 0:
        return None
    import json as _json
    peaks = {}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk_path):
        peaks = _json.load(open(pk_path))
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    bf16_peak = peaks.get("bf16_tflops", 1590.0)
    # dense FP4 : FP8 : bf16 = 9 : 4.5 : 2.25 PFLOP/s (nominal ratios); the
    # FP8 x FP4 MMA (kind::mxf8f6f4) runs at the FP8 rate
    fp4_peak = bf16_peak * (2.0 if wl.afmt == 2 else 4.0)
    kbytes = alg["ffn_bytes"] if one else alg["fc1_bytes"]
    kflops = alg["ffn_flops"] if one else alg["fc1_flops"]
    t_hbm = kbytes / (hbm_peak * 1e9)
    t_tc = kflops / (fp4_peak * 1e12)
    fc1_s = fc1_ms / 1e3
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": kbytes / fc1_s / 1e9, "peak": hbm_peak, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": kflops / fc1_s / 1e12, "peak": fp4_peak, "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = None
    roof["kernel"] = ("FC1 + SwiGLU/requant + FC2 + combine in one launch, decode tensor-core kernel (weights as "
                      "MMA M, <= 16 tokens as N)" if one else
                      "FC1 + fused SwiGLU/requant, decode tensor-core kernel (weights as MMA M, <= 16 tokens as N)"
                      if alg["max_rows"] <= 16 else
                      "FC1 + fused SwiGLU/requant, tcgen05 grouped GEMM (128 x 192 tiles, two MMA issuers)")
    roof["peak_source"] = ("measured (MEASURED_PEAKS.json" +
                           (("; FP8 = bf16 burst x 2" if wl.afmt == 2 else "; FP4 = bf16 burst x 4") +
                            " nominal ratio" if roof["bound"] == "tensor" else "") + ")") if peaks else "fallback"
    if args.workload in FC1_TRAFFIC:
        roof["traffic"] = FC1_TRAFFIC[args.workload][0]
        roof["traffic_source"] = FC1_TRAFFIC[args.workload][1]
    roof["kernel_ms"] = fc1_ms
    if not one:
        roof["fc1_ms"] = fc1_ms
        roof["fc1_tflops"] = alg["fc1_flops"] / fc1_s / 1e12
        roof["fc1_gbs"] = alg["fc1_bytes"] / fc1_s / 1e9
    roof["algorithmic_bytes"] = kbytes
    roof["algorithmic_flops"] = kflops

    ms_step = ms_total / args.steps
    value = tokens_per_s(wl.T, args.steps, ms_total, world)
    e2e_value = tokens_per_s(wl.T, args.steps, e2e_ms, world)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ("mxfp8 x mxfp4" if wl.afmt == 2 else "mxfp4" if wl.fmt == 0 else "nvfp4"),
        "data": "synthetic",
        "config": {"workload": workload_desc(wl), "tokens_per_gpu": wl.T, "experts_touched": alg["touched"],
                   "max_rows_per_expert": alg["max_rows"], "parallelism": f"replicas x{world} (token shards)",
                   "l2": (f"no flush: consecutive steps cycle through {R} layers of this shape with their own "
                          f"weights (working set ~{alg['working_set'] / 1e9:.3f} GB each), so a weight is "
                          f"touched again only after {R * alg['working_set'] / 1e9:.2f} GB > 3x the 126 MB L2"
                          if R > 1 else
                          f"no flush: the step's working set (~{alg['working_set'] / 1e9:.2f} GB) exceeds 3x "
                          f"the 126 MB L2"), "layers_cycled": R,
                   "layer_tflops": alg["layer_flops"] / (ms_step / 1e3) / 1e12},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": wl.T * wl.d * 2 + wl.T * wl.E * 4,
                "d2h_bytes_per_step": wl.T * wl.d * 4,
                "mode": "pinned host in/out every step; copies on two copy streams overlap the neighbouring "
                        "steps' compute (double-buffered device inputs/outputs)"},
        "gpu_launches": launches_per_step * args.steps,
        "step_mode": "CUDA graph of the layer's library calls",
        "stage_ms": dict(stage_ms, note="each stage as its own graph, events between them"),
        "clocks": clk.summary(),
    }
    return line


def load_peaks():
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    return json.load(open(pk_path)) if os.path.exists(pk_path) else {}


def gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    return int(vis.split(",")[local_rank]) if vis else local_rank


def dense_weight(N, K, fmt, seed, device):
    """one N x K weight matrix ~ N(0, 0.02) from the seeded generator (the
    workload's W1 stream of expert 0), quantised by the library"""
    import torch
    import synth
    from synth.workloads import W_SIGMA
    from block_scaled_fp4_topk_b200 import ds4g
    buf = torch.empty((N, K), dtype=torch.float32, device=device)
    synth.cuda_fill_normal_f32(buf.data_ptr(), N * K, seed, synth.STREAM_W1, W_SIGMA, 0,
                               torch.cuda.current_stream().cuda_stream)
    w = ds4g.ds4g_quantize_mx(buf, fmt)
    del buf
    return w


def oracle_dense_sample(wl, budget_s):
    """the oracle's quantisation + GEMM of the first m activation rows against
    the full weight matrix; m grows until a run takes a share of the budget"""
    import oracle
    import synth
    from synth import workloads
    M, N, K = wl.T, wl.I, wl.d
    W = oracle.quantize(workloads.host_w1(wl, 0), wl.fmt)
    x = synth.bf16_bits_to_f32(workloads.host_x_bits(wl))
    m = 1
    while True:
        t0 = time.perf_counter()
        xq = oracle.quantize(x[:m], wl.fmt)
        oracle.expert_gemm_rows(xq, np.arange(m), W, (0, N))
        dt = time.perf_counter() - t0
        if dt > budget_s / 4 or m >= M:
            return dt, m
        m = min(M, m * 2)


def run_dense(args, rank, world, dev, wl):
    """One dense FP4 GEMM call per step (the pages' single-GEMM shape): MX
    quantisation of the M bf16 activation rows and the GEMM against one
    N x K weight matrix (one expert, offsets [0, M]), fp32 out, all through
    the C ABI.  Consecutive steps cycle through R weight copies whose total is
    more than 3x L2, so no call finds its weights in L2."""
    import torch
    import synth
    from block_scaled_fp4_topk_b200 import ds4g
    M, N, K = wl.T, wl.I, wl.d
    blk = 32 if wl.fmt == 0 else 16
    st = torch.cuda.current_stream()
    wbytes = N * (K // 2 + K // blk)
    R = -(-3 * L2_BYTES // wbytes) + 1
    ws = [dense_weight(N, K, wl.fmt, r, dev) for r in range(R)]
    x = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    synth.cuda_fill_normal_bf16(x.data_ptr(), x.numel(), rank, synth.STREAM_X, 1.0, 0, st.cuda_stream)
    xq = ds4g.Fp4Tensor.empty(M, K, wl.fmt, dev)
    qws = torch.empty(16, dtype=torch.uint8, device=dev)
    offs = torch.tensor([0, M], dtype=torch.int32, device=dev)
    out = torch.empty((M, N), dtype=torch.float32, device=dev)

    def call(w):
        ds4g.ds4g_quantize_mx(x, wl.fmt, out=xq, workspace=qws)
        ds4g.ds4g_grouped_gemm_fp4(xq, offs, 1, M, w, N, ds4g.EPI_NONE, out=out)

    call(ws[0])
    torch.cuda.synchronize()
    ds4g.ds4g_check_device()
    graphs, qgraphs, ggraphs = [], [], []
    for w in ws:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(w)
        graphs.append(g)
        gq, gg = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gq):
            ds4g.ds4g_quantize_mx(x, wl.fmt, out=xq, workspace=qws)
        with torch.cuda.graph(gg):
            ds4g.ds4g_grouped_gemm_fp4(xq, offs, 1, M, w, N, ds4g.EPI_NONE, out=out)
        qgraphs.append(gq)
        ggraphs.append(gg)
    for i in range(max(args.warmup, R)):
        graphs[i % R].replay()
    torch.cuda.synchronize()
    if args.steps is None:
        args.steps = calibrate_steps(lambda i: graphs[i % R].replay(), st, world, dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_index(dev.index)) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for i in range(args.steps):
            graphs[i % R].replay()
        e1.record(st)
        torch.cuda.synchronize()
        ms_total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ds4g.ds4g_check_device()
    # the GEMM alone, bracketed by events on its stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for i in range(args.steps):
        evs[i][0].record(st)
        qgraphs[i % R].replay()
        evs[i][1].record(st)
        ggraphs[i % R].replay()
        evs[i][2].record(st)
    torch.cuda.synchronize()
    gemm_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    quant_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    # end to end: the activations from pinned host memory and the result back
    # to pinned host memory in every call
    xh = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
    xh.copy_(x)
    oh = torch.empty((M, N), dtype=torch.float32, pin_memory=True)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(st)
    for i in range(args.steps):
        x.copy_(xh, non_blocking=True)
        graphs[i % R].replay()
        oh.copy_(out, non_blocking=True)
    a1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), world, dev)
    if rank != 0:
        return None
    peaks = load_peaks()
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    gbytes = wbytes + M * (K // 2 + K // blk) + M * N * 4
    flops = 2.0 * M * N * K
    us = 1e3 * ms_total / args.steps
    roof = {"bound": "hbm", "achieved": gbytes / (gemm_ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
            "traffic": None, "algorithmic_bytes": gbytes, "gemm_us": 1e3 * gemm_ms, "quantize_us": 1e3 * quant_ms,
            "gemm_tflops": flops / (gemm_ms / 1e3) / 1e12,
            "kernel": ("decode tensor-core GEMM (weights as MMA M)" if M <= 16 else
                       "tcgen05 grouped GEMM (128 x 256 tiles)"),
            "peak_source": "measured (MEASURED_PEAKS.json)" if peaks else "fallback"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    return {
        "metric": "dense FP4 GEMM time per call", "value": us, "unit": "us", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "mxfp4",
        "data": "synthetic", "config": {"workload": workload_desc(wl), "M": M, "N": N, "K": K,
                                        "l2": f"no flush: consecutive calls cycle through {R} weight copies "
                                              f"({R * wbytes / 1e9:.2f} GB > 3x the 126 MB L2)"},
        "roofline": roof,
        "e2e": {"value": 1e3 * e2e_ms / args.steps, "unit": "us", "h2d_bytes_per_step": M * K * 2,
                "d2h_bytes_per_step": M * N * 4, "mode": "pinned host in/out every call, in stream order"},
        "gpu_launches": 2 * args.steps, "clocks": clk.summary(),
        "context": "the Triton FP4 page quotes 6.4 ms per FP4 MoE GEMM call on DGX Spark (sm_121): other "
                   "hardware and another call, not a target",
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from synth import workloads
    wl = workloads.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return 0
        if args.steps is None:
            args.steps = 10
        if wl.dense:
            # each step: the oracle's quantisation + GEMM of 2 activation rows,
            # reported as time per call of the full M rows
            import oracle
            import synth
            from synth import workloads as _w
            W = oracle.quantize(_w.host_w1(wl, 0), wl.fmt)
            x = synth.bf16_bits_to_f32(_w.host_x_bits(wl))
            m = min(2, wl.T)
            tot_t = 0.0
            for i in range(args.warmup + args.steps):
                t0 = time.perf_counter()
                oracle.expert_gemm_rows(oracle.quantize(x[:m], wl.fmt), np.arange(m), W, (0, wl.I))
                if i >= args.warmup:
                    tot_t += time.perf_counter() - t0
            v = 1e6 * tot_t / args.steps / m * wl.T
            print(json.dumps({
                "impl": "reference", "metric": "dense FP4 GEMM time per call", "value": v, "unit": "us",
                "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": workload_desc(wl)},
                "cpu_baseline": {"value": v, "unit": "us", "cores": cpu_cores(), "kind": "oracle",
                                 "sample": f"each step: {m} of the {wl.T} rows, scaled to {wl.T} rows"},
                "e2e": {"value": v, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            }), flush=True)
            return 0
        for _ in range(args.warmup):
            oracle_sample(wl, 1)
        tot_t, tot_n = 0.0, 0
        ntok = 2 if wl.T >= 2 else 1
        for _ in range(args.steps):
            dt, n = oracle_sample(wl, ntok)
            tot_t += dt
            tot_n += n
        v = tot_n / tot_t
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl)},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": f"each step: the first {ntok} tokens of the workload (full layer over the "
                                       f"experts they touch)"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    line = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if not args.no_cpu_baseline:
            if wl.dense:
                dt, m = oracle_dense_sample(wl, args.cpu_budget_s)
                line["cpu_baseline"] = {"value": 1e6 * dt / m * wl.T, "unit": "us", "cores": cpu_cores(),
                                        "kind": "oracle",
                                        "sample": f"quantisation + GEMM of the first {m} of {wl.T} rows against "
                                                  f"the full weight matrix, {dt:.2f} s, scaled to {wl.T} rows"}
            else:
                line["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget_s)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
