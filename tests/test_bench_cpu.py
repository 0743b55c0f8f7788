"""The bench's host side on CPU: the reference arm (the oracle timed on the
host cores) prints a contract-shaped JSON line, and the roofline's byte
accounting reproduces the per-expert weight bytes of the two formats."""
import json
import os
import subprocess
import sys
from types import SimpleNamespace

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def _wl(fmt, T=1, k=6, E=256, d=7168, I=2048):
    return SimpleNamespace(fmt=fmt, T=T, k=k, E=E, d=d, I=I, S=T * k)


def test_byte_accounting_per_expert():
    """one touched expert with one row: FC1 reads that expert's packed W1 and
    its scales once, plus the row in and h out; the layer adds W2"""
    d, I = 7168, 2048
    offsets = np.zeros(257, np.int32)
    offsets[4:] = 1                                # expert 3 holds the only row
    wl = _wl(0, T=1, k=1)
    a = bench.algorithmic(wl, offsets)
    act = (d // 2 + d // 32) + (I // 2 + I // 32)  # the row of a (FC1 input) and of h (FC1 output)
    assert a["touched"] == 1 and a["max_rows"] == 1
    assert a["fc1_bytes"] - act == 15_597_568      # 2I x (d/2 + d/32): packed E2M1 + UE8M0 per 32
    assert a["fc1_flops"] == 2.0 * 1 * 2 * I * d
    assert a["layer_flops"] == a["fc1_flops"] + 2.0 * 1 * d * I
    wn = _wl(1, T=1, k=1)
    n = bench.algorithmic(wn, offsets)
    act_n = (d // 2 + d // 16) + (I // 2 + I // 16)
    w2_n = d * (I // 2 + I // 16)
    assert (n["fc1_bytes"] - act_n) + w2_n == 24_772_608   # NVFP4: UE4M3 per 16, W1 + W2 of one expert


def test_reference_arm_dense_gemm():
    """--workload dense_m1: the oracle's quantisation + GEMM, reported as time
    per call (lower is better)"""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "dense_m1", "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "us" and d["higher_is_better"] is False and d["value"] > 0
    assert d["config"]["workload"].startswith("dense FP4 GEMM M=1 N=4096 K=7168")


def test_default_workload_is_the_largest_layer():
    """with no flags the bench times the largest configuration, prefill
    T = 16384 NVFP4"""
    import argparse
    old = sys.argv
    sys.argv = ["bench.py"]
    try:
        a = bench.parse()
    finally:
        sys.argv = old
    assert a.workload == "prefill16k" and a.steps is None and a.warmup >= 3
    from synth import workloads
    wl = workloads.WORKLOADS[a.workload]
    assert (wl.T, wl.fmt) == (16384, 1)


def test_prefill16k_traffic_is_the_scaled_stand_in_capture():
    """roofline.traffic of the default run = the DRAM bytes ncu counted for one
    FC1 launch of the current kernel on the 64-expert stand-in (963,205,376
    read + 27,490,560 written) scaled by the two launches' algorithmic bytes,
    each from its own routing (here the oracle's, which the GPU's routing
    matches bit for bit)"""
    import oracle
    import synth
    from synth import workloads
    alg = {}
    for name in ("prof_prefill16k", "prefill16k"):
        wl = workloads.WORKLOADS[name]
        idx, _ = oracle.route_topk(synth.logits(wl.T, wl.E, 0, wl.bias_sigma), wl.k)
        offsets = np.concatenate([[0], np.cumsum(np.bincount(idx.ravel(), minlength=wl.E))]).astype(np.int32)
        alg[name] = bench.algorithmic(wl, offsets)
    assert alg["prof_prefill16k"]["touched"] == 51 and alg["prefill16k"]["touched"] == 172
    assert alg["prof_prefill16k"]["fc1_bytes"] == 969_670_656 and alg["prefill16k"]["fc1_bytes"] == 3_350_200_320
    measured = 963_205_376 + 27_490_560
    scaled = round(measured * alg["prefill16k"]["fc1_bytes"] / alg["prof_prefill16k"]["fc1_bytes"])
    assert bench.FC1_TRAFFIC["prefill16k"][0] == scaled
