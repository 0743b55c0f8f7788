"""The one-launch decode FFN's item walk (csrc/gemv_tc.cu, ds4g_moe_ffn_fp4),
restated on the CPU and checked on random routings.

Items are numbered per GEMM from the expert offsets: each expert with rows
has ceil(rows / 16) row groups times its weight tiles (FC1: I / 64 tiles of 64
gate + 64 up rows; FC2: d / 128 tiles).  CTA u of U takes FC1 items
u, u + U, ... and then FC2 items (U - 1 - u), (U - 1 - u) + U, ... (the
reverse CTA order, so that CTAs with one FC1 item more take fewer FC2 items).
An FC2 item of expert e may start only once every FC1 item of e has finished,
and every CTA is resident.

Checked: every item of both GEMMs is taken exactly once; each CTA's FC1
items come before its FC2 items; and the walk cannot deadlock: CTAs advancing
in any random order, each blocked only by its next FC2 item's expert, always
finish."""
import random

import numpy as np
import pytest


def _ceil_div(a, b):
    return -(-a // b)


def _walk(U, n1, n2):
    seqs = []
    for u in range(U):
        n0 = _ceil_div(n1 - u, U) if n1 > u else 0
        seq, n = [], 0
        while True:
            if n < n0:
                seq.append((0, u + n * U))
            else:
                t = (U - 1 - u) + (n - n0) * U
                if t >= n2:
                    break
                seq.append((1, t))
            n += 1
        seqs.append(seq)
    return seqs


def _check(counts, wt1, wt2, U, rng):
    groups = [_ceil_div(c, 16) for c in counts]
    pre1 = np.concatenate([[0], np.cumsum([g * wt1 for g in groups])]).astype(int)
    pre2 = np.concatenate([[0], np.cumsum([g * wt2 for g in groups])]).astype(int)
    n1, n2 = int(pre1[-1]), int(pre2[-1])
    seqs = _walk(U, n1, n2)
    assert sorted(t for s in seqs for ph, t in s if ph == 0) == list(range(n1))
    assert sorted(t for s in seqs for ph, t in s if ph == 1) == list(range(n2))
    for s in seqs:
        phases = [ph for ph, _ in s]
        assert phases == sorted(phases)
    expert1 = np.repeat(np.arange(len(counts)), np.diff(pre1))
    expert2 = np.repeat(np.arange(len(counts)), np.diff(pre2))
    left1 = np.diff(pre1).copy()                    # FC1 items of each expert not yet done
    pos = [0] * U
    live = [u for u in range(U) if seqs[u]]
    while live:
        movable = []
        for u in live:
            ph, t = seqs[u][pos[u]]
            if ph == 0 or left1[expert2[t]] == 0:
                movable.append(u)
        assert movable, "deadlock: every CTA waits for FC1 items that no CTA will run"
        u = rng.choice(movable)
        ph, t = seqs[u][pos[u]]
        if ph == 0:
            left1[expert1[t]] -= 1
        pos[u] += 1
        if pos[u] == len(seqs[u]):
            live.remove(u)


@pytest.mark.parametrize("U", [1, 2, 3, 7, 148])
@pytest.mark.parametrize("T,E,k", [(1, 256, 6), (4, 256, 6), (8, 256, 6), (16, 8, 2), (3, 16, 2), (16, 512, 8)])
def test_every_item_once_and_no_deadlock(U, T, E, k):
    rng = random.Random(U * 1000 + T)
    nrng = np.random.default_rng(U * 1000 + T)
    for _ in range(3):
        counts = np.zeros(E, int)
        for _ in range(T):
            counts[nrng.choice(E, k, replace=False)] += 1
        _check(list(counts), 32, 56, U, rng)          # I = 2048 (32 FC1 tiles), d = 7168 (56 FC2 tiles)
