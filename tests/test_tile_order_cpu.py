"""The prefill GEMM's tile numbering (csrc/gemm_tc.cu, tile_of), restated on
the CPU and checked on random expert layouts and band widths.

prefix[e] counts the 128-row tiles of the experts before e.  Tile t lies in
band t / (U nb) (U = all row tiles, nb column tiles a band, the last band
possibly narrower); inside a band, tiles go expert by expert, then column
tile, then row tile.  Checked: every (expert, column tile, row tile) comes
exactly once; a band's tiles stay inside its columns; and within a band each
expert's tiles are consecutive, so that every expert adds into the band's
output columns before the next band starts (the order the combine epilogue
relies on to find those columns in L2)."""
import random


def _ceil_div(a, b):
    return (a + b - 1) // b


def _tile_of(t, prefix, offsets, n_tiles, nb, bm=128):
    E = len(offsets) - 1
    U = prefix[E]
    nbands = (n_tiles + nb - 1) // nb
    band = min(t // (U * nb), nbands - 1)
    nbb = min(nb, n_tiles - band * nb)
    local = t - band * U * nb
    lo, hi = 0, E - 1                 # largest e with prefix[e] * nbb <= local
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if prefix[mid] * nbb <= local:
            lo = mid
        else:
            hi = mid - 1
    beg, end = offsets[lo], offsets[lo + 1]
    mt = _ceil_div(end - beg, bm)
    le = local - prefix[lo] * nbb
    return band, lo, band * nb + le // mt, beg + (le % mt) * bm


def test_band_order_covers_every_tile_once():
    rng = random.Random(1)
    for trial in range(300):
        E = rng.randint(1, 40)
        seg = [rng.choice([0, 0, 1, 5, 127, 128, 129, 300, 1000]) for _ in range(E)]
        offsets = [0]
        for x in seg:
            offsets.append(offsets[-1] + x)
        prefix = [0]
        for x in seg:
            prefix.append(prefix[-1] + _ceil_div(x, 128))
        n_tiles = rng.randint(1, 40)
        nb = rng.randint(1, n_tiles)
        tiles = [_tile_of(t, prefix, offsets, n_tiles, nb) for t in range(prefix[E] * n_tiles)]
        expect = {(e, nt, offsets[e] + m * 128) for e in range(E) for nt in range(n_tiles)
                  for m in range(_ceil_div(seg[e], 128))}
        got = [(e, nt, m0) for _, e, nt, m0 in tiles]
        assert len(got) == len(expect) and set(got) == expect, trial
        for band, e, nt, m0 in tiles:
            assert band * nb <= nt < min(n_tiles, (band + 1) * nb), trial
            assert offsets[e] <= m0 < offsets[e + 1], trial
        # bands in order; inside a band, each expert's tiles in one run
        bands = [b for b, *_ in tiles]
        assert bands == sorted(bands), trial
        for b in set(bands):
            experts = [e for bb, e, _, _ in tiles if bb == b]
            runs = [e for i, e in enumerate(experts) if i == 0 or experts[i - 1] != e]
            assert len(runs) == len(set(runs)), trial
