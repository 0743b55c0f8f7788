"""A CPU model of the decode GEMM's ring protocol (csrc/gemv_tc.cu), run under
random interleavings, out-of-order completion of asynchronous copies and
random stalls of the MMA issuers (one pair falling behind the other, as a
wait on the epilogue or, in the one-launch FFN, on another CTA's results
makes it do).

Two producer / issuer pairs take alternate scale stages (pair sit & 1), each
producer waiting on every barrier of its scale stage before issuing its
copies.  Scale stage sit uses scale slot sit % SF_STAGES and data slots
2 sit, 2 sit + 1 (mod STAGES); one transposer takes the scale stages in
order.  A parity wait cannot tell the phase it waits for from the one two
phases earlier, so the model records an error whenever a wait starts while its
barrier is two or more phases behind (the real wait would pass early), and
whenever an issuer reads a slot holding another stage's data.

The layouts in the kernel: 6 scale slots (MXFP4) or 4 (NVFP4) with 10 data
slots, and 4 with 9 for the split NVFP4 kernel.  The negative control is the
earlier MXFP4 layout, 5 scale slots shared alternately by the pairs, where
the model must find the early pass."""
import random

import pytest


class _Bar:
    def __init__(self):
        self.done, self.arr, self.tx = 0, 0, 0

    def arrive(self, tx=0):
        self.arr += 1
        self.tx += tx
        if self.arr > 1:
            raise RuntimeError("arrival overflow")
        self._check()

    def land(self, tx):
        self.tx -= tx
        self._check()

    def _check(self):
        if self.arr == 1 and self.tx == 0:
            self.done += 1
            self.arr = 0


def _run(sf_stages, stages, nsit, seed):
    rng = random.Random(seed)
    sf_full = [_Bar() for _ in range(sf_stages)]
    sf_ready = [_Bar() for _ in range(sf_stages)]
    sf_empty = [_Bar() for _ in range(sf_stages)]
    full = [_Bar() for _ in range(stages)]
    empty = [_Bar() for _ in range(stages)]
    held_sf, held = {}, {}
    errors, async_ev, commit_q = [], [], {0: [], 1: []}

    def wait_full(b, use):
        if b.done > use + 1:
            errors.append("slot refilled before it was read")
        return b.done > use

    def wait_empty(b, use):
        if b.done < use - 1:
            errors.append("empty wait two phases behind: a parity wait passes early")
        return b.done >= use

    def slots(sit):
        r = sit % sf_stages
        d = [((2 * sit + i) % stages, (2 * sit + i) // stages) for i in (0, 1)]
        return r, sit // sf_stages, d

    def producer(p):
        for sit in range(p, nsit, 2):
            r, ru, d = slots(sit)
            # every barrier of the scale stage before any copy
            while not wait_empty(sf_empty[r], ru):
                yield
            for s, u in d:
                while not wait_empty(empty[s], u):
                    yield
            sf_full[r].arrive(1)

            def land_sf(r=r, sit=sit):
                held_sf[r] = sit
                sf_full[r].land(1)
            async_ev.append(land_sf)
            for i, (s, u) in enumerate(d):
                full[s].arrive(1)

                def land(s=s, tag=(sit, i)):
                    held[s] = tag
                    full[s].land(1)
                async_ev.append(land)
            yield

    def transposer():
        for sit in range(nsit):
            r, ru, _ = slots(sit)
            while not wait_full(sf_full[r], ru):
                yield
            sf_ready[r].arrive()
            yield

    def issuer(p):
        for sit in range(p, nsit, 2):
            r, ru, d = slots(sit)
            while not wait_full(sf_ready[r], ru):
                yield
            for s, u in d:
                while not wait_full(full[s], u):
                    yield
            if held_sf.get(r) != sit:
                errors.append(f"issuer {p} read scales of {held_sf.get(r)} for {sit}")
            for i, (s, _) in enumerate(d):
                if held.get(s) != (sit, i):
                    errors.append(f"issuer {p} read data {held.get(s)} for {(sit, i)}")
            for s, _ in d:
                commit_q[p].append(lambda s=s: empty[s].arrive())
            commit_q[p].append(lambda r=r: sf_empty[r].arrive())
            for _ in range(rng.choice([0, 0, 0, 5, 40])):   # a stall: one pair falls behind
                yield

    live = [producer(0), producer(1), transposer(), issuer(0), issuer(1)]
    steps = 0
    while live or async_ev or commit_q[0] or commit_q[1]:
        steps += 1
        if steps > 200_000:
            return "deadlock"
        u = rng.random()
        try:
            if u < 0.25 and async_ev:
                async_ev.pop(rng.randrange(len(async_ev)))()
            elif u < 0.4 and (commit_q[0] or commit_q[1]):
                commit_q[rng.choice([q for q in (0, 1) if commit_q[q]])].pop(0)()
            elif live:
                g = rng.choice(live)
                try:
                    next(g)
                except StopIteration:
                    live.remove(g)
        except RuntimeError as e:
            return str(e)
        if errors:
            return errors[0]
    return "ok"


@pytest.mark.parametrize("sf_stages,stages", [(6, 10), (4, 10), (4, 9)])
@pytest.mark.parametrize("nsit", [3, 7, 12, 30])
def test_kernel_layouts_never_alias(sf_stages, stages, nsit):
    for seed in range(40):
        assert _run(sf_stages, stages, nsit, seed) == "ok", (sf_stages, stages, nsit, seed)


def test_five_shared_scale_slots_alias():
    """negative control: the earlier 5-slot MXFP4 scale ring lets a wait pass
    early in some schedule"""
    bad = sum(_run(5, 10, nsit, seed) != "ok" for nsit in (12, 30) for seed in range(60))
    assert bad > 0
