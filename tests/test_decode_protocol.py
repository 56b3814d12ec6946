"""The fused decode step's hand-off from scan to gather, on the CPU.

select_stream_kernel<D, S> with S > 0 (landmark_guided_chunk_b200/csrc/select_stream.cu)
scans each CTA's contiguous range of landmark tiles; a CTA that finishes its
range hands its partial top-k lists to the rows it touched, and the CTA whose
hand-off completes a row merges it and publishes the row's kmax unit
descriptors (chunk + 1 and weight, or an empty marker past keff).  Then the
CTA's worker warps claim units u = 0, 1, 2, ... from one global counter (row
u / kmax, slot u % kmax), wait with a bound for the unit's descriptor, add the
chunk's weighted output into the row's accumulator, and bump the row's
counter; the warp whose bump completes the row's kmax slots converts it to O.

This model replays that with random scan lengths, publication orders and
unit times, and checks that every unit is claimed once, every row is
converted exactly once and only after all of its slots were added, and that
nothing waits forever -- when every CTA is resident at once, which is why the
launch is cooperative and hsa_forward fuses only when the grid fits the
device.  With fewer resident slots than CTAs the same hand-off can stall: a
worker waits on a row that only a CTA still queued behind it can publish.
The kernel's bounded wait then expires instead of hanging; the model reports
that as a timeout.
"""
import random

import pytest

EMPTY = "empty"


def run(nctas, nres, nrows, tiles_per_row, kmax, workers, seed):
    """Returns ("ok" | "timeout", per-row conversion counts, claimed units)."""
    rng = random.Random(seed)
    total = nrows * tiles_per_row
    per = -(-total // nctas)
    ranges = [(c * per, min(total, (c + 1) * per)) for c in range(nctas)]
    touched = [sorted({t // tiles_per_row for t in range(lo, hi)}) for lo, hi in ranges]
    need = [sum(r in t for t in touched) for r in range(nrows)]
    keff = [rng.randint(0, kmax) for _ in range(nrows)]
    handed = [0] * nrows
    desc = [None] * (nrows * kmax)
    added = [0] * nrows
    att_cnt = [0] * nrows
    converted = [0] * nrows
    claimed = []
    ctr = [0]

    def cta(c):
        lo, hi = ranges[c]
        for _ in range(max(1, hi - lo) * rng.randint(1, 3)):   # the scan of its range
            yield None
        for r in touched[c]:                                   # hand-off; the last one merges and publishes
            handed[r] += 1
            if handed[r] == need[r]:
                for i in range(kmax):
                    desc[r * kmax + i] = ("chunk", i) if i < keff[r] else EMPTY
            yield None
        for _ in range(workers):
            yield ("spawn", worker())

    def worker():
        while True:
            u = ctr[0]
            ctr[0] += 1
            if u >= nrows * kmax:
                return
            claimed.append(u)
            row = u // kmax
            while desc[u] is None:                             # bounded on the device
                yield "wait"
            if desc[u] != EMPTY:
                for _ in range(rng.randint(1, 4)):             # K/V copy, scores, PV, reductions
                    yield None
                added[row] += 1
            else:
                added[row] += 1                                # an empty slot still counts
            att_cnt[row] += 1
            if att_cnt[row] == kmax:                           # this warp completes the row
                assert added[row] == kmax
                converted[row] += 1
            yield None

    queue = list(range(nctas))
    live = {}                                                  # agent id -> (cta, generator)
    next_id = [0]

    def start(c):
        live[next_id[0]] = (c, cta(c))
        next_id[0] += 1

    resident = {}
    while queue and len(resident) < nres:
        c = queue.pop(0)
        resident[c] = 1
        start(c)
    while live:
        progressed = False
        for aid in rng.sample(list(live), len(live)):
            c, g = live[aid]
            try:
                step = next(g)
            except StopIteration:
                del live[aid]
                resident[c] -= 1
                if resident[c] == 0:                           # the CTA exits: its slot frees up
                    del resident[c]
                    if queue:
                        n = queue.pop(0)
                        resident[n] = 1
                        start(n)
                progressed = True
                continue
            if isinstance(step, tuple) and step[0] == "spawn":
                live[next_id[0]] = (c, step[1])
                next_id[0] += 1
                resident[c] += 1
                progressed = True
            elif step != "wait":
                progressed = True
        if not progressed:
            return "timeout", converted, claimed
    return "ok", converted, claimed


@pytest.mark.parametrize("seed", range(40))
def test_every_row_is_converted_once_when_all_ctas_are_resident(seed):
    rng = random.Random(1000 + seed)
    nctas = rng.randint(1, 12)
    nrows = rng.randint(1, 10)
    kmax = rng.choice([1, 4, 16, 32])
    status, converted, claimed = run(nctas, nctas, nrows, rng.randint(1, 40), kmax, rng.randint(1, 7), seed)
    assert status == "ok"
    assert converted == [1] * nrows
    assert sorted(claimed) == list(range(nrows * kmax))


def test_a_grid_beyond_the_resident_ctas_can_stall():
    """Two resident slots, three CTAs: the third CTA's rows are published only after it runs, but the
    first two never exit while their workers wait on those rows."""
    status, converted, _ = run(nctas=3, nres=2, nrows=3, tiles_per_row=4, kmax=4, workers=2, seed=0)
    assert status == "timeout"
    assert converted[2] == 0
