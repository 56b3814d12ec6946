"""The TMA ring of the streaming decode scan, on the CPU.

select_stream_kernel (landmark_guided_chunk_b200/csrc/select_stream.cu) streams
landmark tiles through NST ring stages: one producer thread fills stage
k % NST with tile k (after the stage's consumer released its previous tile)
and consumer warp k % NCW waits for that stage's phase, scores the tile and
releases it.  The kernel requires NST to be a multiple of NCW, so that each
stage has one consumer, which waits the stage's phases in order.  This model
replays the producer and the consumers with the kernel's phase formulas, TMA
loads landing in any order, and checks that the kernel's configuration
(12 stages, 6 consumer warps) finishes with every waiter testing its stage only
while the stage has completed the awaited phase or the one before (a
parity-only wait misreads anything else) -- and that the layout the
requirement excludes (12 stages over 8 warps, the configuration behind a GPU
fault this kernel once had) breaks that: a warp waits on a stage one phase
ahead of it and would take the previous tile for its own.
"""
import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count, f"{self.name}: over-arrived"
        if self.arrived == self.count:
            self.arrived = 0
            self.phase += 1


class ParityAlias(AssertionError):
    pass


def run(ntile, nst, ncw, seed):
    rng = random.Random(seed)
    full = [Bar(f"full{s}", 1) for s in range(nst)]
    empty = [Bar(f"empty{s}", 1) for s in range(nst)]
    landing = []   # TMA loads in flight (stage barriers)

    def producer():
        for k in range(ntile):
            s, u = k % nst, k // nst
            if u > 0:
                yield (empty[s], u - 1)
            landing.append(full[s])

    def consumer(w):
        for k in range(w, ntile, ncw):
            s, u = k % nst, k // nst
            yield (full[s], u)
            empty[s].arrive()

    roles = [producer()] + [consumer(w) for w in range(ncw)]
    waiting = [None] * len(roles)
    alive = set(range(len(roles)))

    def ready(r):
        if waiting[r] is None:
            return True
        bar, ph = waiting[r]
        # a parity wait is right only while the barrier has completed ph or ph + 1 phases: two
        # more and it reads as open, one fewer and the phase before reads as this one
        if not ph <= bar.phase <= ph + 1:
            raise ParityAlias(f"{bar.name}: waiter for phase {ph} sees phase {bar.phase}")
        return bar.phase > ph

    for _ in range(10 ** 6):
        if not alive:
            return
        choices = [("role", r) for r in alive if ready(r)] + ([("tma", 0)] if landing else [])
        assert choices, "deadlock"
        kind, x = rng.choice(choices)
        if kind == "tma":
            landing.pop(rng.randrange(len(landing))).arrive()
            continue
        try:
            waiting[x] = next(roles[x])
        except StopIteration:
            alive.discard(x)
            waiting[x] = None
    raise AssertionError("did not finish")


@pytest.mark.parametrize("ntile", [1, 5, 12, 13, 40, 200])
def test_kernel_ring_finishes_without_parity_alias(ntile):
    for seed in range(50):
        run(ntile, nst=12, ncw=6, seed=seed)


def test_ring_with_shared_stages_aliases():
    """12 stages over 8 consumer warps: stage s is consumed by several warps for consecutive phases,
    and a later warp can test the stage after it has moved two phases on."""
    seen = 0
    for seed in range(200):
        try:
            run(200, nst=12, ncw=8, seed=seed)
        except ParityAlias:
            seen += 1
    assert seen > 0
