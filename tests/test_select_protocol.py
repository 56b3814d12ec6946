"""The barrier protocol of the tensor-core prefill scoring, on the CPU.

select_tc_kernel (landmark_guided_chunk_b200/csrc/select_tc.cu) hands data
between a TMA producer thread (a CTA's query tile in nkb K-boxes, then the tile's
landmark slices through a ring of NSTAGE stages), the MMA thread (one TMEM
accumulator per slice, two in turn) and four epilogue warps (the fused
top-k).  A tile whose causal range holds no chunk is skipped by every role.
This model replays the three roles with the kernel's phase formulas, TMA loads
and tcgen05 commits completing after random delays (loads in any order,
commits in issue order), over random per-tile slice counts, and checks that
every role finishes and that every waiter tests its barrier only while the
barrier has completed the awaited phase or the one before (a parity-only wait
misreads anything else).  A change to the kernel's barriers, counts or phase
arithmetic has to be mirrored here.
"""
import random

import pytest

NSTAGE, NEPI = 2, 4


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count, f"{self.name}: over-arrived"
        if self.arrived == self.count:
            self.arrived = 0
            self.phase += 1


def run(slices, nkb, seed):
    """slices: the number of landmark slices of each of this CTA's tiles (0 = skipped)."""
    rng = random.Random(seed)
    a_full = [Bar(f"a_full{kb}", 1) for kb in range(nkb)]
    a_empty = [Bar(f"a_empty{kb}", 1) for kb in range(nkb)]
    b_full = [Bar(f"b_full{s}", 1) for s in range(NSTAGE)]
    b_empty = [Bar(f"b_empty{s}", 1) for s in range(NSTAGE)]
    t_full = [Bar(f"t_full{b}", 1) for b in range(2)]
    t_empty = [Bar(f"t_empty{b}", NEPI) for b in range(2)]
    tma, mma = [], []

    def producer():
        g = ta = 0
        for ns in slices:
            if ns == 0:
                continue
            for kb in range(nkb):
                if ta > 0:
                    yield (a_empty[kb], ta - 1)
                tma.append(a_full[kb])
            ta += 1
            for _ in range(ns):
                s, i = g % NSTAGE, g // NSTAGE
                if i > 0:
                    yield (b_empty[s], i - 1)
                tma.append(b_full[s])
                g += 1

    def issuer():
        g = ta = 0
        for ns in slices:
            if ns == 0:
                continue
            pa = ta
            ta += 1
            for n in range(ns):
                s, i, buf, u = g % NSTAGE, g // NSTAGE, g & 1, g >> 1
                yield (b_full[s], i)
                if u > 0:
                    yield (t_empty[buf], u - 1)
                commits = []
                for kb in range(nkb):
                    if n == 0:
                        yield (a_full[kb], pa)
                    if n == ns - 1:
                        commits.append(a_empty[kb])
                mma.append(commits + [b_empty[s], t_full[buf]])
                g += 1

    def epilogue(w):
        g = 0
        for ns in slices:
            for _ in range(ns):
                buf, u = g & 1, g >> 1
                yield (t_full[buf], u)
                t_empty[buf].arrive()
                g += 1

    roles = [producer(), issuer()] + [epilogue(w) for w in range(NEPI)]
    waiting = [None] * len(roles)
    alive = set(range(len(roles)))

    def ready(r):
        if waiting[r] is None:
            return True
        bar, ph = waiting[r]
        assert ph <= bar.phase <= ph + 1, f"{bar.name}: waiter for phase {ph} sees phase {bar.phase} (parity alias)"
        return bar.phase > ph

    for _ in range(10 ** 6):
        if not alive:
            return
        choices = [("role", r) for r in alive if ready(r)]
        choices += [("tma", 0)] if tma else []
        choices += [("mma", 0)] if mma else []
        assert choices, "deadlock: " + ", ".join(f"role {r} waits {waiting[r][0].name} phase {waiting[r][1]}"
                                                 for r in alive)
        kind, x = rng.choice(choices)
        if kind == "tma":
            tma.pop(rng.randrange(len(tma))).arrive()
        elif kind == "mma":
            for bar in mma.pop(0):
                bar.arrive()
        else:
            try:
                waiting[x] = next(roles[x])
            except StopIteration:
                alive.discard(x)
                waiting[x] = None
    raise AssertionError("did not finish")


@pytest.mark.parametrize("nkb", [1, 2, 4, 8])
def test_protocol_finishes_without_parity_alias(nkb):
    rng = random.Random(nkb)
    for trial in range(60):
        ntile = rng.randint(1, 9)
        slices = [rng.choice([0, 1, 1, 2, 3, 5, 8]) for _ in range(ntile)]
        run(slices, nkb, seed=trial)
