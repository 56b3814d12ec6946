"""The barrier protocol of the warp-specialized tensor-core backward, on the CPU.

bwd_tcw_kernel (landmark_guided_chunk_b200/csrc/backward.cu) runs four roles
that hand tiles to each other through mbarriers: producer warps (row info,
Q/dO gathers, K/V per chunk run), softmax warps, drain warps and one MMA
thread.  The asynchronous completions are cp.async arrivals (a thread's
arrival lands once its earlier copies have) and tcgen05 commits (in issue
order, once the MMAs before them are done).  This model replays every role's
loop with the kernel's phase formulas, under random interleavings and random
completion delays, over random sequences of chunk runs, and checks that:
  * every role finishes (no wait that can never be satisfied), and
  * every waiter tests its barrier only while the barrier has completed the
    phase it waits for or the one before (an mbarrier wait compares parity
    only: two phases further on reads as open, one phase short reads the
    previous phase as this one).
A change to the kernel's barriers, counts or phase arithmetic has to be
mirrored here.
"""
import random

import pytest

NW_P, NW_S, NW_D, NWI = 4, 4, 4, 4


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase = name, count, 0, 0

    def arrive(self, n=1):
        self.arrived += n
        assert self.arrived <= self.count, f"{self.name}: over-arrived"
        if self.arrived == self.count:
            self.arrived = 0
            self.phase += 1


class Kernel:
    def __init__(self, buckets):
        self.tiles = buckets
        self.n = len(buckets)
        B = Bar
        self.q_full = [B(f"q_full{b}", 32 * NW_P) for b in range(2)]
        self.q_empty = [B(f"q_empty{b}", 1) for b in range(2)]
        self.dq_full = [B(f"dq_full{b}", 1) for b in range(2)]
        self.dq_empty = [B(f"dq_empty{b}", NW_D) for b in range(2)]
        self.zg_full, self.zg_empty = B("zg_full", 1), B("zg_empty", NW_S)
        self.kv_full, self.kv_empty = B("kv_full", 32 * NW_P), B("kv_empty", 1)
        self.ds_full, self.ds_empty = B("ds_full", NW_S), B("ds_empty", 1)
        self.info_full = [B(f"info_full{s}", NW_P) for s in range(NWI)]
        self.info_empty = [B(f"info_empty{s}", NW_D) for s in range(NWI)]
        self.cp_pending = {w: [] for w in range(NW_P)}   # per producer warp, in issue order
        self.mma_pending = []                            # commits, in issue order

    # ---- roles: generators that yield ("wait", bar, phase index)
    def producer(self, w):
        prev, nload = -1, 0
        for i in range(self.n):
            b, si = i & 1, i % NWI
            if self.tiles[i] != prev:
                if nload > 0:
                    yield ("wait", self.kv_empty, nload - 1)
                self.cp_pending[w].append([self.kv_full])
                nload += 1
                prev = self.tiles[i]
            if i >= 2:
                yield ("wait", self.q_empty[b], (i >> 1) - 1)
            if i >= NWI:
                yield ("wait", self.info_empty[si], i // NWI - 1)
            self.info_full[si].arrive(1)
            self.cp_pending[w].append([self.q_full[b]])

    def softmax(self, w):
        for i in range(self.n):
            si = i % NWI
            yield ("wait", self.info_full[si], i // NWI)
            yield ("wait", self.zg_full, i)
            if i >= 1:
                yield ("wait", self.ds_empty, i - 1)
            self.zg_empty.arrive(1)
            self.ds_full.arrive(1)

    def drain(self, w):
        for i in range(self.n):
            si = i % NWI
            yield ("wait", self.info_full[si], i // NWI)
            self.info_empty[si].arrive(1)
            yield ("wait", self.dq_full[i & 1], i >> 1)
            self.dq_empty[i & 1].arrive(1)

    def issuer(self):
        def mma1(i, newc, li):
            b = i & 1
            yield ("wait", self.q_full[b], i >> 1)
            if newc:
                yield ("wait", self.kv_full, li)
            if i >= 1:
                yield ("wait", self.zg_empty, i - 1)
            self.mma_pending.append([self.zg_full])

        def mma2(i, first, endc):
            b = i & 1
            yield ("wait", self.ds_full, i)
            if i >= 2:
                yield ("wait", self.dq_empty[b], (i >> 1) - 1)
            self.mma_pending.append([self.dq_full[b], self.ds_empty, self.q_empty[b]] +
                                    ([self.kv_empty] if endc else []))

        first_prev = end_prev = False
        prev, li = -1, -1
        for i in range(self.n):
            bk = self.tiles[i]
            bk_next = self.tiles[i + 1] if i + 1 < self.n else -1
            newc, endc = bk != prev, bk_next != bk
            if newc:
                li += 1
            if i >= 1 and newc:
                yield from mma2(i - 1, first_prev, end_prev)
            yield from mma1(i, newc, li)
            if i >= 1 and not newc:
                yield from mma2(i - 1, first_prev, end_prev)
            first_prev, end_prev, prev = newc, endc, bk
        yield from mma2(self.n - 1, first_prev, end_prev)


def run(buckets, seed):
    rng = random.Random(seed)
    k = Kernel(buckets)
    roles = ([k.producer(w) for w in range(NW_P)] + [k.softmax(w) for w in range(NW_S)] +
             [k.drain(w) for w in range(NW_D)] + [k.issuer()])
    waiting = [None] * len(roles)   # the (bar, phase) each role is blocked on
    alive = set(range(len(roles)))

    def ready(r):
        if waiting[r] is None:
            return True
        bar, ph = waiting[r]
        # a parity wait is right only while the barrier has completed ph or ph + 1 phases
        assert ph <= bar.phase <= ph + 1, f"{bar.name}: waiter for phase {ph} sees phase {bar.phase} (parity alias)"
        return bar.phase > ph

    steps = 0
    while alive:
        steps += 1
        assert steps < 10 ** 6
        runnable = [r for r in alive if ready(r)]
        asyncs = [("cp", w) for w in range(NW_P) if k.cp_pending[w]] + ([("mma", 0)] if k.mma_pending else [])
        choices = [("role", r) for r in runnable] + asyncs
        assert choices, "deadlock: " + ", ".join(f"role {r} waits {waiting[r][0].name} phase {waiting[r][1]}"
                                                 for r in alive)
        kind, x = rng.choice(choices)
        if kind == "cp":
            for bar in k.cp_pending[x].pop(0):
                bar.arrive(32)
        elif kind == "mma":
            for bar in k.mma_pending.pop(0):
                bar.arrive(1)
        else:
            try:
                _, bar, ph = next(roles[x])
                waiting[x] = (bar, ph)
            except StopIteration:
                alive.discard(x)
                waiting[x] = None
    # the asynchronous completions still in flight land (the kernel drains them before it exits)
    while any(k.cp_pending.values()) or k.mma_pending:
        for w in range(NW_P):
            while k.cp_pending[w]:
                for bar in k.cp_pending[w].pop(0):
                    bar.arrive(32)
        while k.mma_pending:
            for bar in k.mma_pending.pop(0):
                bar.arrive(1)
    return k


def _runs(rng, n):
    """A CTA's tile list: n tiles in runs of one bucket each (random run lengths)."""
    out, b = [], 0
    while len(out) < n:
        out += [b] * rng.randint(1, 6)
        b += rng.randint(1, 3)
    return out[:n]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 17, 40])
def test_protocol_finishes_without_parity_alias(n):
    rng = random.Random(n)
    for trial in range(60):
        buckets = _runs(rng, n)
        k = run(buckets, seed=1000 * n + trial)
        # every tile passed every stage once
        assert k.zg_full.phase == n and k.ds_full.phase == n
        assert k.dq_full[0].phase + k.dq_full[1].phase == n


def test_one_chunk_per_tile_and_one_long_run():
    for buckets in ([0] * 33, list(range(33))):
        for seed in range(40):
            run(buckets, seed)
