"""The barrier protocol of the tensor-core prefill attention, on the CPU.

att_main_kernel (landmark_guided_chunk_b200/csrc/attend_tc.cu) hands each tile
through mbarriers between two producer warps (row info into a ring of NINFO
slots, Q rows into nsq stages), a K/V loader thread (one TMA load per run of
tiles sharing a chunk, nskv stages), the MMA thread, four softmax warps and
eight O-drain warps; S, P and O are double-buffered by tile parity.  The
asynchronous completions are the producers' cp.async arrivals, the TMA loads
and the tcgen05 commits.  This model replays each role with the kernel's phase
formulas for both stage configurations (S = 64: nsq = nskv = 2; S = 128: one
each), under random interleavings and completion delays, over random tile
sequences, and checks that every role finishes, that every waiter tests its
barrier only while it has completed the awaited phase or the one before (a
parity-only wait misreads anything else), and the one hand-off with no
barrier: QK of tile i overwrites
the S buffer of tile i-2, so the softmax must have read that tile by then
(it has, through p_full, before PV(i-2) is issued).  A change to the
kernel's barriers, counts or phase arithmetic has to be mirrored here.
"""
import random

import pytest

NINFO, NPROD_WARPS, NSOFT, NDRAIN = 4, 2, 4, 8


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
    def __init__(self, tiles, nsq, nskv):
        self.t, self.n, self.nsq, self.nskv = tiles, len(tiles), nsq, nskv
        B = Bar
        self.q_full = [B(f"q_full{s}", 32 * NPROD_WARPS) for s in range(nsq)]
        self.q_empty = [B(f"q_empty{s}", 1) for s in range(nsq)]
        self.kv_full = [B(f"kv_full{s}", 1) for s in range(nskv)]
        self.kv_empty = [B(f"kv_empty{s}", 1) for s in range(nskv)]
        self.s_full = [B(f"s_full{b}", 1) for b in range(2)]
        self.p_full = [B(f"p_full{b}", NSOFT) for b in range(2)]
        self.p_empty = [B(f"p_empty{b}", 1) for b in range(2)]
        self.o_full = [B(f"o_full{b}", 1) for b in range(2)]
        self.o_empty = [B(f"o_empty{b}", NDRAIN) for b in range(2)]
        self.l_full = [B(f"l_full{b}", NSOFT) for b in range(2)]
        self.l_empty = [B(f"l_empty{b}", NDRAIN) for b in range(2)]
        self.info_full = [B(f"info_full{s}", 32 * NPROD_WARPS) for s in range(NINFO)]
        self.info_empty = [B(f"info_empty{s}", NDRAIN) for s in range(NINFO)]
        self.cp_pending = {w: [] for w in range(NPROD_WARPS)}
        self.tma_pending = []
        self.mma_pending = []
        self.s_read = [0] * NSOFT   # tiles whose S each softmax warp has finished reading

    def producer(self, w):
        for i in range(self.n):
            si, ii = i % NINFO, i // NINFO
            if ii > 0:
                yield ("wait", self.info_empty[si], ii - 1)
            self.info_full[si].arrive(32)
            sq, iq = i % self.nsq, i // self.nsq
            if iq > 0:
                yield ("wait", self.q_empty[sq], iq - 1)
            self.cp_pending[w].append(self.q_full[sq])

    def loader(self):
        nload, prev = 0, None
        for i in range(self.n):
            if self.t[i] == prev:
                continue
            prev = self.t[i]
            skv, ikv = nload % self.nskv, nload // self.nskv
            if ikv > 0:
                yield ("wait", self.kv_empty[skv], ikv - 1)
            self.tma_pending.append(self.kv_full[skv])
            nload += 1

    def issuer(self):
        loads = []   # load index of each tile, as the kernel derives it from the tile records
        prev, nl = None, 0
        for i in range(self.n):
            if self.t[i] != prev:
                prev, nl = self.t[i], nl + 1
            loads.append(nl - 1)
        waited = [-1]

        def issue_qk(i, li):
            sq, iq, skv, ikv = i % self.nsq, i // self.nsq, li % self.nskv, li // self.nskv
            yield ("wait", self.q_full[sq], iq)
            if li != waited[0]:
                yield ("wait", self.kv_full[skv], ikv)
                waited[0] = li
            # QK(i) writes the S buffer of tile i - 2: every softmax warp must be done reading it
            assert i < 2 or min(self.s_read) >= i - 1, f"QK({i}) would overwrite S of tile {i - 2} before it is read"
            self.mma_pending.append([self.s_full[i & 1], self.q_empty[sq]])

        early = self.nskv >= 2
        if self.n == 0:
            return
        yield from issue_qk(0, loads[0])
        for i in range(self.n):
            b, k = i & 1, i >> 1
            li, li_next = loads[i], loads[i + 1] if i + 1 < self.n else -1
            if early and li_next >= 0:
                yield from issue_qk(i + 1, li_next)
            yield ("wait", self.p_full[b], k)
            if k > 0:
                yield ("wait", self.o_empty[b], k - 1)
            commits = [self.o_full[b], self.p_empty[b]]
            if li_next != li:
                commits.append(self.kv_empty[li % self.nskv])
            self.mma_pending.append(commits)
            if not early and li_next >= 0:
                yield from issue_qk(i + 1, li_next)

    def softmax(self, w):
        for i in range(self.n):
            b, k = i & 1, i >> 1
            yield ("wait", self.s_full[b], k)
            self.s_read[w] = i + 1
            if k > 0:
                yield ("wait", self.p_empty[b], k - 1)
            self.p_full[b].arrive(1)
            if k > 0:
                yield ("wait", self.l_empty[b], k - 1)
            self.l_full[b].arrive(1)

    def drain(self, w):
        for i in range(self.n):
            b, k, si = i & 1, i >> 1, i % NINFO
            yield ("wait", self.info_full[si], i // NINFO)
            self.info_empty[si].arrive(1)
            yield ("wait", self.l_full[b], k)
            self.l_empty[b].arrive(1)
            yield ("wait", self.o_full[b], k)
            self.o_empty[b].arrive(1)


def run(tiles, nsq, nskv, seed):
    rng = random.Random(seed)
    k = Kernel(tiles, nsq, nskv)
    roles = ([k.producer(w) for w in range(NPROD_WARPS)] + [k.loader(), k.issuer()] +
             [k.softmax(w) for w in range(NSOFT)] + [k.drain(w) for w in range(NDRAIN)])
    waiting = [None] * len(roles)
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
        choices = [("role", r) for r in alive if ready(r)]
        choices += [("cp", w) for w in range(NPROD_WARPS) if k.cp_pending[w]]
        choices += [("tma", 0)] if k.tma_pending else []
        choices += [("mma", 0)] if k.mma_pending else []
        assert choices, "deadlock: " + ", ".join(f"role {r} waits {waiting[r][0].name} phase {waiting[r][1]}"
                                                 for r in alive)
        kind, x = rng.choice(choices)
        if kind == "cp":
            k.cp_pending[x].pop(0).arrive(32)
        elif kind == "tma":
            k.tma_pending.pop(rng.randrange(len(k.tma_pending))).arrive(1)   # loads land in any order
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
    return k


def _tiles(rng, n):
    """Tile records (phase, chunk): runs of tiles sharing one chunk, phases in order."""
    out, p, c = [], 0, 0
    while len(out) < n:
        out += [(p, c)] * rng.randint(1, 5)
        c += rng.randint(1, 4)
        if rng.random() < 0.2:
            p, c = p + 1, 0
    return out[:n]


@pytest.mark.parametrize("nsq,nskv", [(2, 2), (1, 1)])
@pytest.mark.parametrize("n", [1, 2, 3, 5, 9, 24])
def test_protocol_finishes_without_parity_alias(n, nsq, nskv):
    rng = random.Random(17 * n + nsq)
    for trial in range(40):
        k = run(_tiles(rng, n), nsq, nskv, seed=trial)
        assert sum(b.phase for b in k.o_full) == n and sum(b.phase for b in k.p_full) == n
