"""Host-side model of the synchronisation protocol of the persistent prefill
attention kernel (attend_tc_kernel), checked under random interleavings.

Each role of a CTA is a generator that performs, in the kernel's order, its
waits and arrivals on mbarriers: the list builder (warp 10), the TMA
producer (warp 0), the MMA issuer (warp 1) and the eight softmax warps
(four per M tile). Asynchronous hardware is modelled as separate actors:
TMA loads complete in any order; tcgen05 operations and their commits run in
issue order on one tensor-core queue. A random scheduler interleaves
everything. The test requires that

  * every role finishes (no deadlock for any unit / tile sequence);
  * no wait targets a phase two or more behind its barrier's current phase
    (a parity wait would alias and hang or pass wrongly);
  * the data hazards the barriers exist for never occur: a QK overwrites
    S_x only after every softmax warp of M tile x finished the previous
    tile; a unit's first PV (which overwrites O_x) runs only after those
    warps read O_x in the previous unit's epilogue; Q, K and V stages and
    block-list buffers are refilled only after their last readers are done.
"""
import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count, self.name
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


class Model:
    def __init__(self, tiles, rng):
        self.tiles = tiles  # key tiles of each unit this CTA walks, in order
        self.rng = rng
        b = Bar
        self.list_full = [b("list_full0", 1), b("list_full1", 1)]
        self.list_empty = [b("list_empty0", 9), b("list_empty1", 9)]
        self.bar_q, self.q_empty = b("bar_q", 1), b("q_empty", 1)
        self.k_full = [b("k_full0", 1), b("k_full1", 1)]
        self.k_empty = [b("k_empty0", 1), b("k_empty1", 1)]
        self.v_full = [b("v_full0", 1), b("v_full1", 1)]
        self.v_empty = [b("v_empty0", 1), b("v_empty1", 1)]
        self.s_full = [b("s_full0", 1), b("s_full1", 1)]
        self.p_full = [b("p_full0", 4), b("p_full1", 4)]
        self.o_done = [b("o_done0", 1), b("o_done1", 1)]
        self.drain = b("drain", 1)
        self.tma = []          # pending TMA completions (any order)
        self.tq = []           # tensor-core queue: ops and commits, in order
        # progress records for the hazard checks
        self.qk_done = [[], []]          # global tiles whose QK_x has executed
        self.pv_done = [[], []]
        self.sm_tiles_done = [[0] * 4, [0] * 4]   # tiles finished per softmax warp
        self.epi_done = [[0] * 4, [0] * 4]        # unit epilogues that read O, per warp
        self.list_users_done = [0, 0]             # list buffer readers released

    # ------------------------------------------------------------ actions
    def wait(self, bar, phase):
        # a parity wait for `phase`: fine once bar.done == phase + 1; aliased
        # if the barrier is already two or more phases past it
        while True:
            assert bar.done <= phase + 1, f"{bar.name}: waiting for phase {phase}, at {bar.done}"
            if bar.done == phase + 1:
                return
            yield

    def load(self, bar, check=None):
        if check:
            check()
        self.tma.append(bar)

    def op(self, fn):
        self.tq.append(fn)

    def commit(self, bar):
        self.tq.append(bar.arrive)

    # ------------------------------------------------------------ roles
    def builder(self):
        for k in range(len(self.tiles)):
            bf = k & 1
            if k >= 2:
                yield from self.wait(self.list_empty[bf], (k >> 1) - 1)
            self.list_full[bf].arrive()
            yield

    def producer(self):
        g0 = 0
        for k, n in enumerate(self.tiles):
            bf = k & 1
            yield from self.wait(self.list_full[bf], k >> 1)
            if k >= 1:
                yield from self.wait(self.q_empty, k - 1)
            prev_last = g0 - 1  # last global tile of unit k-1: its QKs read the Q buffer

            def q_free(prev_last=prev_last):
                for x in range(2):
                    assert all(g in self.qk_done[x] for g in range(max(prev_last - 8, 0), prev_last + 1)), \
                        "Q refilled before the previous unit's QKs ran"
            self.load(self.bar_q, q_free)
            for t in range(n):
                g, s = g0 + t, (g0 + t) & 1
                if g >= 2:
                    yield from self.wait(self.k_empty[s], (g >> 1) - 1)

                def k_free(g=g):
                    for x in range(2):
                        assert g < 2 or (g - 2) in self.qk_done[x], "K stage refilled too early"
                self.load(self.k_full[s], k_free)
                if g >= 2:
                    yield from self.wait(self.v_empty[s], (g >> 1) - 1)

                def v_free(g=g):
                    for x in range(2):
                        assert g < 2 or (g - 2) in self.pv_done[x], "V stage refilled too early"
                self.load(self.v_full[s], v_free)
                yield
            self.list_empty[bf].arrive()
            g0 += n

    def mma(self):
        g0 = 0
        for k, n in enumerate(self.tiles):
            bf = k & 1
            yield from self.wait(self.list_full[bf], k >> 1)
            s0 = g0 & 1
            yield from self.wait(self.bar_q, k)
            yield from self.wait(self.k_full[s0], g0 >> 1)
            for x in range(2):
                self.op(self.qk(x, g0))
                self.commit(self.s_full[x])
            if n == 1:
                self.commit(self.q_empty)
            self.commit(self.k_empty[s0])
            for t in range(n):
                g, s, s1, more = g0 + t, (g0 + t) & 1, (g0 + t + 1) & 1, t + 1 < n
                yield from self.wait(self.v_full[s], g >> 1)
                if more:
                    yield from self.wait(self.k_full[s1], (g + 1) >> 1)
                for x in range(2):
                    yield from self.wait(self.p_full[x], g)
                    self.op(self.pv(x, g, k if t == 0 else None))
                    if more:
                        self.op(self.qk(x, g + 1))
                        self.commit(self.s_full[x])
                    else:
                        self.commit(self.o_done[x])
                if more and t + 2 == n:
                    self.commit(self.q_empty)
                self.commit(self.v_empty[s])
                if more:
                    self.commit(self.k_empty[s1])
                yield
            g0 += n
        self.commit(self.drain)
        yield from self.wait(self.drain, 0)

    def qk(self, x, g):
        def run():
            # S_x is overwritten: every softmax warp of x finished tile g-1
            assert all(d >= g for d in self.sm_tiles_done[x]), f"QK_{x}({g}) before softmax read S"
            self.qk_done[x].append(g)
        return run

    def pv(self, x, g, unit_start):
        def run():
            if unit_start is not None and unit_start >= 1:
                # accumulate=false: O_x is overwritten after the epilogue read it
                assert all(e >= unit_start for e in self.epi_done[x]), f"PV_{x} overwrote O early"
            self.pv_done[x].append(g)
        return run

    def softmax(self, x, w):
        g0 = 0
        for k, n in enumerate(self.tiles):
            bf = k & 1
            yield from self.wait(self.list_full[bf], k >> 1)
            for t in range(n):
                g = g0 + t
                yield from self.wait(self.s_full[x], g)
                assert g in self.qk_done[x]
                yield  # the softmax of this tile
                self.sm_tiles_done[x][w] = g + 1
                self.p_full[x].arrive()
            self.list_empty[bf].arrive()
            yield from self.wait(self.o_done[x], k)
            self.epi_done[x][w] = k + 1  # O read into registers
            yield  # normalise and store
            g0 += n

    # ------------------------------------------------------------ scheduler
    def run(self, max_steps=200000):
        roles = [self.builder(), self.producer(), self.mma()] + \
                [self.softmax(x, w) for x in range(2) for w in range(4)]
        live = list(range(len(roles)))
        for _ in range(max_steps):
            choices = list(live)
            if self.tma:
                choices.append("tma")
            if self.tq:
                choices.append("tq")
            if not choices:
                return
            c = self.rng.choice(choices)
            if c == "tma":
                self.tma.pop(self.rng.randrange(len(self.tma))).arrive()
            elif c == "tq":
                self.tq.pop(0)()
            else:
                try:
                    next(roles[c])
                except StopIteration:
                    live.remove(c)
        raise AssertionError("did not finish: a role waits forever")


@pytest.mark.parametrize("seed", range(40))
def test_random_units_and_interleavings(seed):
    rng = random.Random(seed)
    tiles = [rng.choice([1, 1, 2, 3, 4, 7, 14]) for _ in range(rng.randint(1, 7))]
    m = Model(tiles, rng)
    m.run()
    assert not m.tma and not m.tq
    total = sum(tiles)
    for x in range(2):
        assert m.qk_done[x] == list(range(total)) and m.pv_done[x] == list(range(total))
        assert m.o_done[x].done == len(tiles)


def test_a_missing_arrival_is_caught():
    """The model detects a broken protocol: without the softmax warps'
    release of the list buffers, the builder waits forever."""
    m = Model([2, 2, 2], random.Random(0))
    m.list_empty[0].count = 10  # one arrival more than the kernel makes
    with pytest.raises(AssertionError):
        m.run(max_steps=20000)
