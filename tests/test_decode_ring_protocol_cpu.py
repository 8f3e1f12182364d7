"""Host model of the decode kernels' shared-memory ring (hga_decode_core.cuh:
one producer thread, eight consumer warps, S stages, mbarrier parity waits),
run under random interleavings.

A parity wait names only two phases: try_wait.parity(P) passes as soon as
the barrier's completed-phase count c has c % 2 != P. The model checks that
every wait that passes is the one its caller means (the stage holds the block
the consumer expects; the stage the producer refills has been released by
its last reader). With S a multiple of the eight consumer warps every use of
a stage belongs to one warp, so this holds for the kernels' S = 8 (bf16) and
S = 16 (E4M3); with S = 10 two warps share a stage and the model finds a
consumer that passes its wait early (the mistake the ring's static_assert
rules out)."""
import random

import pytest

WARPS = 8


class RingModel:
    def __init__(self, S: int, n_blocks: int, seed: int):
        self.S, self.n = S, n_blocks
        self.rng = random.Random(seed)
        self.full = [0] * S      # completed phases of each full barrier
        self.empty = [0] * S     # completed phases of each empty barrier
        self.content = [None] * S
        self.in_flight = []      # (stage, block) copies not yet landed
        self.next_issue = 0
        self.warp_next = list(range(WARPS))  # next block of each consumer warp
        self.reading = [None] * S  # block a consumer is reading from the stage
        self.busy = [None] * WARPS  # stage a warp is reading

    @staticmethod
    def passes(count: int, parity: int) -> bool:
        return (count & 1) != parity

    def step(self) -> bool:
        """One random enabled action; False when nothing is left to do."""
        actions = []
        i = self.next_issue
        if i < self.n:
            s = i % self.S
            if i < self.S or self.passes(self.empty[s], ((i // self.S) - 1) & 1):
                actions.append(("issue", i))
        for k in range(len(self.in_flight)):
            actions.append(("land", k))
        for w in range(WARPS):
            j = self.warp_next[w]
            if self.busy[w] is not None:
                actions.append(("release", w))
            elif j < self.n and self.passes(self.full[j % self.S], (j // self.S) & 1):
                actions.append(("consume", w))
        if not actions:
            return False
        kind, arg = self.rng.choice(actions)
        if kind == "issue":
            s = arg % self.S
            assert self.reading[s] is None, f"stage {s} refilled while block {self.reading[s]} is read"
            self.in_flight.append((s, arg))
            self.next_issue += 1
        elif kind == "land":
            s, blk = self.in_flight.pop(arg)
            self.content[s] = blk
            self.full[s] += 1
        elif kind == "consume":  # the warp's wait passed: it reads the stage
            w = arg
            j = self.warp_next[w]
            s = j % self.S
            assert self.content[s] == j, (
                f"warp {w} passed its wait for block {j} while stage {s} holds {self.content[s]}")
            assert not any(st == s for st, _ in self.in_flight), (
                f"warp {w} reads stage {s} while a copy into it is in flight")
            self.reading[s] = j
            self.busy[w] = s
        else:  # the warp has finished with the stage and releases it
            w = arg
            s = self.busy[w]
            self.reading[s] = None
            self.busy[w] = None
            self.empty[s] += 1
            self.warp_next[w] += WARPS
        return True

    def run(self):
        while self.step():
            pass
        assert self.next_issue == self.n and not self.in_flight
        assert all(self.warp_next[w] >= self.n for w in range(WARPS)), "deadlock"


@pytest.mark.parametrize("S", [8, 16])
@pytest.mark.parametrize("n_blocks", [3, 8, 28, 61, 112])
def test_ring_protocol_holds(S, n_blocks):
    for seed in range(200):
        RingModel(S, n_blocks, seed).run()


def test_ring_with_stages_not_a_multiple_of_the_warps_is_caught():
    """S = 10: some interleaving lets a warp pass its parity wait for a
    stage's third use before the second use's copy has landed."""
    caught = 0
    for seed in range(400):
        try:
            RingModel(10, 28, seed).run()
        except AssertionError:
            caught += 1
    assert caught > 0
