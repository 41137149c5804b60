"""A randomized CPU model of the shared-memory ring that the block quantizer and the fused
RMSNorm kernel use: one producer thread streams items into S slots by TMA, and G
consumer groups of W warps take the items round-robin (group g gets items g, g + G, ...).
Each slot has a `full` mbarrier (one producer arrival plus the TMA's byte count) and an
`empty` mbarrier (one arrival per consumer warp).  Waits are parity waits: a wait for
parity P returns as soon as the barrier's completed-phase count has the other parity,
so it cannot tell phase k from phase k + 2.

The kernels' rule: before its parity wait on `full`, a group first waits for the slot's
previous item (it - S) to be released.  That wait is itself unambiguous because item
it - 2S belongs to the same group ((2S) mod G == 0) and is already done.  The model runs
the protocol under random and biased schedules and checks that a consumer only reads a
slot that holds its own, fully landed item, that the producer only refills a slot its
consumers have released, and that no barrier receives an arrival beyond its count.  A
control that drops the rule must be caught."""
import random

import pytest


class MBarrier:
    """mbarrier: `count` arrivals plus the expected transaction bytes complete a phase."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phases = 0          # completed phases

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phases += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        if self.pending < 0:
            raise AssertionError("arrival beyond the barrier's count")
        self._maybe_complete()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        if self.tx < 0:
            raise AssertionError("more bytes than expected")
        self._maybe_complete()

    def try_wait(self, parity):
        return (self.phases & 1) != parity


def run(S, G, W, n_items, seed, rule=True, bias=None):
    """One schedule.  Raises AssertionError on a protocol violation, else returns the
    number of scheduler steps taken."""
    rng = random.Random(seed)
    full = [MBarrier(1) for _ in range(S)]
    empty = [MBarrier(W) for _ in range(S)]
    slot = [None] * S              # item whose data the slot holds; "busy" while loading
    released = [0] * n_items       # warps that released each item
    inflight = []                  # (slot, item) TMA copies not yet landed

    def producer():
        for it in range(n_items):
            st, ph = it % S, (it // S) & 1
            while not empty[st].try_wait(ph ^ 1):
                yield
            if it >= S and released[it - S] != W:
                raise AssertionError(f"slot {st} refilled with item {it} before item {it - S} was released")
            full[st].arrive_expect_tx(1)
            slot[st] = "busy"
            inflight.append((st, it))
            yield

    def consumer(g, w):
        it = g
        while it < n_items:
            st, ph = it % S, (it // S) & 1
            if rule and it >= S:
                while not empty[st].try_wait(ph ^ 1):
                    yield
            while not full[st].try_wait(ph):
                yield
            if slot[st] != it:
                raise AssertionError(f"group {g} warp {w} read slot {st} for item {it}, slot holds {slot[st]}")
            yield                  # the warp works on the slot
            if slot[st] != it:
                raise AssertionError(f"slot {st} changed under item {it}")
            released[it] += 1
            empty[st].arrive()
            it += G
            yield

    agents = [producer()] + [consumer(g, w) for g in range(G) for w in range(W)]
    weights = [1.0] + [1.0] * (G * W)
    if bias is not None:
        for g in range(G):
            for w in range(W):
                weights[1 + g * W + w] = bias(g, w, rng)
    live = list(range(len(agents)))
    steps = 0
    while live or inflight:
        steps += 1
        if steps > 200000:
            raise AssertionError("no progress")
        if inflight and (not live or rng.random() < 0.3):
            st, it = inflight.pop(rng.randrange(len(inflight)))
            slot[st] = it
            full[st].complete_tx(1)
            continue
        k = rng.choices(live, weights=[weights[i] for i in live])[0]
        try:
            next(agents[k])
        except StopIteration:
            live.remove(k)
    assert all(r == W for r in released), "an item was never released"
    return steps


# the kernels' configuration (slots, groups, warps per group): the block quantizer's ring
# and the fused RMSNorm's ring are both six slots served by four groups of four warps
CONFIGS = [(6, 4, 4)]


def _biases():
    yield None
    yield lambda g, w, rng: 8.0 if g == 0 else 1.0              # one group races ahead
    yield lambda g, w, rng: 0.2 if g == 1 else 1.0              # one group lags
    yield lambda g, w, rng: 0.1 if (g, w) == (2, 3) else 1.0    # one warp lags
    yield lambda g, w, rng: rng.uniform(0.05, 10.0)


@pytest.mark.parametrize("S,G,W", CONFIGS)
def test_ring_rule_holds_under_random_schedules(S, G, W):
    assert (2 * S) % G == 0 and S >= G
    for b, bias in enumerate(_biases()):
        for seed in range(300):
            run(S, G, W, n_items=48, seed=1000 * b + seed, bias=bias)


@pytest.mark.parametrize("S,G,W", CONFIGS)
def test_dropping_the_rule_is_caught(S, G, W):
    """Without the wait on the previous item's release, some schedule lets a group pass
    its parity wait on `full` one phase early and read a slot that holds another item."""
    caught = 0
    for b, bias in enumerate(_biases()):
        for seed in range(300):
            try:
                run(S, G, W, n_items=48, seed=1000 * b + seed, rule=False, bias=bias)
            except AssertionError:
                caught += 1
    assert caught > 0

