"""A randomized CPU model of the fused RMSNorm kernel's row-partial exchange inside a
cluster of C CTAs.  For every 128-row strip s each CTA sends its partial sums of squares
into every CTA's receive buffer part[s % 2][its rank] with st.async, which completes
transaction bytes on the receiver's xready[s % 2] mbarrier.  The receiver's reader warps
(one per consumer group) wait on xready by parity, read all C partials, and thread 0
re-arms xready[s % 2] for strip s + 2.  Every warp then arrives on pdone[(s + 1) % 2]
(its reads of strip s are done and its partials of strip s + 1 are written) and on
rready; a CTA sends strip s + 1 only after pdone[(s + 1) % 2] completes.

Both buffers are double-buffered by strip parity.  The model runs the protocol under
random and biased schedules, with sends landing at random later times, and checks that
a reader sees exactly strip s's partial from every rank, that no send lands in a buffer
its receiver has not finished reading, and that no transaction count goes negative.  Two
controls must be caught: a CTA that sends strip s + 1 as soon as its own pass 1 of that
strip is done (before its reads of strip s and the waits that follow them), and a
single buffer.  (Waiting on rready already implies pdone[(s + 1) % 2] in the kernel:
every warp arrives on both at the same point, so dropping the pdone wait alone changes
nothing.)"""
import random

import pytest


class MBarrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phases = 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phases += 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        if self.pending < 0:
            raise AssertionError("arrival beyond the barrier's count")
        self._maybe_complete()

    def complete_tx(self, n):
        self.tx -= n
        if self.tx < 0:
            raise AssertionError("bytes landed before the phase expected them")
        self._maybe_complete()

    def try_wait(self, parity):
        return (self.phases & 1) != parity


def run(C, ns, seed, early_send=False, buffers=2, bias=None):
    rng = random.Random(seed)
    G = 4                         # consumer groups; group g's reader warp is warp g
    NW = 8                        # warps per CTA in the model (4 readers + 4 others)
    nb = buffers

    class Cta:
        pass

    ctas = []
    for r in range(C):
        c = Cta()
        c.part = [[None] * C for _ in range(nb)]
        c.xready = [MBarrier(1) for _ in range(nb)]
        c.pdone = [MBarrier(NW) for _ in range(nb)]
        c.rready = MBarrier(NW)
        c.reads = {}              # strip -> reader warps done reading its partials
        for s in range(min(nb, ns)):
            c.xready[s % nb].arrive(expect_tx=C)   # armed before the cluster barrier
        ctas.append(c)
    inflight = []                 # (dst, buf, src, strip)

    def send(r, g, s):
        """Group g of CTA r sends its partial of strip s to the ranks c = g, g + 4, ..."""
        for q in range(g, C, G):
            inflight.append((q, s % nb, r, s))

    def warp(r, k):
        me = ctas[r]
        g = k % G
        reader = k < G
        # pass 1 of strip 0, then its exchange
        me.pdone[0].arrive()
        while not me.pdone[0].try_wait(0):
            yield
        if reader:
            send(r, g, 0)
        for s in range(ns):
            sp = s % nb
            more = s + 1 < ns
            yield                                  # pass 1 of the next strip
            if early_send and more and reader:
                send(r, g, s + 1)
            if reader:
                while not me.xready[sp].try_wait((s // nb) & 1):
                    yield
                for src in range(C):
                    if me.part[sp][src] != (s, src):
                        raise AssertionError(f"CTA {r} warp {k} read {me.part[sp][src]} for strip {s} from rank {src}")
                me.reads[s] = me.reads.get(s, 0) + 1
                if k == 0 and s + nb < ns:
                    me.xready[sp].arrive(expect_tx=C)
            if more:
                me.pdone[(s + 1) % nb].arrive()
            me.rready.arrive()
            while not me.rready.try_wait(s & 1):
                yield
            if more and not early_send:
                while not me.pdone[(s + 1) % nb].try_wait(((s + 1) // nb) & 1):
                    yield
                if reader:
                    send(r, g, s + 1)
            yield                                  # pass 2 of strip s

    agents = [warp(r, k) for r in range(C) for k in range(NW)]
    weights = [bias(r, k, rng) if bias else 1.0 for r in range(C) for k in range(NW)]
    live = list(range(len(agents)))
    steps = 0
    while live or inflight:
        steps += 1
        if steps > 400000:
            raise AssertionError("no progress")
        if inflight and (not live or rng.random() < 0.3):
            q, buf, src, s = inflight.pop(rng.randrange(len(inflight)))
            dst = ctas[q]
            old = s - nb
            if old >= 0 and dst.reads.get(old, 0) != G:
                raise AssertionError(f"strip {s} from rank {src} landed in CTA {q} before strip {old} was read")
            dst.part[buf][src] = (s, src)
            dst.xready[buf].complete_tx(1)
            continue
        i = rng.choices(live, weights=[weights[j] for j in live])[0]
        try:
            next(agents[i])
        except StopIteration:
            live.remove(i)
    for c in ctas:
        assert all(c.reads.get(s, 0) == G for s in range(ns)), "a strip was not read"
    return steps


def _biases():
    yield None
    yield lambda r, k, rng: 6.0 if r == 0 else 1.0        # one CTA races ahead
    yield lambda r, k, rng: 0.2 if r == 1 else 1.0        # one CTA lags
    yield lambda r, k, rng: 0.1 if k == 2 else 1.0        # one reader warp lags everywhere
    yield lambda r, k, rng: rng.uniform(0.05, 10.0)


@pytest.mark.parametrize("C", [1, 3, 4])
def test_exchange_holds_under_random_schedules(C):
    for b, bias in enumerate(_biases()):
        for seed in range(120):
            run(C, ns=10, seed=1000 * b + seed, bias=bias)


@pytest.mark.parametrize("control", ["send before the reads", "one buffer"])
def test_controls_are_caught(control):
    caught = 0
    for b, bias in enumerate(_biases()):
        for seed in range(120):
            try:
                if control == "send before the reads":
                    run(4, ns=10, seed=1000 * b + seed, early_send=True, bias=bias)
                else:
                    run(4, ns=10, seed=1000 * b + seed, buffers=1, bias=bias)
            except AssertionError:
                caught += 1
    assert caught > 0, control
