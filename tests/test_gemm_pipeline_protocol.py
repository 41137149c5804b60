"""A randomized CPU model of the block-wise GEMM's pipeline in one CTA (the scaled mode).
One TMA producer fills S stages (full / empty mbarriers); one MMA thread waits for a stage
and for an accumulator buffer (tfull / tempty, two buffers used in turn, one K block
each), issues the K block's MMAs and commits them to the stage's `empty` and the buffer's
`tfull` (commits complete in issue order, at random later times); E epilogue warps wait
for `tfull`, read the buffer, re-fill it and arrive on `tempty`.  The per-tile scales are
double-buffered: at a tile's start each warp waits on sready[tile % 2], then copies the
next tile's scales into the other buffer (copies land at random later times); at the
tile's end it waits for its copies and arrives on sready[(tile + 1) % 2].  The epilogue
pre-fills both accumulators and releases them once before the first tile.

Checked under random and biased schedules: the MMA reads a stage only when it holds that
K block's operands and writes a buffer only after every epilogue warp released its
previous contents; the producer refills a stage only after the MMA that read it
completed; a warp reads a buffer only when it holds its tile's K block and nothing writes
it during the read; a warp reads only its tile's scales, and no scale copy lands in a
buffer a warp still reads; no barrier receives an arrival beyond its count.  Three
controls must be caught: the MMA not waiting on `tempty`, a warp releasing the buffer
before its reads are done, and the scale prefetch issued before the `sready` wait."""
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
            raise AssertionError("bytes before the phase expected them")
        self._maybe_complete()

    def try_wait(self, parity):
        return (self.phases & 1) != parity


def run(tiles, KB, seed, S=4, E=8, mma_waits_tempty=True, release_after_reads=True,
        prefetch_after_sready=True, bias=None):
    rng = random.Random(seed)
    full = [MBarrier(1) for _ in range(S)]
    empty = [MBarrier(1) for _ in range(S)]
    tfull = [MBarrier(1) for _ in range(2)]
    tempty = [MBarrier(E) for _ in range(2)]
    sready = [MBarrier(E) for _ in range(2)]
    stage = [None] * S                 # (tile, kb) held, "busy" while its TMA is in flight
    stage_reader = [None] * S          # (tile, kb) whose MMA still reads the stage
    acc = [None] * 2                   # (tile, kb) whose sums the buffer holds
    acc_writing = [False, False]
    acc_released = [E, E]              # warps that released the buffer's current contents
    readers = [set(), set()]           # warps reading each buffer now
    scales = [None, None]              # tile whose scales each buffer holds
    scale_users = [set(), set()]       # warps whose current tile reads the buffer
    tma = []                           # (stage, (tile, kb))
    mma = []                           # FIFO of (stage, buf, (tile, kb))
    copies = []                        # (buf, tile, warp)
    warp_copies = [0] * E

    def producer():
        it = 0
        for t in range(tiles):
            for kb in range(KB):
                st, ph = it % S, (it // S) & 1
                while not empty[st].try_wait(ph ^ 1):
                    yield
                if stage_reader[st] is not None:
                    raise AssertionError(f"stage {st} refilled while the MMA of {stage_reader[st]} reads it")
                full[st].arrive(expect_tx=1)
                stage[st] = "busy"
                tma.append((st, (t, kb)))
                it += 1
                yield

    def mma_thread():
        it = acc_i = 0
        for t in range(tiles):
            for kb in range(KB):
                st, ph = it % S, (it // S) & 1
                buf = acc_i & 1
                while not full[st].try_wait(ph):
                    yield
                if mma_waits_tempty:
                    while not tempty[buf].try_wait((acc_i >> 1) & 1):
                        yield
                if stage[st] != (t, kb):
                    raise AssertionError(f"MMA of {(t, kb)} read stage {st} holding {stage[st]}")
                if acc_released[buf] != E or readers[buf]:
                    raise AssertionError(f"MMA of {(t, kb)} writes buffer {buf} before its release")
                acc_released[buf] = 0
                acc_writing[buf] = True
                stage_reader[st] = (t, kb)
                mma.append((st, buf, (t, kb)))
                it += 1
                acc_i += 1
                yield

    def epilogue(w):
        for b in range(2):             # pre-fill, release once
            tempty[b].arrive()
        scales_fetch(w, 0, 0)
        while warp_copies[w]:
            yield
        sready[0].arrive()
        acc_i = 0
        for t in range(tiles):
            sb = t & 1
            if not prefetch_after_sready and t + 1 < tiles:
                scales_fetch(w, sb ^ 1, t + 1)
            while not sready[sb].try_wait((t >> 1) & 1):
                yield
            scale_users[sb].add(w)
            if prefetch_after_sready and t + 1 < tiles:
                scales_fetch(w, sb ^ 1, t + 1)
            for kb in range(KB):
                buf = acc_i & 1
                while not tfull[buf].try_wait((acc_i >> 1) & 1):
                    yield
                if acc[buf] != (t, kb) or acc_writing[buf]:
                    raise AssertionError(f"warp {w} read buffer {buf} for {(t, kb)}: holds {acc[buf]}")
                if scales[sb] != t:
                    raise AssertionError(f"warp {w} read scales of tile {scales[sb]} for tile {t}")
                readers[buf].add(w)
                if not release_after_reads:
                    acc_released[buf] += 1
                    tempty[buf].arrive()
                yield                  # the loads, the rescale, the re-fill
                if acc[buf] != (t, kb) or acc_writing[buf]:
                    raise AssertionError(f"buffer {buf} rewritten while warp {w} read {(t, kb)}")
                readers[buf].discard(w)
                if release_after_reads:
                    acc_released[buf] += 1
                    tempty[buf].arrive()
                acc_i += 1
            scale_users[sb].discard(w)
            while warp_copies[w]:
                yield
            sready[sb ^ 1].arrive()
            yield                      # bias, BF16 stores

    def scales_fetch(w, buf, t):
        warp_copies[w] += 1
        copies.append((buf, t, w))

    agents = [producer(), mma_thread()] + [epilogue(w) for w in range(E)]
    weights = [1.0, 1.0] + [bias(w, rng) if bias else 1.0 for w in range(E)]
    live = list(range(len(agents)))
    steps = 0
    while live or tma or mma or copies:
        steps += 1
        if steps > 500000:
            raise AssertionError("no progress")
        r = rng.random()
        if tma and (not live or r < 0.15):
            st, item = tma.pop(rng.randrange(len(tma)))
            stage[st] = item
            full[st].complete_tx(1)
            continue
        if mma and (not live or r < 0.30):
            st, buf, item = mma.pop(0)             # commits complete in issue order
            acc[buf] = item
            acc_writing[buf] = False
            stage_reader[st] = None
            empty[st].arrive()
            tfull[buf].arrive()
            continue
        if copies and (not live or r < 0.40):
            buf, t, w = copies.pop(rng.randrange(len(copies)))
            if scale_users[buf]:
                raise AssertionError(f"scales of tile {t} landed in buffer {buf} while warps {scale_users[buf]} read it")
            scales[buf] = t
            warp_copies[w] -= 1
            continue
        i = rng.choices(live, weights=[weights[j] for j in live])[0]
        try:
            next(agents[i])
        except StopIteration:
            live.remove(i)
    return steps


def _biases():
    yield None
    yield lambda w, rng: 0.2 if w in (0, 1) else 1.0       # the warps next to the producer and MMA lag
    yield lambda w, rng: 6.0 if w == 7 else 1.0            # one warp races ahead
    yield lambda w, rng: rng.uniform(0.05, 10.0)


def test_pipeline_holds_under_random_schedules():
    for b, bias in enumerate(_biases()):
        for seed in range(200):
            run(tiles=5, KB=6, seed=1000 * b + seed, bias=bias)
    for seed in range(200):
        run(tiles=7, KB=1, seed=seed)          # one K block per tile: both buffers per tile boundary


@pytest.mark.parametrize("control", ["mma skips tempty", "release before reads",
                                     "prefetch before sready"])
def test_controls_are_caught(control):
    kw = {"mma skips tempty": dict(mma_waits_tempty=False),
          "release before reads": dict(release_after_reads=False),
          "prefetch before sready": dict(prefetch_after_sready=False)}[control]
    caught = 0
    for b, bias in enumerate(_biases()):
        for seed in range(60):
            try:
                run(tiles=5, KB=6, seed=1000 * b + seed, bias=bias, **kw)
            except AssertionError:
                caught += 1
    assert caught > 0, control
