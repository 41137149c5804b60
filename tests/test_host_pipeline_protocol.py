"""A randomized CPU model of w8a8_linear_host's stream protocol.  The entry point enqueues,
in this order, on the copy-in stream H, the caller's stream S and the copy-out stream D:

    record(start, S); wait(H, start); wait(D, start)
    for chunk i (buffer b = i % 2):
        if i >= 2: wait(H, comp_done[b])          x buffer b no longer read by chunk i - 2
        H: copy x chunk i -> xbuf[b];   record(h2d_done[b], H)
        wait(S, h2d_done[b]);  if i >= 2: wait(S, d2h_done[b])
        S: quantize + GEMM xbuf[b] -> ybuf[b];   record(comp_done[b], S)
        wait(D, comp_done[b])
        D: copy ybuf[b] -> y chunk i;   record(d2h_done[b], D)
    record(start, H); wait(S, start); wait(S, d2h_done) for the last two chunks

with CUDA's semantics: operations on a stream run in order, a wait makes its stream
wait for the event's most recent record at the time the wait was enqueued.  Copies and
the compute take time (they start, then end).  The model runs random schedules and
checks that no copy or compute touches a buffer that another one still uses with a
conflicting access, that every chunk reads the data of its own chunk, and that the
caller's stream reaches its end only after every copy back has ended.  Controls that drop
one of the waits must be caught."""
import random

import pytest


def run(nch, seed, drop=None):
    rng = random.Random(seed)
    streams = {"H": [], "S": [], "D": []}
    events = {}                       # name -> number of records enqueued so far
    fired = {}                        # name -> number of records executed

    def record(stream, ev):
        events[ev] = events.get(ev, 0) + 1
        streams[stream].append(("record", ev, events[ev]))

    def wait(stream, ev):
        streams[stream].append(("wait", ev, events.get(ev, 0)))

    def work(stream, name, reads, writes, chunk):
        streams[stream].append(("work", name, reads, writes, chunk))

    record("S", "start")
    wait("H", "start")
    wait("D", "start")
    for i in range(nch):
        b = i & 1
        if i >= 2 and drop != "H waits comp_done":
            wait("H", f"comp{b}")
        work("H", "copy in", [], [f"x{b}"], i)
        record("H", f"h2d{b}")
        wait("S", f"h2d{b}")
        if i >= 2 and drop != "S waits d2h_done":
            wait("S", f"d2h{b}")
        work("S", "linear", [f"x{b}", "ws"], [f"y{b}", "ws"], i)
        record("S", f"comp{b}")
        wait("D", f"comp{b}")
        work("D", "copy out", [f"y{b}"], [], i)
        record("D", f"d2h{b}")
    if drop != "final waits":
        record("H", "start")
        wait("S", "start")
        for i in range(max(0, nch - 2), nch):
            wait("S", f"d2h{i & 1}")
    streams["S"].append(("end",))

    holds = {}                        # buffer -> chunk whose data it holds
    users = {}                        # buffer -> list of (op, mode) in progress
    running = {}                      # stream -> op in progress
    copied_out = set()

    def can_start(op):
        if op[0] == "wait":
            return fired.get(op[1], 0) >= op[2]
        return True

    steps = 0
    while any(streams.values()) or running:
        steps += 1
        if steps > 100000:
            raise AssertionError("no progress")
        choices = [s for s in streams if s in running or (streams[s] and can_start(streams[s][0]))]
        if not choices:
            raise AssertionError("deadlock")
        s = rng.choice(choices)
        if s in running:                           # finish the running work
            op = running.pop(s)
            _, name, reads, writes, i = op
            for buf in reads + writes:
                users[buf].remove((name, i))
            for buf in writes:
                holds[buf] = i
            if name == "copy out":
                copied_out.add(i)
            continue
        op = streams[s].pop(0)
        if op[0] == "record":
            fired[op[1]] = max(fired.get(op[1], 0), op[2])
        elif op[0] == "wait":
            pass
        elif op[0] == "end":
            if copied_out != set(range(nch)):
                raise AssertionError(f"the caller's stream ended before copies {set(range(nch)) - copied_out} were back")
        else:
            _, name, reads, writes, i = op
            for buf in reads:
                if buf != "ws" and holds.get(buf) != i:
                    raise AssertionError(f"{name} of chunk {i} reads {buf} holding chunk {holds.get(buf)}")
                if any(n != name for n, _ in users.get(buf, [])):
                    raise AssertionError(f"{name} of chunk {i} reads {buf} while {users[buf]} use it")
            for buf in writes:
                if users.get(buf):
                    raise AssertionError(f"{name} of chunk {i} writes {buf} while {users[buf]} use it")
            for buf in reads + writes:
                users.setdefault(buf, []).append((name, i))
            running[s] = op
    return steps


@pytest.mark.parametrize("nch", [1, 2, 3, 8])
def test_host_pipeline_holds_under_random_schedules(nch):
    for seed in range(400):
        run(nch, seed)


@pytest.mark.parametrize("drop", ["H waits comp_done", "S waits d2h_done", "final waits"])
def test_dropped_waits_are_caught(drop):
    caught = 0
    for seed in range(400):
        try:
            run(8, seed, drop=drop)
        except AssertionError:
            caught += 1
    assert caught > 0, drop
