"""A discrete-event model of the backward kernels' barrier protocol (CPU
only), in the style of the forward's model: the issuer (step tiles through
a 4-stage ring loaded one step ahead; per step j the accumulation of step
j-2, then the S/dP MMAs of step j), two row groups taking alternate steps,
and the barriers between them.  As in both kernels of csrc/attention_bwd.cu,
a group writes its P/dS over its own S/dP columns, so the issuer waits for
the group's previous accumulation (x_free) before its next S/dP.

Hazard checks: a stage is never reloaded before the accumulation of the step
it holds has finished, an MMA only reads a stage holding its own step, a
burst never overwrites S/dP (or the P/dS stored over them) that is still to
be read, a group's dS is never overwritten before its accumulation read it,
and every role finishes.  The planted mistakes (no x_free wait before an
S/dP, and a stage reloaded without waiting for its accumulation) must be
caught.
"""
import random

import pytest

from test_ring_protocol_model import Barrier, Hazard, Sim

NS = 4
# tcgen05.mma is asynchronous: the issuing thread only blocks while the
# tensor pipe holds more than this many cycles of issued work, so it runs
# ahead of its MMAs
BACKLOG = 3000


class Then:
    """A commit that records what the finished MMAs released, then arrives."""

    def __init__(self, fn, bar):
        self.fn, self.bar, self.name = fn, bar, bar.name

    def arrive(self, sim, weight=1, tx=0):
        self.fn()
        self.bar.arrive(sim, weight, tx)


def simulate(n, seed, member_rate, skip_xfree_wait=False, skip_empty_wait=False,
             acc_cycles=300):
    stages = NS
    sim = Sim(seed)
    rng = sim.rng
    full = [Barrier("full%d" % s, 1) for s in range(stages)]
    empty = [Barrier("empty%d" % s, 1) for s in range(stages)]
    s_ready = [Barrier("s_ready%d" % w, 1) for w in range(2)]
    x_ready = [Barrier("x_ready%d" % w, 128) for w in range(2)]
    x_free = [Barrier("x_free%d" % w, 1) for w in range(2)]
    own = Barrier("own", 256)
    # stage contents: step held, landed, accumulation finished
    stage = {}
    # tensor memory per group: the step whose S/dP the columns hold, how many
    # of the group's four warps have read it, the step whose P/dS each warp
    # has written over its own lanes, and whether the accumulation that reads
    # them has finished
    cols = [{"step": None, "read": 4, "x": [None] * 4, "x_used": True} for _ in range(2)]

    def start_load(j):
        s = j % stages
        held = stage.get(s)
        if held is not None and not held[2]:
            raise Hazard("stage %d reloaded with step %d while step %d is unfinished"
                         % (s, j, held[0]))
        stage[s] = [j, False, False]

    def landed(j):
        s = j % stages
        if stage[s][0] == j:
            stage[s][1] = True

    def use_stage(j):
        held = stage.get(j % stages)
        if held is None or held[0] != j or not held[1]:
            raise Hazard("MMA of step %d read stage %d holding %s" % (j, j % stages, held))

    def burst(j):
        w = j & 1
        c = cols[w]
        if c["step"] is not None and c["read"] < 4:
            raise Hazard("S/dP of step %d overwrites group %d's unread step %d"
                         % (j, w, c["step"]))
        if not c["x_used"]:
            raise Hazard("S/dP of step %d overwrites group %d's P/dS of steps %s before "
                         "their accumulation" % (j, w, c["x"]))
        use_stage(j)
        c.update(step=j, read=0)

    def accumulate_mma(j):
        w = j & 1
        use_stage(j)
        c = cols[w]
        if any(x != j for x in c["x"]):
            raise Hazard("accumulation of step %d reads P/dS of steps %s" % (j, c["x"]))
        c["x_used"] = False

    def stage_done(j):
        stage[j % stages][2] = True

    def x_done(j):
        cols[j & 1]["x_used"] = True

    def mma(cycles, commits):
        """Queue MMAs on the in-order pipe; their commits arrive when the pipe
        reaches them.  Returns the issuer's own delay."""
        start = max(sim.now, sim.pipe_free)
        sim.pipe_free = start + cycles
        for bar in commits:
            sim.at(sim.pipe_free - sim.now + rng.randint(0, 50),
                   lambda bar=bar: bar.arrive(sim, 1))
        return ("delay", max(20, sim.pipe_free - sim.now - BACKLOG))

    def issuer():
        yield ("wait", own, 0)
        if n > 0:
            start_load(0)
            yield ("copy", full[0], 100, lambda: landed(0))

        def accumulate(j):
            w = j & 1
            yield ("wait", x_ready[w], (j >> 1) & 1)
            accumulate_mma(j)
            yield mma(acc_cycles, [Then(lambda j=j: x_done(j), x_free[w]),
                            Then(lambda j=j: stage_done(j), empty[j % stages])])

        for j in range(n):
            w, k = j & 1, j >> 1
            if j + 1 < n:
                if j + 1 >= stages and not skip_empty_wait:
                    yield ("wait", empty[(j + 1) % stages], ((j + 1 - stages) // stages) & 1)
                start_load(j + 1)
                yield ("copy", full[(j + 1) % stages], 100, lambda j=j: landed(j + 1))
            if j >= 2:
                yield from accumulate(j - 2)
            yield ("wait", full[j % stages], (j // stages) & 1)
            if k > 0 and not skip_xfree_wait:
                yield ("wait", x_free[w], (k - 1) & 1)
            burst(j)
            yield mma(700, [s_ready[w]])
        for jj in range(max(0, n - 2), n):
            yield from accumulate(jj)

    def group_warp(w, quad):
        yield ("delay", rng.randint(50, 600))
        yield ("arrive", own, 32)
        lo = rng.choice([10, 300, 800])
        hi = lo + rng.choice([100, 2000, 8000])
        for k, j in enumerate(range(w, n, 2)):
            yield ("wait", s_ready[w], k & 1)
            c = cols[w]
            if c["step"] != j:
                raise Hazard("group %d read S/dP of step %s for step %d" % (w, c["step"], j))
            yield ("delay", rng.randint(50, 150))
            c["read"] += 1
            busy = rng.random() < member_rate
            yield ("delay", rng.randint(lo, hi) if busy else rng.randint(20, 200))
            # P/dS over the warp's own lanes of the S/dP columns just read
            c["x"][quad] = j
            yield ("delay", rng.randint(30, 100))
            yield ("arrive", x_ready[w], 32)

    roles = {"issuer": issuer()}
    for w in range(2):
        for quad in range(4):
            roles["group%d.%d" % (w, quad)] = group_warp(w, quad)
    sim.roles = roles
    return sim.run()


STEP_COUNTS = (1, 2, 3, 4, 5, 7, 9, 16, 33, 60)


def schedules(count):
    for trial in range(count):
        rng = random.Random(trial)
        yield (rng.choice(STEP_COUNTS), 9100 + trial, rng.choice([0.3, 0.8, 1.0]),
               rng.choice([300, 1500, 4000]))


def test_backward_protocol_has_no_hazard():
    for n, seed, rate, acc in schedules(600):
        try:
            result = simulate(n, seed, rate, acc_cycles=acc)
        except Hazard as e:
            pytest.fail("n=%d seed=%d: %s" % (n, seed, e))
        assert result == "ok", "n=%d seed=%d: %s" % (n, seed, result)


def test_burst_without_accumulation_wait_is_caught():
    caught = 0
    for n, seed, rate, acc in schedules(300):
        try:
            caught += simulate(n, seed, rate, skip_xfree_wait=True, acc_cycles=acc) != "ok"
        except Hazard:
            caught += 1
    assert caught > 0, "the model no longer sees P/dS overwritten before its accumulation"


def test_reload_without_empty_wait_is_caught():
    caught = 0
    for n, seed, rate, acc in schedules(300):
        try:
            caught += simulate(n, seed, rate, skip_empty_wait=True, acc_cycles=acc) != "ok"
        except Hazard:
            caught += 1
    assert caught > 0, "the model no longer sees a stage reloaded under its accumulation"
