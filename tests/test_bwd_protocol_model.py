"""A discrete-event model of the backward kernels' barrier protocol (CPU
only), in the style of the forward's model: the issuer (step tiles through
a 4-stage ring loaded one step ahead; per step j, in dQ the S/dP MMAs of
step j then the accumulation of step j-2, in dKdV the other way round), two
row groups taking alternate steps, and the barriers between them.

Two variants, as in csrc/attention_bwd.cu:
  dQ    a group's S/dP columns are reused once the group has read them
        (sfree); its dS columns once the previous accumulation finished
        (x_free, waited by the group).
  dKdV  P^T and dS^T are written over the group's own S/dP columns, so the
        issuer waits for the group's previous accumulation (x_free) before
        its next S/dP.

Hazard checks: a stage is never reloaded before the accumulation of the step
it holds has finished, an MMA only reads a stage holding its own step, a
burst never overwrites S/dP (or the P/dS stored over them) that is still to
be read, a group's dS is never overwritten before its accumulation read it,
and every role finishes.  The planted mistakes (dKdV without the x_free
wait, and a stage reloaded without waiting for its accumulation) must be
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


def simulate(n, seed, member_rate, variant, skip_xfree_wait=False, skip_empty_wait=False,
             acc_cycles=300):
    stages = NS
    sim = Sim(seed)
    rng = sim.rng
    full = [Barrier("full%d" % s, 1) for s in range(stages)]
    empty = [Barrier("empty%d" % s, 1) for s in range(stages)]
    s_ready = [Barrier("s_ready%d" % w, 1) for w in range(2)]
    sfree = [Barrier("sfree%d" % w, 128) for w in range(2)]
    x_ready = [Barrier("x_ready%d" % w, 128) for w in range(2)]
    x_free = [Barrier("x_free%d" % w, 1) for w in range(2)]
    own = Barrier("own", 256)
    # stage contents: step held, landed, accumulation finished
    stage = {}
    # tensor memory per group: the step whose S/dP the columns hold, how many
    # of the group's four warps have read it; dS (dQ) or P/dS (dKdV) written
    cols = [{"step": None, "read": 4, "x": None, "x_used": True} for _ in range(2)]
    # dQ: the dS columns of each group, per warp (each warp writes its rows)
    dq_x = [[{"step": None, "used": True} for _ in range(4)] for _ in range(2)]

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
        if variant == "dkdv" and not c["x_used"]:
            raise Hazard("S/dP of step %d overwrites group %d's P/dS of step %d before "
                         "its accumulation" % (j, w, c["x"]))
        use_stage(j)
        c.update(step=j, read=0)

    def accumulate_mma(j):
        w = j & 1
        use_stage(j)
        if variant == "dkdv":
            c = cols[w]
            if c["x"] != j:
                raise Hazard("accumulation of step %d reads P/dS of step %s" % (j, c["x"]))
        elif any(x["step"] != j for x in dq_x[w]):
            raise Hazard("accumulation of step %d reads dS of steps %s"
                         % (j, [x["step"] for x in dq_x[w]]))

    def stage_done(j):
        stage[j % stages][2] = True

    def x_done(j):
        w = j & 1
        if variant == "dkdv":
            cols[w]["x_used"] = True
        else:
            for x in dq_x[w]:
                x["used"] = True

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
            if variant == "dkdv" and j >= 2:
                yield from accumulate(j - 2)
            yield ("wait", full[j % stages], (j // stages) & 1)
            if k > 0:
                if variant == "dq":
                    yield ("wait", sfree[w], (k - 1) & 1)
                elif not skip_xfree_wait:
                    yield ("wait", x_free[w], (k - 1) & 1)
            burst(j)
            yield mma(700, [s_ready[w]])
            if variant == "dq" and j >= 2:
                yield from accumulate(j - 2)
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
            if variant == "dq":
                yield ("arrive", sfree[w], 32)
            busy = rng.random() < member_rate
            yield ("delay", rng.randint(lo, hi) if busy else rng.randint(20, 200))
            if variant == "dq":
                if k > 0:
                    yield ("wait", x_free[w], (k - 1) & 1)
                x = dq_x[w][quad]
                if not x["used"]:
                    raise Hazard("group %d warp %d overwrites dS of step %s" % (w, quad, x["step"]))
                x.update(step=j, used=False)
            else:
                c.update(x=j, x_used=False)
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


@pytest.mark.parametrize("variant", ["dq", "dkdv"])
def test_backward_protocol_has_no_hazard(variant):
    for n, seed, rate, acc in schedules(300):
        try:
            result = simulate(n, seed, rate, variant, acc_cycles=acc)
        except Hazard as e:
            pytest.fail("%s n=%d seed=%d: %s" % (variant, n, seed, e))
        assert result == "ok", "%s n=%d seed=%d: %s" % (variant, n, seed, result)


def test_dkdv_without_accumulation_wait_is_caught():
    caught = 0
    for n, seed, rate, acc in schedules(300):
        try:
            caught += simulate(n, seed, rate, "dkdv", skip_xfree_wait=True, acc_cycles=acc) != "ok"
        except Hazard:
            caught += 1
    assert caught > 0, "the model no longer sees P/dS overwritten before its accumulation"


def test_reload_without_empty_wait_is_caught():
    caught = 0
    for n, seed, rate, acc in schedules(300):
        try:
            caught += simulate(n, seed, rate, "dq", skip_empty_wait=True, acc_cycles=acc) != "ok"
        except Hazard:
            caught += 1
    assert caught > 0, "the model no longer sees a stage reloaded under its accumulation"
