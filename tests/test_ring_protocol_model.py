"""A discrete-event model of the attention kernel's barrier protocol, checked
for hazards on randomised schedules (CPU only).

The model follows csrc/attention.cu role by role: the K copy warps (one per
64-column box and step parity, 8-stage ring), the V copy warps (one per box
over every step, 5-stage ring), the score-burst issuer (one N=128 burst per
step pair), the PV issuer (step order) and the eight softmax warps.

mbarriers are modelled with their arrival count, transaction bytes and
phase. A parity wait passes when the current phase's parity differs from the
one asked for, as `mbarrier.try_wait.parity` does. tcgen05.commit arrives
when an in-order MMA pipe reaches it. Copy and compute latencies are drawn
at random, with occasional very slow copies.

Hazard checks: a ring stage is never overwritten before its MMA consumed
it, an MMA only reads a stage holding its own step with every box landed,
no barrier gets more arrivals than its count, and every role finishes (no
deadlock). The planted mistake is the V ring split by step parity with
independent PV queues. With an odd ring length a warp can then test a
stage's barrier two phases behind. The model must catch it.
"""
import heapq
import itertools
import random

import pytest

KS, VS = 8, 5


class Hazard(Exception):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, count, 0, 0
        self.waiters = []

    def passed(self, parity):
        return (self.phase & 1) != parity

    def _maybe_complete(self, sim):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count
            waiters, self.waiters = self.waiters, []
            for role in waiters:
                sim.resume(role)

    def arrive(self, sim, weight=1, tx=0):
        self.tx += tx
        self.pending -= weight
        if self.pending < 0:
            raise Hazard("more arrivals than the count on " + self.name)
        self._maybe_complete(sim)

    def complete_tx(self, sim, nbytes):
        self.tx -= nbytes
        self._maybe_complete(sim)


class Sim:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.now = 0
        self.queue = []
        self.seq = itertools.count()
        self.roles = {}
        self.blocked = {}
        self.done = set()
        self.pipe_free = 0

    def at(self, delay, fn):
        heapq.heappush(self.queue, (self.now + delay, next(self.seq), fn))

    def resume(self, role):
        if self.blocked.pop(role, None) is not None:
            self.at(self.rng.randint(20, 150), lambda: self.step(role))

    def step(self, role):
        try:
            act = next(self.roles[role])
        except StopIteration:
            self.done.add(role)
            return
        kind = act[0]
        if kind == "delay":
            self.at(act[1], lambda: self.step(role))
        elif kind == "wait":
            bar, parity = act[1], act[2]
            if bar.passed(parity):
                self.at(self.rng.randint(20, 150), lambda: self.step(role))
            else:
                self.blocked[role] = (bar.name, parity)
                bar.waiters.append(role)
        elif kind == "poll":
            self.at(self.rng.randint(10, 60), lambda: self.step(role))
        elif kind == "arrive":
            act[1].arrive(self, act[2])
            self.at(self.rng.randint(1, 30), lambda: self.step(role))
        elif kind == "copy":  # arrive.expect_tx, then the bytes land later
            bar, nbytes, land = act[1], act[2], act[3]
            bar.arrive(self, 1, tx=nbytes)
            slow = self.rng.random() < 0.1
            latency = self.rng.randint(6000, 40000) if slow else self.rng.randint(300, 6000)

            def landed(bar=bar, nbytes=nbytes, land=land):
                land()
                bar.complete_tx(self, nbytes)
            self.at(latency, landed)
            self.at(self.rng.randint(200, 900), lambda: self.step(role))
        elif kind == "mma":  # in-order pipe; commits arrive when it gets there
            cycles, commits = act[1], act[2]
            start = max(self.now, self.pipe_free)
            self.pipe_free = start + cycles
            for bar in commits:
                self.at(self.pipe_free - self.now + self.rng.randint(0, 50),
                        lambda bar=bar: bar.arrive(self, 1))
            self.at(max(50, start - self.now + cycles // 2), lambda: self.step(role))
        else:
            raise ValueError(kind)

    def run(self, limit=5e7):
        for role in self.roles:
            self.at(self.rng.randint(0, 100), lambda role=role: self.step(role))
        while self.queue:
            t, _, fn = heapq.heappop(self.queue)
            if t > limit:
                return "timeout"
            self.now = t
            fn()
        return "ok" if len(self.done) == len(self.roles) else "deadlock"


class Ring:
    """Stage occupancy: which step a stage holds, how many boxes landed,
    whether its MMA has consumed it."""

    def __init__(self, name, boxes):
        self.name, self.boxes, self.stage = name, boxes, {}

    def start(self, s, j, box):
        held = self.stage.get((s, box))
        if held is not None and held[0] != j and not held[2]:
            raise Hazard("%s stage %d box %d overwritten by step %d before step %d was used"
                         % (self.name, s, box, j, held[0]))
        self.stage[(s, box)] = [j, False, False]

    def land(self, s, j, box):
        if self.stage[(s, box)][0] == j:
            self.stage[(s, box)][1] = True

    def consume(self, s, j):
        for box in range(self.boxes):
            held = self.stage.get((s, box))
            if held is None or held[0] != j or not held[1]:
                raise Hazard("MMA of step %d read %s stage %d box %d holding %s"
                             % (j, self.name, s, box, held))
            held[2] = True


def simulate(n, seed, member_rate, parity_split_v=False):
    """One CTA walking n steps; returns 'ok', 'deadlock' or 'timeout' and
    raises Hazard on a data hazard."""
    sim = Sim(seed)
    rng = sim.rng
    kfull = [Barrier("kfull%d" % s, 2) for s in range(KS)]
    kempty = [Barrier("kempty%d" % s, 1) for s in range(KS)]
    vfull = [Barrier("vfull%d" % s, 1 if parity_split_v else 2) for s in range(VS)]
    vempty = [Barrier("vempty%d" % s, 1) for s in range(VS)]
    qready, bar_s, sfree = Barrier("qready", 128), Barrier("s", 1), Barrier("sfree", 256)
    bar_p = [Barrier("p%d" % w, 128) for w in range(2)]
    bar_o = [Barrier("o%d" % w, 1) for w in range(2)]
    kring, vring = Ring("K", 2), Ring("V", 1 if parity_split_v else 2)
    keeps = {}

    def member(j, half):
        if (j, half) not in keeps:
            keeps[(j, half)] = rng.random() < member_rate
        return keeps[(j, half)]

    def k_copier(parity, box):
        for j in range(parity, n, 2):
            s = j % KS
            if j >= KS:
                yield ("wait", kempty[s], ((j // KS) - 1) & 1)
            kring.start(s, j, box)
            yield ("copy", kfull[s], 8192, lambda s=s, j=j: kring.land(s, j, box))

    def v_copier_box(box):
        for j in range(n):
            s = j % VS
            if j >= VS:
                yield ("wait", vempty[s], ((j // VS) - 1) & 1)
            vring.start(s, j, box)
            yield ("copy", vfull[s], 8192, lambda s=s, j=j: vring.land(s, j, box))

    def v_copier_parity(parity):  # the planted mistake
        for j in range(parity, n, 2):
            s = j % VS
            if j >= VS:
                yield ("wait", vempty[s], ((j // VS) - 1) & 1)
            vring.start(s, j, 0)
            yield ("copy", vfull[s], 16384, lambda s=s, j=j: vring.land(s, j, 0))

    def score_issuer():
        yield ("wait", qready, 0)
        for t in range((n + 1) // 2):
            j0, s0 = 2 * t, (2 * t) % KS
            two = j0 + 1 < n
            yield ("wait", kfull[s0], (j0 // KS) & 1)
            if two:
                yield ("wait", kfull[s0 + 1], ((j0 + 1) // KS) & 1)
            if t > 0:
                yield ("wait", sfree, (t - 1) & 1)
            kring.consume(s0, j0)
            if two:
                kring.consume(s0 + 1, j0 + 1)
            yield ("mma", 600 if two else 350,
                   [bar_s, kempty[s0]] + ([kempty[s0 + 1]] if two else []))

    def pv_issuer_in_order():
        for j in range(n):
            w, s = j & 1, j % VS
            yield ("wait", vfull[s], (j // VS) & 1)
            yield ("wait", bar_p[w], (j >> 1) & 1)
            vring.consume(s, j)
            yield ("mma", 300, [bar_o[w], vempty[s]])

    def pv_issuer_two_queues():  # goes with the planted mistake
        nxt = [0, 1]
        while nxt[0] < n or nxt[1] < n:
            issued = False
            for w in range(2):
                j = nxt[w]
                if j < n and bar_p[w].passed((j >> 1) & 1) and vfull[j % VS].passed((j // VS) & 1):
                    vring.consume(j % VS, j)
                    yield ("mma", 300, [bar_o[w], vempty[j % VS]])
                    nxt[w] += 2
                    issued = True
            if not issued:
                yield ("poll",)

    def softmax_warp(w, quad):
        if w == 0:
            yield ("delay", rng.randint(100, 800))
            yield ("arrive", qready, 32)
        lo = rng.choice([10, 300, 600])
        hi = lo + rng.choice([100, 2000, 10000])
        for k, j in enumerate(range(w, n, 2)):
            yield ("wait", bar_s, k & 1)
            yield ("delay", rng.randint(50, 150))
            yield ("arrive", sfree, 32)
            busy = member(j, quad // 2)
            yield ("delay", rng.randint(lo, hi) if busy else rng.randint(20, 200))
            if k > 0:
                yield ("wait", bar_o[w], (k - 1) & 1)
            yield ("delay", rng.randint(50, 150))
            yield ("arrive", bar_p[w], 32)
        steps = len(range(w, n, 2))
        if steps:
            yield ("wait", bar_o[w], (steps - 1) & 1)

    roles = {"k0e": k_copier(0, 0), "k0o": k_copier(1, 0),
             "k1e": k_copier(0, 1), "k1o": k_copier(1, 1), "qk": score_issuer()}
    if parity_split_v:
        roles.update({"ve": v_copier_parity(0), "vo": v_copier_parity(1),
                      "pv": pv_issuer_two_queues()})
    else:
        roles.update({"v0": v_copier_box(0), "v1": v_copier_box(1), "pv": pv_issuer_in_order()})
    for w in range(2):
        for quad in range(4):
            roles["softmax%d.%d" % (w, quad)] = softmax_warp(w, quad)
    sim.roles = roles
    return sim.run()


STEP_COUNTS = (1, 2, 3, 5, 6, 9, 12, 17, 40, 41, 101)


def schedules(count):
    for trial in range(count):
        rng = random.Random(trial)
        yield rng.choice(STEP_COUNTS), 7000 + trial, rng.choice([0.3, 0.82, 1.0])


def test_kernel_protocol_has_no_hazard():
    for n, seed, rate in schedules(400):
        try:
            result = simulate(n, seed, rate)
        except Hazard as e:
            pytest.fail("n=%d seed=%d: %s" % (n, seed, e))
        assert result == "ok", "n=%d seed=%d: %s" % (n, seed, result)


def test_parity_split_v_ring_is_caught():
    caught = 0
    for n, seed, rate in schedules(400):
        try:
            caught += simulate(n, seed, rate, parity_split_v=True) != "ok"
        except Hazard:
            caught += 1
    assert caught > 0, "the model no longer sees the two-phase ring hazard"
