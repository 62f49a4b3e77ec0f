"""A discrete-event model of the backward kernels' barrier protocol (CPU
only), in the style of the forward's model.  Both kernels of
csrc/attention_bwd.cu take their steps in pairs: one N=128 burst per product
covers steps 2p and 2p+1, and row group g takes step 2p+g from its half of
the burst's columns.  Two threads issue MMAs into the one in-order tensor
pipe: one the bursts, one the accumulations.

dQ:   a copy warp fills a K ring (3 pair slots, freed by the accumulation)
      and a V ring (2 pair slots, freed by the dP burst); S(p) and dP(p)
      are issued once both groups have read pair p-1's S and dP, the
      accumulation of pair p (dQ += dS K) from each group's dS columns once
      the group has written them.  A group writes dS(p) into its own dS
      columns once the accumulation of pair p-1 has finished.
dKdV: the burst thread also loads a 2-slot ring; S^T(p) once dV of pair
      p-1 has finished (P^T is written over S^T), dP^T(p) once dK of pair
      p-1 has finished (dS^T over dP^T), with separate ready signals so the
      groups start P^T on S^T alone.  dV(p) from each group's P^T as it is
      stored; dK(p) from each group's dS^T, queued after S^T(p+1).

Hazard checks: no ring slot is reloaded before the MMAs that read it have
finished, every MMA reads a slot holding its own pair with its tiles
landed, no burst overwrites columns still to be read or accumulated, every
accumulation reads what its own pair wrote, the epilogue reads the
accumulators after every accumulation, and every role finishes.  The
planted mistakes (one wait left out at a time) must be caught.
"""
import random

import pytest

from test_ring_protocol_model import Barrier, Hazard, Sim

NK, NV, NR = 3, 2, 2
# tcgen05.mma is asynchronous: the issuing thread only blocks while the
# tensor pipe holds more than this many cycles of issued work
BACKLOG = 3000


def mma(sim, cycles, commits, finished=()):
    """Queue MMAs on the in-order pipe.  What they release is recorded when
    the pipe finishes them; their commits arrive after that.  Returns the
    issuer's own delay."""
    start = max(sim.now, sim.pipe_free)
    sim.pipe_free = start + cycles
    for fn in finished:
        sim.at(sim.pipe_free - sim.now, fn)
    for bar in commits:
        sim.at(sim.pipe_free - sim.now + sim.rng.randint(0, 50),
               lambda bar=bar: bar.arrive(sim, 1))
    return ("delay", max(20, sim.pipe_free - sim.now - BACKLOG))


class Slots:
    """A ring of pair slots: the pair a slot holds, whether its tiles have
    landed, and whether the MMAs reading it have finished."""

    def __init__(self, name, count):
        self.name, self.count, self.held = name, count, {}

    def load(self, p):
        s = p % self.count
        h = self.held.get(s)
        if h is not None and not h["done"]:
            raise Hazard("%s slot %d reloaded with pair %d while pair %d is in use"
                         % (self.name, s, p, h["pair"]))
        self.held[s] = {"pair": p, "landed": False, "done": False}

    def land(self, p):
        h = self.held[p % self.count]
        if h["pair"] == p:
            h["landed"] = True

    def use(self, p, what):
        h = self.held.get(p % self.count)
        if h is None or h["pair"] != p or not h["landed"]:
            raise Hazard("%s of pair %d read %s slot %d holding %s"
                         % (what, p, self.name, p % self.count, h))

    def release(self, p):
        h = self.held[p % self.count]
        if h["pair"] == p:
            h["done"] = True


def compute_time(rng):
    lo = rng.choice([10, 300, 800])
    return lo, lo + rng.choice([100, 2000, 8000])


def simulate_dq(n, seed, member_rate, skip=None, acc_cycles=512):
    sim = Sim(seed)
    rng = sim.rng
    pairs = (n + 1) // 2
    kfull = [Barrier("kfull%d" % s, 1) for s in range(NK)]
    kempty = [Barrier("kempty%d" % s, 1) for s in range(NK)]
    vfull = [Barrier("vfull%d" % s, 1) for s in range(NV)]
    vempty = [Barrier("vempty%d" % s, 1) for s in range(NV)]
    sd_ready = Barrier("sd_ready", 1)
    read = Barrier("read", 8)
    x_ready = [Barrier("x_ready%d" % g, 4) for g in range(2)]
    x_free = Barrier("x_free", 1)
    own = Barrier("own", 8)
    done = Barrier("done", 2)
    kring, vring = Slots("K", NK), Slots("V", NV)
    # tensor memory: the pair whose S / dP each group's columns hold and how
    # many of its warps read them; each warp's dS rows: the pair written and
    # whether the accumulation reading them has finished
    sd = [{"pair": None, "read": 4} for _ in range(2)]
    ds = [[{"pair": None, "free": True} for _ in range(4)] for _ in range(2)]
    acc = {"done": 0}

    def steps_in(p):
        return 2 if 2 * p + 1 < n else 1

    def loader():
        for p in range(pairs):
            if p >= NK and skip != "kempty":
                yield ("wait", kempty[p % NK], ((p - NK) // NK) & 1)
            kring.load(p)
            yield ("copy", kfull[p % NK], 100 * steps_in(p), lambda p=p: kring.land(p))
            if p >= NV:
                yield ("wait", vempty[p % NV], ((p - NV) // NV) & 1)
            vring.load(p)
            yield ("copy", vfull[p % NV], 100 * steps_in(p), lambda p=p: vring.land(p))

    def burst(p):
        for g in range(2):
            if sd[g]["pair"] is not None and sd[g]["read"] < 4:
                raise Hazard("S/dP of pair %d overwrite group %d's unread pair %d"
                             % (p, g, sd[g]["pair"]))
            sd[g].update(pair=p, read=0)
        kring.use(p, "S")
        vring.use(p, "dP")

    def accumulate_mma(q, g):
        kring.use(q, "accumulation")
        if any(x["pair"] != q for x in ds[g]):
            raise Hazard("accumulation of pair %d reads group %d's dS of pairs %s"
                         % (q, g, [x["pair"] for x in ds[g]]))
        for x in ds[g]:
            x["free"] = False

    def acc_done(q):
        for g in range(2):
            for x in ds[g]:
                if x["pair"] == q:
                    x["free"] = True
        acc["done"] += steps_in(q)

    def burst_issuer():
        yield ("wait", own, 0)
        for p in range(pairs):
            yield ("wait", kfull[p % NK], (p // NK) & 1)
            yield ("wait", vfull[p % NV], (p // NV) & 1)
            if p > 0 and skip != "read":
                yield ("wait", read, (p - 1) & 1)
            burst(p)
            yield mma(sim, 1024, [sd_ready, vempty[p % NV]], [lambda p=p: vring.release(p)])
        yield mma(sim, 1, [done])

    def acc_issuer():
        for q in range(pairs):
            for g in range(steps_in(q)):
                yield ("wait", x_ready[g], q & 1)
                accumulate_mma(q, g)
            yield mma(sim, acc_cycles * steps_in(q), [x_free, kempty[q % NK]],
                      [lambda q=q: acc_done(q), lambda q=q: kring.release(q)])
        yield mma(sim, 1, [done])

    def group_warp(g, quad):
        yield ("delay", rng.randint(50, 600))
        yield ("arrive", own, 1)
        lo, hi = compute_time(rng)
        for p in range(pairs):
            yield ("wait", sd_ready, p & 1)
            mine = 2 * p + g < n
            if mine:
                if sd[g]["pair"] != p:
                    raise Hazard("group %d read S/dP of pair %s for pair %d"
                                 % (g, sd[g]["pair"], p))
                yield ("delay", rng.randint(50, 150))
                sd[g]["read"] += 1
            yield ("arrive", read, 1)
            if not mine:
                continue
            busy = rng.random() < member_rate
            yield ("delay", rng.randint(lo, hi) if busy else rng.randint(20, 200))
            if p > 0 and skip != "x_free":
                yield ("wait", x_free, (p - 1) & 1)
            x = ds[g][quad]
            if not x["free"]:
                raise Hazard("group %d warp %d overwrites dS of pair %s before its accumulation"
                             % (g, quad, x["pair"]))
            x["pair"] = p
            yield ("delay", rng.randint(30, 100))
            yield ("arrive", x_ready[g], 1)
        yield ("wait", done, 0)
        if acc["done"] != n:
            raise Hazard("epilogue read dQ after %d of %d accumulations" % (acc["done"], n))

    roles = {"loader": loader(), "bursts": burst_issuer(), "accumulations": acc_issuer()}
    for g in range(2):
        for quad in range(4):
            roles["group%d.%d" % (g, quad)] = group_warp(g, quad)
    sim.roles = roles
    return sim.run()


def simulate_dkdv(n, seed, member_rate, skip=None, acc_cycles=512):
    sim = Sim(seed)
    rng = sim.rng
    pairs = (n + 1) // 2
    full = [Barrier("full%d" % s, 1) for s in range(NR)]
    s_ready = Barrier("s_ready", 1)
    dp_ready = Barrier("dp_ready", 1)
    st_issued = Barrier("st_issued", 1)
    p_ready = [Barrier("p_ready%d" % g, 4) for g in range(2)]
    ds_ready = [Barrier("ds_ready%d" % g, 4) for g in range(2)]
    xv_free = Barrier("xv_free", 1)
    xk_free = Barrier("xk_free", 1)
    own = Barrier("own", 8)
    done = Barrier("done", 2)
    ring = Slots("Q/dO", NR)
    # tensor memory per group and warp (each warp writes its own rows): the
    # S^T columns hold ("S", pair) until P^T is written over them, the dP^T
    # columns ("dP", pair) until dS^T; "used" once the accumulation reading
    # them has finished
    st = [[{"what": None, "pair": None, "used": True} for _ in range(4)] for _ in range(2)]
    dpt = [[{"what": None, "pair": None, "used": True} for _ in range(4)] for _ in range(2)]
    acc = {"dv": 0, "dk": 0, "released": {}}

    def steps_in(p):
        return 2 if 2 * p + 1 < n else 1

    def load(p):
        ring.load(p)
        yield ("copy", full[p % NR], 100 * steps_in(p), lambda p=p: ring.land(p))

    def burst(cols, what, p, reader):
        for g in range(2):
            for x in cols[g]:
                if not x["used"]:
                    raise Hazard("%s of pair %d overwrites %s of pair %s before %s read it"
                                 % (what, p, x["what"], x["pair"], reader))
                x.update(what=what, pair=p, used=False)
        ring.use(p, what)

    def accumulate_mma(cols, what, q, g):
        ring.use(q, "accumulation")
        for x in cols[g]:
            if x["what"] != what or x["pair"] != q:
                raise Hazard("accumulation of pair %d reads %s/%s for %s"
                             % (q, x["what"], x["pair"], what))

    def finished(cols, q, kind):
        for g in range(2):
            for x in cols[g]:
                if x["pair"] == q:
                    x["used"] = True
        acc[kind] += steps_in(q)
        acc["released"][q] = acc["released"].get(q, 0) + 1
        if acc["released"][q] == 2:
            ring.release(q)

    def burst_issuer():
        if pairs > 0:
            yield from load(0)
        if pairs > 1:
            yield from load(1)
        yield ("wait", own, 0)
        for p in range(pairs):
            yield ("wait", full[p % NR], (p // NR) & 1)
            if p > 0 and skip != "xv_free":
                yield ("wait", xv_free, (p - 1) & 1)
            burst(st, "S", p, "dV")
            yield mma(sim, 512, [s_ready])
            yield ("arrive", st_issued, 1)
            if p > 0 and skip != "xk_free":
                yield ("wait", xk_free, (p - 1) & 1)
            if 1 <= p and p + 1 < pairs:
                yield from load(p + 1)
            burst(dpt, "dP", p, "dK")
            yield mma(sim, 512, [dp_ready])
        yield mma(sim, 1, [done])

    def acc_issuer():
        for p in range(pairs):
            for g in range(steps_in(p)):
                yield ("wait", p_ready[g], p & 1)
                accumulate_mma(st, "P", p, g)
            yield mma(sim, acc_cycles * steps_in(p), [xv_free],
                      [lambda p=p: finished(st, p, "dv")])
            # dK after the next pair's S^T, so that its P^T phase starts early
            if p + 1 < pairs:
                yield ("wait", st_issued, (p + 1) & 1)
            for g in range(steps_in(p)):
                yield ("wait", ds_ready[g], p & 1)
                accumulate_mma(dpt, "dS", p, g)
            yield mma(sim, acc_cycles * steps_in(p), [xk_free],
                      [lambda p=p: finished(dpt, p, "dk")])
        yield mma(sim, 1, [done])

    def group_warp(g, quad):
        yield ("delay", rng.randint(50, 600))
        yield ("arrive", own, 1)
        lo, hi = compute_time(rng)
        for p in range(pairs):
            yield ("wait", s_ready, p & 1)
            if 2 * p + g >= n:
                continue
            x = st[g][quad]
            if x["what"] != "S" or x["pair"] != p:
                raise Hazard("group %d warp %d read %s/%s for S^T of pair %d"
                             % (g, quad, x["what"], x["pair"], p))
            yield ("delay", rng.randint(50, 150))
            busy = rng.random() < member_rate
            yield ("delay", rng.randint(lo, hi) if busy else rng.randint(20, 200))
            x["what"] = "P"
            yield ("arrive", p_ready[g], 1)
            if skip != "dp_ready":
                yield ("wait", dp_ready, p & 1)
            x = dpt[g][quad]
            if x["what"] != "dP" or x["pair"] != p:
                raise Hazard("group %d warp %d read %s/%s for dP^T of pair %d"
                             % (g, quad, x["what"], x["pair"], p))
            yield ("delay", rng.randint(30, 400))
            x["what"] = "dS"
            yield ("arrive", ds_ready[g], 1)
        yield ("wait", done, 0)
        if acc["dv"] != n or acc["dk"] != n:
            raise Hazard("epilogue read dK/dV after %d/%d of %d accumulations"
                         % (acc["dv"], acc["dk"], n))

    roles = {"bursts": burst_issuer(), "accumulations": acc_issuer()}
    for g in range(2):
        for quad in range(4):
            roles["group%d.%d" % (g, quad)] = group_warp(g, quad)
    sim.roles = roles
    return sim.run()


STEP_COUNTS = (0, 1, 2, 3, 4, 5, 7, 9, 16, 33, 60)
KERNELS = {"dq": simulate_dq, "dkdv": simulate_dkdv}


def schedules(count):
    for trial in range(count):
        rng = random.Random(trial)
        yield (rng.choice(STEP_COUNTS), 9100 + trial, rng.choice([0.3, 0.8, 1.0]),
               rng.choice([200, 512, 1500, 4000]))


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_backward_protocol_has_no_hazard(kernel):
    for n, seed, rate, acc in schedules(400):
        try:
            result = KERNELS[kernel](n, seed, rate, acc_cycles=acc)
        except Hazard as e:
            pytest.fail("%s n=%d seed=%d: %s" % (kernel, n, seed, e))
        assert result == "ok", "%s n=%d seed=%d: %s" % (kernel, n, seed, result)


@pytest.mark.parametrize("kernel,skip,what", [
    ("dq", "x_free", "dS overwritten before its accumulation"),
    ("dq", "read", "S/dP overwritten before both groups read them"),
    ("dq", "kempty", "a K slot reloaded under its accumulation"),
    ("dkdv", "xv_free", "P^T overwritten before dV read it"),
    ("dkdv", "xk_free", "dS^T overwritten before dK read it"),
    ("dkdv", "dp_ready", "dP^T read before its burst finished"),
])
def test_planted_mistake_is_caught(kernel, skip, what):
    caught = 0
    for n, seed, rate, acc in schedules(300):
        try:
            caught += KERNELS[kernel](n, seed, rate, skip=skip, acc_cycles=acc) != "ok"
        except Hazard:
            caught += 1
    assert caught > 0, "the model no longer sees " + what
