"""The chunked prefill's barrier protocol (csrc/prefill.cu), checked as an
explicit-state model on the CPU.

The model has the kernel's roles for one CTA pair over n stages:
  - per CTA, four softmax warps, four K-dequantising warps and four
    V-dequantising warps (each warp arrives once per stage, as its 32 lanes
    do together);
  - rank 0's MMA thread, which waits, and queues Q K^T, P V and commits;
  - the tensor pipe, which runs that queue in order (a commit arrives on its
    barriers, in both CTAs, once everything queued before it is done).
Barriers count arrivals and complete phases as mbarriers do; a parity wait
passes while the barrier's current phase has the other parity. Every wait
names the phase it means, and the model fails when a wait passes on another
phase, when a tile is overwritten before its reader is done or read before
it is written, when O is rescaled or read while a P V is owed, or when no
role can move (the kernel's bounded waits would run out).

Schedules are random with a random speed per role, so one CTA or one warp
can fall far behind another. The protocol as built passes every schedule;
the two earlier forms of it (one P-ready barrier for all stages; the
epilogue's parity wait on the P V barrier) fail, which shows that the model
can see those races."""
import random

import pytest

NS = 3        # shared-memory slots of K^ and V^
WARPS = 4     # warps per role per CTA


class Violation(Exception):
    pass


class Bar:
    def __init__(self, count):
        self.count, self.done, self.pending = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.done += 1
            self.pending = 0

    def passes(self, parity):
        return (self.done & 1) != parity


class Model:
    def __init__(self, n_st, rng, split_pready=True, drain_epilogue=True):
        self.n, self.rng = n_st, rng
        self.split_pready, self.drain_epilogue = split_pready, drain_epilogue
        arrivals = 2 * WARPS  # both CTAs' warps of one role
        self.kready = [Bar(arrivals) for _ in range(NS)]
        self.vready = [Bar(arrivals) for _ in range(NS)]
        self.pready = [Bar(arrivals) for _ in range(2 if split_pready else 1)]
        self.qready = Bar(arrivals)
        # per CTA, signalled by the commits
        self.sfull = [[Bar(1), Bar(1)] for _ in range(2)]
        self.kfree = [[Bar(1) for _ in range(NS)] for _ in range(2)]
        self.vfree = [[Bar(1) for _ in range(NS)] for _ in range(2)]
        self.odone = [Bar(1) for _ in range(2)]
        self.drain = [Bar(1) for _ in range(2)]
        # tile states per (CTA, slot, warp): what the slot holds
        self.k = [[[None] * WARPS for _ in range(NS)] for _ in range(2)]
        self.v = [[[None] * WARPS for _ in range(NS)] for _ in range(2)]
        self.s = [[[None] * WARPS for _ in range(2)] for _ in range(2)]
        self.pv_done = 0
        self.queue = []

    # ---- the roles, as generators yielding ("wait", bar, parity, phase) or None (a step)
    def mma(self):
        yield ("wait", self.qready, 0, 0)
        for j in range(self.n):
            b, u = j % NS, j // NS
            yield ("wait", self.kready[b], u & 1, u)
            self.queue += [("qk", j), ("commit", [self.sfull[c][j & 1] for c in (0, 1)]),
                           ("commit", [self.kfree[c][b] for c in (0, 1)])]
            yield None
            if j >= 1:
                yield from self.pv(j - 1)
        yield from self.pv(self.n - 1)
        self.queue.append(("commit", self.drain[:]))

    def pv(self, i):
        if self.split_pready:
            yield ("wait", self.pready[i & 1], (i >> 1) & 1, i >> 1)
        else:
            yield ("wait", self.pready[0], i & 1, i)
        b, u = i % NS, i // NS
        yield ("wait", self.vready[b], u & 1, u)
        self.queue += [("pv", i), ("commit", self.odone[:]), ("commit", [self.vfree[c][b] for c in (0, 1)])]
        yield None

    def softmax(self, c, w, speed_rescale):
        self.qready.arrive()
        yield None
        for j in range(self.n):
            sb = j & 1
            yield ("wait", self.sfull[c][sb], (j >> 1) & 1, j >> 1)
            if self.s[c][sb][w] != ("S", j):
                raise Violation(f"softmax {c}.{w} stage {j} reads {self.s[c][sb][w]}")
            yield None
            self.s[c][sb][w] = ("P", j)
            if j >= 1 and self.rng.random() < speed_rescale:   # the running max moved: rescale O
                yield ("wait", self.odone[c], (j - 1) & 1, j - 1)
                if self.pv_done != j:
                    raise Violation(f"softmax {c}.{w} rescales O at stage {j} with {self.pv_done} P V done")
                yield None
            (self.pready[j & 1] if self.split_pready else self.pready[0]).arrive()
            yield None
        if self.drain_epilogue:
            yield ("wait", self.drain[c], 0, 0)
        else:
            yield ("wait", self.odone[c], (self.n - 1) & 1, self.n - 1)
        if self.pv_done != self.n:
            raise Violation(f"softmax {c}.{w} reads O with {self.pv_done} of {self.n} P V done")

    def producer(self, c, w, kind):
        tiles, ready, free = ((self.k, self.kready, self.kfree[c]) if kind == "k" else
                              (self.v, self.vready, self.vfree[c]))
        used = "Kused" if kind == "k" else "Vused"
        for j in range(self.n):
            b, u = j % NS, j // NS
            if u >= 1:
                yield ("wait", free[b], (u - 1) & 1, u - 1)
            if tiles[c][b][w] not in (None, (used, j - NS)):
                raise Violation(f"{kind} producer {c}.{w} overwrites {tiles[c][b][w]} with stage {j}")
            tiles[c][b][w] = j
            yield None
            ready[b].arrive()
            yield None

    def tensor_step(self):
        op = self.queue.pop(0)
        if op[0] == "qk":
            j = op[1]
            for c in (0, 1):
                for w in range(WARPS):
                    if self.k[c][j % NS][w] != j:
                        raise Violation(f"Q K^T {j} reads K {self.k[c][j % NS][w]}")
                    self.k[c][j % NS][w] = ("Kused", j)
                    if self.s[c][j & 1][w] not in (None, ("Pdone", j - 2)):
                        raise Violation(f"Q K^T {j} overwrites {self.s[c][j & 1][w]} (CTA {c} warp {w})")
                    self.s[c][j & 1][w] = ("S", j)
        elif op[0] == "pv":
            i = op[1]
            if self.pv_done != i:
                raise Violation(f"P V {i} after {self.pv_done}")
            for c in (0, 1):
                for w in range(WARPS):
                    if self.s[c][i & 1][w] != ("P", i):
                        raise Violation(f"P V {i} reads {self.s[c][i & 1][w]} (CTA {c} warp {w})")
                    self.s[c][i & 1][w] = ("Pdone", i)
                    if self.v[c][i % NS][w] != i:
                        raise Violation(f"P V {i} reads V {self.v[c][i % NS][w]}")
                    self.v[c][i % NS][w] = ("Vused", i)
            self.pv_done += 1
        else:
            for bar in op[1]:
                bar.arrive()

    def run(self):
        rescale = self.rng.random()
        roles = [self.mma()]
        for c in (0, 1):
            for w in range(WARPS):
                roles += [self.softmax(c, w, rescale), self.producer(c, w, "k"), self.producer(c, w, "v")]
        speed = [self.rng.expovariate(1.0) + 1e-3 for _ in range(len(roles) + 1)]  # last: the tensor pipe
        cur = [None] * len(roles)
        live = [True] * len(roles)
        for r in range(len(roles)):
            cur[r] = next(roles[r], "end")
            live[r] = cur[r] != "end"
        while True:
            ready = []
            for r, y in enumerate(cur):
                if live[r] and (y is None or y[1].passes(y[2])):
                    ready.append(r)
            if self.queue:
                ready.append(len(roles))
            if not ready:
                if any(live):
                    raise Violation("no role can move (a bounded wait would run out)")
                return
            r = self.rng.choices(ready, weights=[speed[x] for x in ready])[0]
            if r == len(roles):
                self.tensor_step()
                continue
            y = cur[r]
            if y is not None:
                bar, phase = y[1], y[3]
                if bar.done != phase + 1:
                    raise Violation(f"a wait for phase {phase} passed with {bar.done} phases done")
            cur[r] = next(roles[r], "end")
            live[r] = cur[r] != "end"


def _violations(runs, seed, **kw):
    rng = random.Random(seed)
    found = []
    for k in range(runs):
        n = rng.randint(1, 7)
        try:
            Model(n, rng, **kw).run()
        except Violation as e:
            found.append((k, n, str(e)))
    return found


def test_protocol_as_built_holds_under_skewed_schedules():
    assert _violations(3000, seed=1) == []


@pytest.mark.parametrize("kw", [dict(split_pready=False), dict(drain_epilogue=False)],
                         ids=["one_pready", "odone_epilogue"])
def test_model_sees_the_earlier_races(kw):
    assert _violations(3000, seed=2, **kw)
