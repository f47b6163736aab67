"""A discrete-event model of the verify kernel's barrier protocol
(lossless_draft_verify_vc_b200/csrc/vc_verify.cu), run on the CPU.

The kernel waits on mbarriers by phase parity: a wait for completion #e of a
barrier passes as soon as the barrier's completed-phase count has the parity
of e + 1.  That is only right if, when the wait starts, the barrier has
completed e or e + 1 phases: fewer and the wait passes early, more and it
waits for a phase that belongs to a later tile.  The model replays the
kernel's three roles with random latencies and checks that precondition at
every wait, that every role finishes (no deadlock), and that every load and
MMA happens exactly once:

* loader: Q, K and V of tiles 0 .. NS - 1 (NS stages: 2, or 4 when one block
  takes two row tiles), then K of tile j once the S MMAs of tile j - NS
  released stage j mod NS and V of tile j once the P.V MMAs of tile j - NS
  did, in the order those happen (K one tile ahead of V);
* MMA thread: S of tiles 0 and 1 (after Q and their K), then per tile i,
  once every softmax warp has stored P(i) (barrier p<i & 1>): P.V(i) once
  V(i) landed, and S(i + 2) into S buffer i & 1 once P.V(i) is done and
  K(i + 2) landed; each S group also releases its K stage, each P.V group
  its V stage;
* softmax warps (4, or 8 when one block takes two row tiles), each on its
  own clock: per tile i, wait S(i), work, wait P.V(i - 1) when it rescales
  O (the lazy rule makes that rare), store P, arrive on p<i & 1> and go on
  to tile i + 1 without waiting for the MMA thread; at the end wait for the
  last P.V.

Barriers: k<j> v<j> (stage landed), kf<j> vf<j> (stage released) for
j < NS, s0 s1 (S buffers), p0 p1 (P stored: one arrival per softmax warp
completes a phase), pv0 pv1 (P.V per buffer), q.  The tensor pipe runs MMA
groups in issue order; a group's commits fire when it ends.
"""

import heapq
import itertools
import random

import pytest


class _Sim:
    def __init__(self, rng):
        self.rng, self.t, self.q, self.seq = rng, 0.0, [], itertools.count()
        self.count = {}
        self.waiters = {}
        self.pipe_free = 0.0
        self.group = []
        self.arrivals = {}

    def done(self, name):
        return self.count.get(name, 0)

    def complete(self, name):
        self.count[name] = self.done(name) + 1
        keep = []
        for target, gen in self.waiters.pop(name, []):
            if self.count[name] >= target:
                self.schedule(0.0, gen)
            else:
                keep.append((target, gen))
        if keep:
            self.waiters[name] = keep

    def schedule(self, dt, gen):
        heapq.heappush(self.q, (self.t + dt, next(self.seq), gen))

    def fire_after(self, dt, name):
        def gen():
            self.complete(name)
            return
            yield
        heapq.heappush(self.q, (self.t + dt, next(self.seq), gen()))

    def run(self):
        while self.q:
            self.t, _, gen = heapq.heappop(self.q)
            try:
                req = next(gen)
            except StopIteration:
                continue
            self.handle(req, gen)

    def handle(self, req, gen):
        kind = req[0]
        if kind == "wait":
            _, name, e = req
            c = self.done(name)
            assert c in (e, e + 1), f"wait for {name} #{e} found {c} completed phases"
            if c == e + 1:
                self.schedule(0.0, gen)
            else:
                self.waiters.setdefault(name, []).append((e + 1, gen))
        elif kind == "sleep":
            self.schedule(req[1], gen)
        elif kind == "load":
            self.fire_after(self.rng.uniform(5, 60), req[1])
            self.schedule(0.0, gen)
        elif kind == "mma":
            start = max(self.t, self.pipe_free)
            self.pipe_free = start + req[2]
            for name in (req[1] if isinstance(req[1], tuple) else (req[1],)):
                self.fire_after(self.pipe_free - self.t, name)
            self.schedule(self.rng.uniform(0, req[2]), gen)  # the issue may block part of the time
        elif kind == "arrive":  # one arrival; the phase completes at `count` arrivals
            _, name, count = req
            a = self.arrivals.get(name, 0) + 1
            if a == count:
                a = 0
                self.complete(name)
            self.arrivals[name] = a
            self.schedule(0.0, gen)
        elif kind == "group":
            self.group.append(gen)
            if len(self.group) == 2:
                for g in self.group:
                    self.schedule(0.0, g)
                self.group = []


def _run_protocol(n, rng, NS, warps, stale_p_wait=False):
    sim = _Sim(rng)
    finished = []
    stored = [0] * n  # softmax warps that have stored P of each tile

    def loader():
        yield ("load", "q")
        for j in range(min(NS, n)):
            yield ("load", f"k{j % NS}")
            yield ("load", f"v{j % NS}")
        nk = nv = min(NS, n)
        while nk < n or nv < n:
            is_k = nk < n and nk <= nv + 1
            j = nk if is_k else nv
            yield ("wait", (f"kf{j % NS}" if is_k else f"vf{j % NS}"), j // NS - 1)
            yield ("load", (f"k{j % NS}" if is_k else f"v{j % NS}"))
            if is_k:
                nk = j + 1
            else:
                nv = j + 1
        finished.append("loader")

    def mma():
        def issue_s(i):
            yield ("wait", f"k{i % NS}", i // NS)
            yield ("mma", (f"s{i & 1}", f"kf{i % NS}"), rng.uniform(3, 30))

        yield ("sleep", rng.uniform(0, 20))
        yield ("wait", "q", 0)
        for i in range(min(2, n)):
            yield from issue_s(i)
        for i in range(n):
            yield ("wait", f"p{i & 1}", max(0, (i >> 1) - 1) if stale_p_wait else i >> 1)
            assert stored[i] == warps, f"P.V({i}) issued before every warp stored P({i})"
            yield ("wait", f"v{i % NS}", i // NS)
            yield ("mma", (f"pv{i & 1}", f"vf{i % NS}"), rng.uniform(5, 60))
            if i + 2 < n:
                yield ("wait", f"pv{i & 1}", i >> 1)
                yield from issue_s(i + 2)
        finished.append("mma")

    def softmax():
        yield ("sleep", rng.uniform(0, 20))
        for i in range(n):
            yield ("wait", f"s{i & 1}", i >> 1)
            yield ("sleep", rng.uniform(5, 80))
            if i > 0 and rng.random() < 0.3:  # only a warp that rescales O waits for P.V(i - 1)
                yield ("wait", f"pv{(i - 1) & 1}", (i - 1) >> 1)
            yield ("sleep", rng.uniform(0, 10))  # P stored
            stored[i] += 1
            yield ("arrive", f"p{i & 1}", warps)
        yield ("wait", f"pv{(n - 1) & 1}", (n - 1) >> 1)
        finished.append("softmax")

    for g in (loader(), mma(), *[softmax() for _ in range(warps)]):
        sim.schedule(0.0, g)
    sim.run()
    assert sorted(finished) == ["loader", "mma"] + ["softmax"] * warps, "a role never finished (deadlock)"
    assert sim.done("p0") + sim.done("p1") == n
    for kind in ("s", "pv"):
        assert sim.done(f"{kind}0") + sim.done(f"{kind}1") == n, kind
    for kind in ("k", "v", "kf", "vf"):
        assert sum(sim.done(f"{kind}{j}") for j in range(NS)) == n, kind
    assert sim.done("q") == 1


@pytest.mark.parametrize("NS,warps", [(2, 4), (2, 8), (4, 8)])
@pytest.mark.parametrize("ntiles", list(range(1, 12)))
def test_parity_waits_never_early_or_late(ntiles, NS, warps):
    rng = random.Random(1000 + ntiles + 100 * NS + warps)
    for _ in range(100):
        _run_protocol(ntiles, rng, NS, warps)


def test_model_catches_a_wait_on_a_stale_phase():
    """Planting a mistake in the model: a loader whose V wait targets P.V of
    tile j - 4 instead of j - 2 meets a barrier two phases ahead of that
    wait in some runs; the checker must notice in one of them."""
    rng = random.Random(7)

    def bad_run(n):
        sim = _Sim(rng)

        def loader():
            for j in range(min(2, n)):
                yield ("load", f"k{j & 1}")
                yield ("load", f"v{j & 1}")
            # wrong: V of tile j waits for P.V of tile j - 4 (two phases early)
            for j in range(2, n):
                yield ("wait", f"s{j & 1}", (j - 2) >> 1)
                yield ("load", f"k{j & 1}")
                yield ("wait", f"pv{j & 1}", max(0, ((j - 2) >> 1) - 1))
                yield ("load", f"v{j & 1}")

        def mma():
            for i in range(min(2, n)):
                yield ("wait", f"k{i & 1}", i >> 1)
                yield ("mma", f"s{i & 1}", 5.0)
            for i in range(n):
                yield ("wait", f"v{i & 1}", i >> 1)
                yield ("mma", f"pv{i & 1}", 40.0)
                if i + 2 < n:
                    yield ("wait", f"pv{i & 1}", i >> 1)
                    yield ("wait", f"k{i & 1}", (i + 2) >> 1)
                    yield ("mma", f"s{i & 1}", 5.0)

        for g in (loader(), mma()):
            sim.schedule(0.0, g)
        sim.run()

    with pytest.raises(AssertionError):
        for _ in range(50):
            bad_run(8)


def test_model_catches_a_p_wait_on_a_stale_phase():
    """Planting a mistake in the model: an MMA thread that waits for the "P
    stored" phase of tile i - 2 instead of tile i issues P.V before every
    softmax warp has stored P; the checker must notice in one of the runs."""
    rng = random.Random(11)
    with pytest.raises(AssertionError):
        for _ in range(50):
            _run_protocol(8, rng, 2, 4, stale_p_wait=True)
