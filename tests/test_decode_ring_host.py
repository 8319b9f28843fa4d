"""The decode kernel's shared-memory ring, modelled on the host (no GPU).

csrc/gemv.cu streams each CTA's units (a row-tile group x a K slab) through a
ring of `stages` shared-memory stages.  One producer thread arms a stage's
`full` barrier with the bytes it expects, then issues the weight copies and, for
the product-only variant, the activation copies.  Four consumer warps wait on
`full`, multiply, and arrive on `empty`.  With static weights the producer
issues the first unit's weight copies before the dependency wait, and the main
loop then adds only its activation copies, whose bytes the earlier arm already
counted.  This model restates that loop and the kernel's parity arithmetic, runs
it under random interleavings with copies landing in any order, and checks:
- no deadlock;
- no arrival in a wrong phase;
- no waiter two phases behind;
- each consumer reads a stage whose weights and activations both belong to its unit.
"""
import random

import pytest

DEC_WARPS = 4


def test_model_constants_match_kernel_source():
    """The model's warp count and prefetch rule are the kernel's (csrc/gemv.cu)."""
    import os
    import re
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "ternary_weight_linear_bitlinear_b200", "csrc", "gemv.cu")
    src = open(path).read()
    m = re.search(r"constexpr int kDecWarps = (\d+);", src)
    assert m and int(m.group(1)) == DEC_WARPS
    # the number of units whose weights are requested before the dependency wait
    assert "const int first = units < 1 ? units : 1;" in src
    assert "} else if (!a.static_weights || u >= first) {" in src


class Protocol(AssertionError):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.completed, self.pending = 0, count

    def arrive(self, phase, n=1):
        if phase != self.completed:
            raise Protocol("%s: arrival for phase %d while phase %d is open"
                           % (self.name, phase, self.completed))
        self.pending -= n
        if self.pending < 0:
            raise Protocol("%s: too many arrivals" % self.name)
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def done(self, phase):
        if self.completed >= phase + 2:
            raise Protocol("%s: waiter for phase %d is two phases behind" % (self.name, phase))
        return self.completed > phase


class TxBarrier(Barrier):
    """A `full` barrier: one arrival (the arm, with its expected byte count)
    plus every expected copy completes a phase.  Copies may land before the
    arm of their phase is seen by other threads, but never before it is issued
    (the producer arms, then copies)."""

    def __init__(self, name):
        super().__init__(name, 1)
        self.expect = None      # copies the open phase still waits for

    def arm(self, phase, copies):
        if phase != self.completed or self.expect is not None:
            raise Protocol("%s: armed for phase %d while phase %d is open"
                           % (self.name, phase, self.completed))
        self.expect = copies
        self.pending = 1
        self._arrive_internal()

    def copy_landed(self, phase):
        if phase != self.completed or self.expect is None or self.expect <= 0:
            raise Protocol("%s: copy for phase %d lands in phase %d" % (self.name, phase, self.completed))
        self.expect -= 1
        self._check()

    def _arrive_internal(self):
        self.pending = 0
        self._check()

    def _check(self):
        if self.pending == 0 and self.expect == 0:
            self.completed += 1
            self.expect = None
            self.pending = 1


class Ring:
    def __init__(self, units, stages, nrow, T, static, fused, seed):
        self.rng = random.Random(seed)
        self.units, self.stages, self.nrow, self.T = units, stages, nrow, T
        self.static, self.fused = static, fused
        self.full = [TxBarrier("full[%d]" % s) for s in range(stages)]
        self.empty = [Barrier("empty[%d]" % s, DEC_WARPS) for s in range(stages)]
        self.w_tag = [[None] * nrow for _ in range(stages)]
        self.x_tag = [[None] * T for _ in range(stages)]
        self.copies = []

    def producer(self):
        S, U = self.stages, self.units
        xcopies = 0 if self.fused else self.T

        def issue_w(u, st):
            self.full[st].arm(u // S, self.nrow + xcopies)
            for r in range(self.nrow):
                def land(u=u, st=st, r=r):
                    self.w_tag[st][r] = u
                    self.full[st].copy_landed(u // S)
                self.copies.append(land)

        def issue_x(u, st):
            for t in range(xcopies):
                def land(u=u, st=st, t=t):
                    self.x_tag[st][t] = u
                    self.full[st].copy_landed(u // S)
                self.copies.append(land)

        first = min(U, 1)
        if self.static:
            for u in range(first):
                issue_w(u, u)
        yield None                       # the dependency wait: anything may interleave here
        st, rnd = 0, 0
        for u in range(U):
            if rnd > 0:
                yield self.empty[st], rnd - 1
                issue_w(u, st)
            elif not self.static or u >= first:
                issue_w(u, st)
            issue_x(u, st)
            st += 1
            if st == S:
                st, rnd = 0, rnd + 1

    def consumer(self, w):
        S = self.stages
        for u in range(self.units):
            st = u % S
            yield self.full[st], u // S
            if any(tag != u for tag in self.w_tag[st]):
                raise Protocol("warp %d unit %d: weights of units %s" % (w, u, self.w_tag[st]))
            if not self.fused and any(tag != u for tag in self.x_tag[st]):
                raise Protocol("warp %d unit %d: activations of units %s" % (w, u, self.x_tag[st]))
            self.empty[st].arrive(u // S)

    def run(self, max_events=10 ** 6):
        agents = [self.producer()] + [self.consumer(w) for w in range(DEC_WARPS)]
        waiting, live = {}, list(range(len(agents)))
        for _ in range(max_events):
            runnable = [a for a in live
                        if a not in waiting or waiting[a] is None or waiting[a][0].done(waiting[a][1])]
            choices = [("agent", a) for a in runnable] + ([("copy", None)] if self.copies else [])
            if not choices:
                if live:
                    raise Protocol("deadlock")
                break
            kind, a = self.rng.choice(choices)
            if kind == "copy":
                self.copies.pop(self.rng.randrange(len(self.copies)))()
                continue
            waiting.pop(a, None)
            try:
                waiting[a] = next(agents[a])
            except StopIteration:
                live.remove(a)
        else:
            raise Protocol("did not finish")
        assert not self.copies
        # The producer's drain: the last stages' phases all completed.
        for u in range(max(0, self.units - self.stages), self.units):
            assert self.full[u % self.stages].completed > u // self.stages


@pytest.mark.parametrize("seed", range(60))
def test_decode_ring_random_interleavings(seed):
    rng = random.Random(500 + seed)
    Ring(units=rng.randint(1, 24), stages=rng.randint(2, 6), nrow=rng.randint(1, 2),
         T=rng.choice([1, 2, 3]), static=rng.random() < 0.5, fused=rng.random() < 0.5,
         seed=seed).run()


def test_decode_ring_model_catches_a_missing_release():
    # With three consumer warps counted on `empty` instead of four, a stage is
    # refilled while a warp may still read it: the model sees a phase overrun.
    with pytest.raises(Protocol):
        for seed in range(30):
            r = Ring(units=12, stages=2, nrow=2, T=2, static=True, fused=False, seed=seed)
            r.empty = [Barrier("empty[%d]" % s, DEC_WARPS - 1) for s in range(2)]
            r.run()
