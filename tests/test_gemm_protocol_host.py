"""The CTA-pair prefill GEMM's synchronisation protocol, modelled on the host
(no GPU).

csrc/gemm_tc.cu runs, in each CTA of a cluster pair, a TMA producer, a relay, two
expander groups and an epilogue, and in the leader one MMA issuer.  They meet at
mbarriers whose phases they name by parity.  This model restates each role's loop
with the kernel's ring constants and phase/parity arithmetic, and runs it under
random interleavings.  Copies, MMAs and commits complete asynchronously after
random delays, and the MMAs and commits complete in issue order.  The model checks:
- every wait completes (no deadlock);
- an arrival never lands in a phase other than the one it is meant for;
- a waiter never falls two phases behind, where a parity wait would alias;
- every MMA step reads tokens and codes written for that step;
- every tile's accumulator reaches its epilogue whole.
"""
import collections
import random

import pytest

# The kernel's constants (csrc/gemm_tc.cu, namespace pair).
K_STAGES = 5
K_PSLOTS = 6
K_PAHEAD = 6
K_ACC_BUFS = 2
K_READY_COUNT = 2 + 2 * 4      # two relays + one expander group (4 warps) per CTA
EXP_WARPS = 4                  # warps per expander group
EPI_WARPS = 4


def _source_constants(fname):
    """constexpr int values of a kernel source, by name."""
    import os
    import re
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "ternary_weight_linear_bitlinear_b200", "csrc", fname)
    text = open(path).read()
    out = {}
    for name, expr in re.findall(r"constexpr int (k\w+) = ([^;]+);", text):
        try:
            out[name] = eval(expr, {}, dict(out))
        except Exception:
            pass
    return out


def test_model_constants_match_kernel_source():
    """The model runs on the kernel's own ring constants: a change in the
    kernel that the model does not follow fails here."""
    c = _source_constants("gemm_tc.cu")
    assert c["kStages"] == K_STAGES
    assert c["kPSlots"] == K_PSLOTS
    assert c["kPAhead"] == K_PAHEAD
    assert c["kAccBufs"] == K_ACC_BUFS
    assert c["kReadyCount"] == K_READY_COUNT
    assert c["kEpiWarps"] == EPI_WARPS


class Protocol(AssertionError):
    pass


class Barrier:
    """An mbarrier: `count` arrivals (plus any expected transaction bytes,
    modelled as one extra arrival by the copy) complete a phase."""

    def __init__(self, name, count):
        self.name, self.count = name, count
        self.completed = 0          # phases completed so far
        self.pending = count

    def arrive(self, phase, n=1):
        if phase != self.completed:
            raise Protocol("%s: arrival for phase %d while phase %d is open"
                           % (self.name, phase, self.completed))
        self.pending -= n
        if self.pending < 0:
            raise Protocol("%s: too many arrivals in phase %d" % (self.name, phase))
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def done(self, phase):
        """A wait for `phase` by parity: true once it completed; the waiter must
        not be two phases behind (the parity would name a later phase)."""
        if self.completed >= phase + 2:
            raise Protocol("%s: waiter for phase %d is two phases behind (%d completed)"
                           % (self.name, phase, self.completed))
        return self.completed > phase


class Model:
    def __init__(self, num_k, tiles, seed):
        assert num_k % 2 == 0
        self.rng = random.Random(seed)
        self.num_k, self.tiles = num_k, tiles
        self.total = num_k * tiles
        self.total_units = self.total // 2
        R = (0, 1)
        self.full = {(r, s): Barrier("full[%d][%d]" % (r, s), 2) for r in R for s in range(K_STAGES)}
        self.freed = {(r, s): Barrier("freed[%d][%d]" % (r, s), 1) for r in R for s in range(K_STAGES)}
        self.ready = {s: Barrier("ready[%d]" % s, K_READY_COUNT) for s in range(K_STAGES)}
        self.pfull = {(r, p): Barrier("pfull[%d][%d]" % (r, p), 2) for r in R for p in range(K_PSLOTS)}
        self.pempty = {(r, p): Barrier("pempty[%d][%d]" % (r, p), 2 * EXP_WARPS)
                       for r in R for p in range(K_PSLOTS)}
        self.acc_full = {(r, b): Barrier("acc_full[%d][%d]" % (r, b), 1)
                         for r in R for b in range(K_ACC_BUFS)}
        self.acc_empty = {b: Barrier("acc_empty[%d]" % b, 2 * EPI_WARPS) for b in range(K_ACC_BUFS)}
        # What each buffer holds, as the step or unit it was written for.
        self.tok = {}       # (r, s) -> step
        self.codes = {}     # (r, s) -> step
        self.packed = {}    # (r, slot) -> unit
        self.acc = {}       # buf -> (tile, steps accumulated)
        self.copies = []    # in-flight copies: callables, any order
        self.tensor = collections.deque()   # MMAs and commits, in issue order
        self.epilogue_seen = {0: [], 1: []}

    # -------------------------------------------------------------- roles ---
    def producer(self, r):
        u_issued = 0

        def issue_unit(u):
            slot = u % K_PSLOTS
            b = self.pfull[(r, slot)]
            b.arrive(u // K_PSLOTS)                      # arrive.expect_tx

            def land(u=u, slot=slot, b=b):
                self.packed[(r, slot)] = u
                b.arrive(u // K_PSLOTS)                  # complete_tx
            self.copies.append(land)

        def units_through(last_step):
            nonlocal u_issued
            while u_issued < self.total_units and 2 * u_issued <= last_step:
                if u_issued >= K_PSLOTS:
                    yield self.pempty[(r, u_issued % K_PSLOTS)], u_issued // K_PSLOTS - 1
                issue_unit(u_issued)
                u_issued += 1

        yield from units_through(K_PAHEAD - 1)
        for step in range(self.total):
            s = step % K_STAGES
            if step >= K_STAGES:
                yield self.freed[(r, s)], step // K_STAGES - 1
            b = self.full[(r, s)]
            b.arrive(step // K_STAGES)

            def land(step=step, s=s, b=b):
                self.tok[(r, s)] = step
                b.arrive(step // K_STAGES)
            self.copies.append(land)
            yield from units_through(step + K_PAHEAD)

    def relay(self, r):
        for g in range(self.total):
            s = g % K_STAGES
            yield self.full[(r, s)], g // K_STAGES
            self.ready[s].arrive(g // K_STAGES)

    def expander(self, r, grp):
        for g in range(grp, self.total, 2):
            s, u = g % K_STAGES, g // 2
            sp = u % K_PSLOTS
            yield self.pfull[(r, sp)], u // K_PSLOTS
            if self.packed.get((r, sp)) != u:
                raise Protocol("expander %d/%d step %d read unit %s" % (r, grp, g, self.packed.get((r, sp))))
            if g >= K_STAGES:
                yield self.freed[(r, s)], g // K_STAGES - 1
            self.codes[(r, s)] = g
            self.ready[s].arrive(g // K_STAGES, EXP_WARPS)
            self.pempty[(r, sp)].arrive(u // K_PSLOTS, EXP_WARPS)

    def mma(self):
        step = 0
        for i in range(self.tiles):
            buf, use = i % K_ACC_BUFS, i // K_ACC_BUFS
            if use > 0:
                yield self.acc_empty[buf], use - 1
            for kt in range(self.num_k):
                s = step % K_STAGES
                yield self.ready[s], step // K_STAGES
                for r in (0, 1):
                    if self.tok.get((r, s)) != step or self.codes.get((r, s)) != step:
                        raise Protocol("MMA step %d: stage %d holds tokens %s / codes %s in CTA %d"
                                       % (step, s, self.tok.get((r, s)), self.codes.get((r, s)), r))

                def run(i=i, buf=buf, kt=kt, step=step, s=s):
                    # The MMAs read the stage when they execute.
                    for r in (0, 1):
                        if self.tok.get((r, s)) != step or self.codes.get((r, s)) != step:
                            raise Protocol("stage %d overwritten before step %d's MMAs ran" % (s, step))
                    t, n = self.acc.get(buf, (None, 0))
                    if kt == 0:
                        t, n = i, 0
                    elif t != i:
                        raise Protocol("accumulator %d holds tile %s during tile %d" % (buf, t, i))
                    self.acc[buf] = (t, n + 1)
                self.tensor.append(run)
                phase = step // K_STAGES
                self.tensor.append(lambda s=s, phase=phase: [self.freed[(r, s)].arrive(phase)
                                                            for r in (0, 1)])
                step += 1
            self.tensor.append(lambda buf=buf, use=use: [self.acc_full[(r, buf)].arrive(use)
                                                        for r in (0, 1)])

    def epilogue(self, r):
        for i in range(self.tiles):
            buf, use = i % K_ACC_BUFS, i // K_ACC_BUFS
            yield self.acc_full[(r, buf)], use
            if self.acc.get(buf) != (i, self.num_k):
                raise Protocol("epilogue %d tile %d found accumulator %s" % (r, i, self.acc.get(buf)))
            self.epilogue_seen[r].append(i)
            self.acc_empty[buf].arrive(use, EPI_WARPS)

    # ---------------------------------------------------------- scheduler ---
    def run(self, max_events=10 ** 6):
        agents = [self.producer(0), self.producer(1), self.relay(0), self.relay(1),
                  self.expander(0, 0), self.expander(0, 1), self.expander(1, 0),
                  self.expander(1, 1), self.mma(), self.epilogue(0), self.epilogue(1)]
        waiting = {}        # agent index -> (barrier, phase) it waits on
        live = list(range(len(agents)))
        for _ in range(max_events):
            runnable = [a for a in live if a not in waiting or waiting[a][0].done(waiting[a][1])]
            choices = [("agent", a) for a in runnable]
            if self.copies:
                choices.append(("copy", None))
            if self.tensor:
                choices.append(("tensor", None))
            if not choices:
                if live:
                    raise Protocol("deadlock: %s" % {a: (w[0].name, w[1]) for a, w in waiting.items()})
                break
            kind, a = self.rng.choice(choices)
            if kind == "copy":
                self.copies.pop(self.rng.randrange(len(self.copies)))()
            elif kind == "tensor":
                self.tensor.popleft()()
            else:
                waiting.pop(a, None)
                try:
                    waiting[a] = next(agents[a])
                except StopIteration:
                    live.remove(a)
        else:
            raise Protocol("did not finish")
        assert not self.copies and not self.tensor
        for r in (0, 1):
            assert self.epilogue_seen[r] == list(range(self.tiles))


@pytest.mark.parametrize("seed", range(40))
def test_pair_gemm_protocol_random_interleavings(seed):
    rng = random.Random(1000 + seed)
    num_k = rng.choice([2, 4, 6, 8, 32])
    tiles = rng.choice([1, 2, 3, 5])
    Model(num_k, tiles, seed).run()


def test_protocol_model_catches_a_miscounted_barrier():
    # The model is sharp enough to matter: with the relays left out of the
    # `ready` count, a stage's phase completes on the expanders' arrivals alone
    # and the relays' arrivals then land in the next phase.
    global K_READY_COUNT
    saved = K_READY_COUNT
    try:
        K_READY_COUNT = 2 * 4    # expanders only
        with pytest.raises(Protocol):
            for seed in range(20):
                Model(8, 3, seed).run()
    finally:
        K_READY_COUNT = saved
