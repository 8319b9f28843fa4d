"""The tensor-core decode kernel's synchronisation protocol, modelled on the
host (no GPU).

csrc/gemv_tc.cu runs in each CTA a TMA producer (one thread), eight writer
warps that turn a stage's packed codes into the tensor-memory A operand, one
MMA-issuing thread and four epilogue warps.  They meet at mbarriers named by
parity: `full` / `empty` per stage, `a_full` / `a_free` per A buffer,
`acc_full` / `acc_free` per accumulator.  This model restates each role's
loop with the kernel's constants and parity arithmetic, over a CTA's segments
(a segment is a run of k-tiles of one 128-row block, cut into units of up to
ks k-tiles), and runs it under random interleavings.  Copies land in any
order; MMAs and commits complete in issue order.  It checks:
- every wait completes (no deadlock);
- no arrival lands in a phase other than its own, no waiter falls two
  phases behind (where a parity wait would alias);
- every MMA reads an A buffer that all eight writer warps filled for its
  k-tile, and a stage that holds its unit, also when it executes;
- every segment's accumulator reaches the epilogue whole.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "ternary_weight_linear_bitlinear_b200", "csrc", "gemv_tc.cu")

A_BUFS = 4
ACC_BUFS = 2
WRITER_WARPS = 8
EPI_WARPS = 4
STAGES = 4
KS = 4


def test_model_constants_match_kernel_source():
    src = open(SRC).read()
    consts = dict(re.findall(r"constexpr int (k\w+) = (\d+);", src))
    assert int(consts["kABufs"]) == A_BUFS
    assert int(consts["kAccBufs"]) == ACC_BUFS
    assert int(consts["kWriterWarps"]) == WRITER_WARPS
    assert "mbar_init(smem_u32(&sh.a_full[b]), kWriterWarps);" in src
    assert "mbar_init(smem_u32(&sh.acc_free[b]), 4);" in src
    assert "*stages = 4;" in src and "int k = 4;" in src
    # the writer waits for the MMA of k-tile ka - kABufs before refilling
    assert "(uint32_t)(ka / kABufs - 1) & 1u" in src
    assert "(uint32_t)(ka / kABufs) & 1u" in src


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


class Model:
    def __init__(self, segments, seed, a_full_count=WRITER_WARPS):
        """segments: k-tile counts of the CTA's segments, in order."""
        self.rng = random.Random(seed)
        self.segments = segments
        # units: (segment, first k-tile, k-tiles)
        self.units = []
        for sg, nk in enumerate(segments):
            for kb in range(0, nk, KS):
                self.units.append((sg, kb, min(KS, nk - kb)))
        # a full phase: the producer's arm plus the weight and token copies
        self.full = [Barrier("full[%d]" % s, 3) for s in range(STAGES)]
        self.empty = [Barrier("empty[%d]" % s, 1) for s in range(STAGES)]
        self.a_full = [Barrier("a_full[%d]" % b, a_full_count) for b in range(A_BUFS)]
        self.a_free = [Barrier("a_free[%d]" % b, 1) for b in range(A_BUFS)]
        self.acc_full = [Barrier("acc_full[%d]" % b, 1) for b in range(ACC_BUFS)]
        self.acc_free = [Barrier("acc_free[%d]" % b, EPI_WARPS) for b in range(ACC_BUFS)]
        self.stage_w, self.stage_x = {}, {}      # stage -> unit index its copies hold
        self.a = {b: [None] * WRITER_WARPS for b in range(A_BUFS)}   # k-tile per warp part
        self.acc = {}                            # buffer -> (segment, k-tiles accumulated)
        self.copies, self.tensor = [], []
        self.seen = []

    def producer(self):
        for u in range(len(self.units)):
            st, rnd = u % STAGES, u // STAGES
            if rnd > 0:
                yield self.empty[st], rnd - 1
            self.full[st].arrive(rnd)            # arrive.expect_tx

            def land_w(u=u, st=st, rnd=rnd):
                self.stage_w[st] = u
                self.full[st].arrive(rnd)

            def land_x(u=u, st=st, rnd=rnd):
                self.stage_x[st] = u
                self.full[st].arrive(rnd)
            self.copies += [land_w, land_x]

    def writer(self, w):
        ka = 0
        for u, (sg, kb, nkb) in enumerate(self.units):
            st = u % STAGES
            yield self.full[st], u // STAGES
            if self.stage_w.get(st) != u:
                raise Protocol("writer %d: stage %d holds unit %s, not %d" % (w, st, self.stage_w.get(st), u))
            for kk in range(nkb):
                abuf = ka % A_BUFS
                if ka >= A_BUFS:
                    yield self.a_free[abuf], ka // A_BUFS - 1
                self.a[abuf][w] = ka
                self.a_full[abuf].arrive(ka // A_BUFS)
                ka += 1

    def mma(self):
        ka = 0
        u = 0
        for sg, nk in enumerate(self.segments):
            ab, use = sg % ACC_BUFS, sg // ACC_BUFS
            if use > 0:
                yield self.acc_free[ab], use - 1
            while u < len(self.units) and self.units[u][0] == sg:
                _, kb, nkb = self.units[u]
                st = u % STAGES
                yield self.full[st], u // STAGES
                for kk in range(nkb):
                    abuf = ka % A_BUFS
                    yield self.a_full[abuf], ka // A_BUFS
                    if self.a[abuf] != [ka] * WRITER_WARPS:
                        raise Protocol("MMA k-tile %d: A buffer %d holds %s" % (ka, abuf, self.a[abuf]))

                    def run(ka=ka, abuf=abuf, st=st, u=u, sg=sg, first=(kb == 0 and kk == 0), ab=ab):
                        if self.a[abuf] != [ka] * WRITER_WARPS:
                            raise Protocol("A buffer %d rewritten before k-tile %d's MMAs ran" % (abuf, ka))
                        if self.stage_x.get(st) != u:
                            raise Protocol("stage %d rewritten before unit %d's MMAs ran" % (st, u))
                        s_, n = self.acc.get(ab, (None, 0))
                        if first:
                            s_, n = sg, 0
                        elif s_ != sg:
                            raise Protocol("accumulator %d holds segment %s during %d" % (ab, s_, sg))
                        self.acc[ab] = (s_, n + 1)
                    self.tensor.append(run)
                    self.tensor.append(lambda abuf=abuf, p=ka // A_BUFS: self.a_free[abuf].arrive(p))
                    ka += 1
                self.tensor.append(lambda st=st, p=u // STAGES: self.empty[st].arrive(p))
                u += 1
            self.tensor.append(lambda ab=ab, use=use: self.acc_full[ab].arrive(use))

    def epilogue(self):
        for sg, nk in enumerate(self.segments):
            ab, use = sg % ACC_BUFS, sg // ACC_BUFS
            yield self.acc_full[ab], use
            if self.acc.get(ab) != (sg, nk):
                raise Protocol("epilogue segment %d found accumulator %s" % (sg, self.acc.get(ab)))
            self.seen.append(sg)
            self.acc_free[ab].arrive(use, EPI_WARPS)

    def run(self, max_events=10 ** 6):
        agents = [self.producer(), self.mma(), self.epilogue()] + \
                 [self.writer(w) for w in range(WRITER_WARPS)]
        waiting, live = {}, list(range(len(agents)))
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
                self.tensor.pop(0)()
            else:
                waiting.pop(a, None)
                try:
                    waiting[a] = next(agents[a])
                except StopIteration:
                    live.remove(a)
        else:
            raise Protocol("did not finish")
        assert not self.copies and not self.tensor
        assert self.seen == list(range(len(self.segments)))


@pytest.mark.parametrize("seed", range(60))
def test_decode_tc_protocol_random_interleavings(seed):
    rng = random.Random(2000 + seed)
    segments = [rng.randint(1, 14) for _ in range(rng.randint(1, 4))]
    Model(segments, seed).run()


def test_decode_tc_model_catches_a_miscounted_barrier():
    # With a_full completing after seven writer warps instead of eight, the
    # MMA may read an A buffer a warp has not filled yet: the model sees it.
    with pytest.raises(Protocol):
        for seed in range(60):
            Model([9, 5], seed, a_full_count=WRITER_WARPS - 1).run()
