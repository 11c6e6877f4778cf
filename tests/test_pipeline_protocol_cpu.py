"""Model checks of the kernels' mbarrier protocols (CPU; race detection in
place of compute-sanitizer, which is not available).

The forward kernel (fa_fwd.cu: two query tiles per CTA, a shared K/V ring,
S_q(t+1) issued after PV_q(t), lazy O rescale without a wait), the backward
kernel (fa_bwd.cu: K/V once, Q and dO rings of two stages, the dQ drain
staged through the tile's dO buffer) and the paged decode kernel
(fa_decode.cu: S^T double buffer issued a tile ahead, P and its products
doubled by tile parity, stages refilled after their P V product, the tail
tile's V rows zeroed by the softmax warps) and the wide forward's keep-word
ring (fa_fwd_wide.cu with dropout) are restated as roles that step
through their waits, arrivals and tensor-core operations: a TMA producer
whose copies complete in any order, an MMA issuer whose operations and
commits complete asynchronously but in issue order, and the softmax /
elementwise / drain warps.  Random interleavings must finish with

  * no deadlock,
  * every parity wait seeing its barrier at the awaited phase or one before
    it (never two phases on, where the parity would alias),
  * every buffer holding the expected tile when read and never refilled or
    overwritten while a reader is pending,
  * no O rescale against a queued PV.

Planted slips in the restated protocols are caught, which shows the checks
bite.  A change to a kernel's barrier protocol is to be mirrored here."""

import random

import pytest


class Bar:
    """mbarrier: ``count`` arrivals complete a phase; ``done`` phases so far."""

    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self, n=1):
        for _ in range(n):
            self.pending += 1
            if self.pending == self.count:
                self.pending = 0
                self.done += 1


class Protocol:
    """Common scheduler: roles are generators yielding ('wait', bar, phase) or None."""

    def __init__(self, rng):
        self.rng = rng
        self.fifo, self.loads, self.errors = [], [], []

    def ready(self, bar, k):
        if bar.done >= k + 2:
            self.errors.append(f"parity alias on {bar.name}: waiting for phase {k}, {bar.done} done")
        return bar.done >= k + 1

    def run(self, roles):
        pending = [None] * len(roles)
        alive = list(range(len(roles)))
        for _ in range(500000):
            if not (alive or self.fifo or self.loads):
                return
            choices = [("role", r) for r in alive if pending[r] is None or self.ready(pending[r][1], pending[r][2])]
            if self.fifo:
                choices.append(("mma", None))
            if self.loads:
                choices.append(("load", None))
            if not choices:
                self.errors.append("deadlock: " + str({r: (pending[r][1].name, pending[r][2]) for r in alive}))
                return
            kind, r = self.rng.choice(choices)
            if kind == "mma":
                self.fire_mma()
            elif kind == "load":
                self.fire_load()
            else:
                pending[r] = None
                try:
                    pending[r] = next(roles[r])
                except StopIteration:
                    alive.remove(r)
            if self.errors:
                return
        self.errors.append("no termination")


class Forward(Protocol):
    def __init__(self, rng, nt0, nt1, nq, S, p_rescale, slip=None):
        super().__init__(rng)
        self.nt = [nt0, nt1 if nq == 2 else 0]
        self.nq, self.S, self.p_rescale, self.slip = nq, S, p_rescale, slip
        self.nt_all = nt1 if nq == 2 else nt0
        self.q = Bar("q")
        self.kfull = [Bar(f"kfull{s}") for s in range(S)]
        self.vfull = [Bar(f"vfull{s}") for s in range(S)]
        self.kvempty = [Bar(f"kvempty{s}") for s in range(S)]
        self.s_ready = [Bar(f"s_ready{q}") for q in range(2)]
        self.p_ready = [Bar(f"p_ready{q}", 4) for q in range(2)]
        self.o_ready = [Bar(f"o_ready{q}") for q in range(2)]
        self.kst, self.vst, self.readers = [None] * S, [None] * S, [0] * S
        self.sbuf, self.sreading, self.pwritten = [None, None], [set(), set()], {}
        self.o_pv, self.pv_queued = [-1, -1], [0, 0]

    def producer(self):
        if self.nt_all == 0:
            return
        self.loads.append(("q", None))
        for t in range(self.nt_all):
            s = t % self.S
            # the slip: from the ring's third use of a stage on, refill without waiting for its release
            if t >= self.S and not (self.slip == "early_stage_reuse" and t >= 2 * self.S):
                yield ("wait", self.kvempty[s], t // self.S - 1)
            if self.readers[s]:
                self.errors.append(f"stage {s} refilled while read (tile {t})")
            self.loads.append(("k", (s, t)))
            self.loads.append(("v", (s, t)))
            yield None

    def mma(self):
        if self.nt_all == 0:
            return
        yield ("wait", self.q, 0)
        yield ("wait", self.kfull[0], 0)
        for q in range(self.nq):
            if self.nt[q]:
                self.issue_s(q, 0, 0)
        for t in range(self.nt_all):
            s, s1 = t % self.S, (t + 1) % self.S
            yield ("wait", self.vfull[s], t // self.S)
            next_k = False
            for q in range(self.nq):
                if t >= self.nt[q]:
                    continue
                yield ("wait", self.p_ready[q], t)
                self.readers[s] += 1
                self.pv_queued[q] += 1
                self.fifo.append(("pv", q, t, s))
                if t == self.nt[q] - 1:
                    self.fifo.append(("commit", self.o_ready[q]))
                else:
                    if not next_k:
                        yield ("wait", self.kfull[s1], (t + 1) // self.S)
                        next_k = True
                    self.issue_s(q, t + 1, s1)
            self.fifo.append(("commit", self.kvempty[s]))
            yield None

    def issue_s(self, q, t, s):
        self.readers[s] += 1
        self.fifo.append(("s", q, t, s))
        self.fifo.append(("commit", self.s_ready[q]))

    def softmax(self, q, w):
        for t in range(self.nt[q]):
            yield ("wait", self.s_ready[q], t)
            if self.sbuf[q] != ("S", t):
                self.errors.append(f"tile {q} warp {w} t {t}: buffer holds {self.sbuf[q]}")
            self.sreading[q].add(w)
            yield None
            if t > 0 and self.rng.random() < self.p_rescale:
                if self.o_pv[q] != t - 1 or self.pv_queued[q]:
                    self.errors.append(f"tile {q} t {t}: O rescaled at PV {self.o_pv[q]}, {self.pv_queued[q]} queued")
                yield None
            self.sreading[q].discard(w)
            self.pwritten.setdefault((q, t), set()).add(w)
            if len(self.pwritten[(q, t)]) == 4:
                self.sbuf[q] = ("P", t)
            self.p_ready[q].arrive()
            yield None
        if self.nt[q]:
            yield ("wait", self.o_ready[q], 0)
            if self.o_pv[q] != self.nt[q] - 1:
                self.errors.append(f"tile {q}: epilogue with O at PV {self.o_pv[q]}")

    def fire_load(self):
        kind, arg = self.loads.pop(self.rng.randrange(len(self.loads)))
        if kind == "q":
            self.q.arrive()
        elif kind == "k":
            self.kst[arg[0]] = arg[1]
            self.kfull[arg[0]].arrive()
        else:
            self.vst[arg[0]] = arg[1]
            self.vfull[arg[0]].arrive()

    def fire_mma(self):
        op = self.fifo.pop(0)
        if op[0] == "commit":
            op[1].arrive()
            return
        kind, q, t, s = op
        if kind == "s":
            if self.kst[s] != t:
                self.errors.append(f"S{q}({t}) read a K stage holding {self.kst[s]}")
            if self.sreading[q]:
                self.errors.append(f"S{q}({t}) overwrote S while it was read")
            if self.sbuf[q] is not None and self.sbuf[q][0] == "P" and self.sbuf[q][1] > self.o_pv[q]:
                self.errors.append(f"S{q}({t}) overwrote P before its PV")
            self.sbuf[q] = ("S", t)
        else:
            if self.vst[s] != t or len(self.pwritten.get((q, t), ())) != 4:
                self.errors.append(f"PV{q}({t}): V stage holds {self.vst[s]}, P incomplete")
            self.o_pv[q] = t
            self.pv_queued[q] -= 1
        self.readers[s] -= 1

    def check(self):
        self.run([self.producer(), self.mma()] + [self.softmax(q, w) for q in range(self.nq) for w in range(4)])
        return self.errors


class Backward(Protocol):
    def __init__(self, rng, nq, slip=None):
        super().__init__(rng)
        self.nq, self.slip = nq, slip
        self.kvfull = Bar("kvfull")
        self.qfull = [Bar(f"qfull{s}") for s in range(2)]
        self.dofull = [Bar(f"dofull{s}") for s in range(2)]
        self.empty = [Bar(f"empty{s}") for s in range(2)]
        self.dostage = [Bar(f"dostage{s}") for s in range(2)]
        self.sready, self.dpready = Bar("sready"), Bar("dpready")
        self.pready, self.dsready = Bar("pready", 8), Bar("dsready", 8)
        self.dsfree, self.dqready, self.dqfree = Bar("dsfree"), Bar("dqready"), Bar("dqfree", 4)
        self.dkdv = Bar("dkdvready")
        self.qst, self.dost = [None, None], [None, None]
        self.q_readers, self.do_readers = [0, 0], [0, 0]
        self.tm_s = self.tm_dp = self.ds_smem = None
        self.s_reading, self.dp_reading = set(), set()
        self.p_written, self.ds_written = {}, {}
        self.ds_readers, self.dq_reading, self.staging, self.dv_last = 0, False, None, -1
        # TMEM columns within the S^T block: warp w (group g = w // 4, lanes of
        # quadrant w % 4) reads S^T columns [64 g, 64 g + 64) and writes its
        # P^T over [64 g, 64 g + 32); the slip puts it at [32 g, 32 g + 32),
        # over the other group's unread S^T
        self.s_loaded = [-1] * 8

    def producer(self):
        self.loads.append(("kv", None))
        for it in range(self.nq):
            s = it & 1
            if it >= 2:
                yield ("wait", self.empty[s], (it >> 1) - 1)
            if self.q_readers[s]:
                self.errors.append(f"Q stage {s} refilled while read (tile {it})")
            self.loads.append(("q", (s, it)))
            yield None
            if it >= 2 and self.slip != "no_dostage_wait":
                yield ("wait", self.dostage[s], (it >> 1) - 1)
            if self.do_readers[s] or self.staging == it - 2:
                self.errors.append(f"dO stage {s} refilled while in use (tile {it})")
            self.loads.append(("do", (s, it)))
            yield None

    def mma(self):
        yield ("wait", self.kvfull, 0)
        yield ("wait", self.qfull[0], 0)
        self.op("S", 0, 0, self.sready)
        yield ("wait", self.dofull[0], 0)
        self.op("dP", 0, 0, self.dpready)
        for it in range(self.nq):
            s, s1, more = it & 1, (it + 1) & 1, it + 1 < self.nq
            yield ("wait", self.pready, it)
            self.op("dV", it, s)
            if more:
                yield ("wait", self.qfull[s1], (it + 1) >> 1)
                self.op("S", it + 1, s1, self.sready)
            yield ("wait", self.dsready, it)
            self.op("dQ", it, None, self.dqready)
            self.op("dK", it, s, self.empty[s])
            self.fifo.append(("commit", self.dsfree))
            if more:
                if self.slip != "no_dqfree_wait":
                    yield ("wait", self.dqfree, it)
                yield ("wait", self.dofull[s1], (it + 1) >> 1)
                self.op("dP", it + 1, s1, self.dpready)
            yield None
        self.fifo.append(("commit", self.dkdv))

    def op(self, kind, it, s, commit=None):
        if kind in ("S", "dK"):
            self.q_readers[s] += 1
        if kind in ("dV", "dP"):
            self.do_readers[s] += 1
        if kind in ("dQ", "dK"):
            self.ds_readers += 1
        self.fifo.append(("op", kind, it, s))
        if commit is not None:
            self.fifo.append(("commit", commit))

    def drain(self):
        for it in range(self.nq):
            s = it & 1
            yield ("wait", self.dqready, it)
            if self.tm_dp != ("dQ", it) or self.do_readers[s] or self.dost[s] != ("dO", it):
                self.errors.append(f"drain {it}: dQ cols {self.tm_dp}, dO stage {self.dost[s]}")
            self.dq_reading, self.staging = True, it
            self.dost[s] = ("staging", it)
            yield None
            self.dq_reading = False
            self.dqfree.arrive(4)  # all of dQ is out of TMEM
            yield None
            self.staging = None  # the reduce-adds have read the staging buffer
            self.dostage[s].arrive()
            yield None

    def elementwise(self, w):
        for it in range(self.nq):
            s = it & 1
            yield ("wait", self.qfull[s], it >> 1)
            yield ("wait", self.sready, it)
            if self.tm_s != ("S", it) or self.qst[s] != it:
                self.errors.append(f"warp {w} tile {it}: S cols {self.tm_s}, vectors of {self.qst[s]}")
            self.s_reading.add(w)
            self.s_loaded[w] = it
            yield None
            self.s_reading.discard(w)
            g, partner = w // 4, (w + 4) % 8
            p_cols = range(32 * g, 32 * g + 32) if self.slip == "shared_p_cols" else range(64 * g, 64 * g + 32)
            partner_cols = range(64 * (1 - g), 64 * (1 - g) + 64)
            if self.s_loaded[partner] < it and set(p_cols) & set(partner_cols):
                self.errors.append(f"warp {w} tile {it}: P^T written over S^T warp {partner} has not read")
            self.p_written.setdefault(it, set()).add(w)
            if len(self.p_written[it]) == 8:
                self.tm_s = ("P", it)
            self.pready.arrive()
            yield ("wait", self.dpready, it)
            if self.tm_dp != ("dP", it) or self.qst[s] != it:
                self.errors.append(f"warp {w} tile {it}: dP cols {self.tm_dp}, vectors of {self.qst[s]}")
            self.dp_reading.add(w)
            yield None
            self.dp_reading.discard(w)
            if it > 0:
                yield ("wait", self.dsfree, it - 1)
            if self.ds_readers:
                self.errors.append(f"warp {w} tile {it}: dS written while read")
            self.ds_written.setdefault(it, set()).add(w)
            if len(self.ds_written[it]) == 8:
                self.ds_smem = ("dS", it)
            self.dsready.arrive()
            yield None
        yield ("wait", self.dkdv, 0)

    def fire_load(self):
        kind, arg = self.loads.pop(self.rng.randrange(len(self.loads)))
        if kind == "kv":
            self.kvfull.arrive()
        elif kind == "q":
            self.qst[arg[0]] = arg[1]
            self.qfull[arg[0]].arrive()
        else:
            self.dost[arg[0]] = ("dO", arg[1])
            self.dofull[arg[0]].arrive()

    def fire_mma(self):
        e = self.fifo.pop(0)
        if e[0] == "commit":
            e[1].arrive()
            return
        _, kind, it, s = e
        if kind == "S":
            busy = self.tm_s is not None and self.tm_s[0] == "P" and self.dv_last < self.tm_s[1]
            if self.qst[s] != it or self.s_reading or busy:
                self.errors.append(f"S{it}: Q stage {self.qst[s]}, S/P cols {self.tm_s} in use")
            self.tm_s = ("S", it)
            self.q_readers[s] -= 1
        elif kind == "dP":
            if self.dost[s] != ("dO", it) or self.dp_reading or self.dq_reading:
                self.errors.append(f"dP{it}: dO stage {self.dost[s]}, dP/dQ cols {self.tm_dp} in use")
            self.tm_dp = ("dP", it)
            self.do_readers[s] -= 1
        elif kind == "dV":
            if self.tm_s != ("P", it) or self.dost[s] != ("dO", it):
                self.errors.append(f"dV{it}: S cols {self.tm_s}, dO stage {self.dost[s]}")
            self.dv_last = it
            self.do_readers[s] -= 1
        elif kind == "dQ":
            if self.ds_smem != ("dS", it) or self.dp_reading or self.dq_reading:
                self.errors.append(f"dQ{it}: dS {self.ds_smem}, dP cols in use")
            self.tm_dp = ("dQ", it)
            self.ds_readers -= 1
        else:  # dK
            if self.ds_smem != ("dS", it) or self.qst[s] != it:
                self.errors.append(f"dK{it}: dS {self.ds_smem}, Q stage {self.qst[s]}")
            self.ds_readers -= 1
            self.q_readers[s] -= 1

    def check(self):
        self.run([self.producer(), self.mma(), self.drain()] + [self.elementwise(w) for w in range(8)])
        return self.errors


class Decode(Protocol):
    """fa_decode.cu: one thread issues the page copies and both products; the
    four softmax warps move together (named barriers), so they are one role
    whose p_ready arrival counts four."""

    def __init__(self, rng, n, S, tail, p_rescale, slip=None):
        super().__init__(rng)
        self.n, self.S, self.tail, self.p_rescale, self.slip = n, S, tail, p_rescale, slip
        self.kfull = [Bar(f"kfull{s}") for s in range(S)]
        self.vfull = [Bar(f"vfull{s}") for s in range(S)]
        self.s_ready = [Bar(f"s_ready{b}") for b in range(2)]
        self.p_ready = [Bar(f"p_ready{b}", 4) for b in range(2)]
        self.pv_done = [Bar(f"pv_done{b}") for b in range(2)]
        self.kst, self.vst, self.readers = [None] * S, [None] * S, [0] * S
        self.sbuf, self.s_reading = [None, None], [False, False]
        self.pbuf, self.p_readers = [None, None], [0, 0]
        self.o_pv, self.pv_queued = -1, 0

    def load(self, it):
        st = it % self.S
        if self.readers[st]:
            self.errors.append(f"stage {st} refilled while read (tile {it})")
        self.loads.append(("k", (st, it)))
        self.loads.append(("v", (st, it)))

    def issue_s(self, it):
        st = it % self.S
        yield ("wait", self.kfull[st], it // self.S)
        self.readers[st] += 1
        self.fifo.append(("s", it, st))
        self.fifo.append(("commit", self.s_ready[it & 1]))

    def producer(self):
        n, S = self.n, self.S
        if n == 0:  # a split without tiles issues nothing
            return
        issued = 0
        while issued < min(S - 1, n):
            self.load(issued)
            issued += 1
        yield from self.issue_s(0)
        for it in range(n):
            # the freed stage is refilled before the wait for the next tile's K
            if issued < n:
                if it >= 1 and self.slip != "no_refill_wait":
                    yield ("wait", self.pv_done[(it - 1) & 1], (it - 1) >> 1)
                self.load(issued)
                issued += 1
            if it + 1 < n:
                yield from self.issue_s(it + 1)
            if self.slip == "single_p_ready":
                yield ("wait", self.p_ready[0], it)
            else:
                yield ("wait", self.p_ready[it & 1], it >> 1)
            yield ("wait", self.vfull[it % S], it // S)
            self.readers[it % S] += 1
            self.p_readers[it & 1] += 1
            self.pv_queued += 1
            self.fifo.append(("pv", it, it % S))
            self.fifo.append(("commit", self.pv_done[it & 1]))
            yield None

    def softmax(self):
        n, S = self.n, self.S
        for it in range(n):
            b = it & 1
            yield ("wait", self.s_ready[b], it >> 1)
            if self.sbuf[b] != ("S", it):
                self.errors.append(f"softmax {it}: S buffer {b} holds {self.sbuf[b]}")
            self.s_reading[b] = True
            yield None
            if self.tail and it == n - 1:
                # zero the V rows past the sequence once the tile's V has landed
                yield ("wait", self.vfull[it % S], it // S)
                if self.vst[it % S] != it or self.readers[it % S]:
                    self.errors.append(f"softmax {it}: V stage holds {self.vst[it % S]} while zeroed")
            if it >= 2:
                yield ("wait", self.pv_done[b], (it - 2) >> 1)
            if self.p_readers[b]:
                self.errors.append(f"softmax {it}: P buffer {b} written while a product reads it")
            self.pbuf[b] = it
            rescale = it > 0 and self.rng.random() < self.p_rescale
            if rescale:
                yield ("wait", self.pv_done[(it - 1) & 1], (it - 1) >> 1)
                if self.o_pv != it - 1 or self.pv_queued:
                    self.errors.append(f"softmax {it}: O rescaled at PV {self.o_pv}, {self.pv_queued} queued")
            self.s_reading[b] = False
            self.p_ready[0 if self.slip == "single_p_ready" else b].arrive(4)
            yield None
        if n:
            yield ("wait", self.pv_done[(n - 1) & 1], (n - 1) >> 1)
            if self.o_pv != n - 1:
                self.errors.append(f"epilogue with O at PV {self.o_pv}")

    def fire_load(self):
        kind, (st, it) = self.loads.pop(self.rng.randrange(len(self.loads)))
        if kind == "k":
            self.kst[st] = it
            self.kfull[st].arrive()
        else:
            self.vst[st] = it
            self.vfull[st].arrive()

    def fire_mma(self):
        e = self.fifo.pop(0)
        if e[0] == "commit":
            e[1].arrive()
            return
        kind, it, st = e
        b = it & 1
        if kind == "s":
            if self.kst[st] != it or self.s_reading[b]:
                self.errors.append(f"S{it}: K stage holds {self.kst[st]}, buffer {b} in use")
            self.sbuf[b] = ("S", it)
        else:
            if self.vst[st] != it or self.pbuf[b] != it:
                self.errors.append(f"PV{it}: V stage holds {self.vst[st]}, P buffer holds {self.pbuf[b]}")
            self.o_pv = it
            self.pv_queued -= 1
            self.p_readers[b] -= 1
        self.readers[st] -= 1

    def check(self):
        self.run([self.producer(), self.softmax()])
        return self.errors


def _forward_cases():
    for S in (2, 4):
        for nq in (1, 2):
            for nt0 in range(0, 6):
                for nt1 in range(max(nt0, 1), 7):
                    if nq == 1 and nt1 != nt0:
                        continue
                    yield S, nq, nt0, nt1


def test_forward_protocol():
    rng = random.Random(1)
    for S, nq, nt0, nt1 in _forward_cases():
        for _ in range(12):
            errors = Forward(rng, nt0, nt1, nq, S, rng.choice([0.0, 0.5, 1.0])).check()
            assert not errors, (S, nq, nt0, nt1, errors[:2])


def test_backward_protocol():
    rng = random.Random(2)
    for nq in list(range(1, 8)) + [11]:
        for _ in range(80):
            errors = Backward(rng, nq).check()
            assert not errors, (nq, errors[:2])


def test_forward_slip_is_caught():
    rng = random.Random(3)
    assert any(Forward(rng, 6, 6, 1, 2, 0.0, slip="early_stage_reuse").check() for _ in range(40))


@pytest.mark.parametrize("slip", ["no_dqfree_wait", "no_dostage_wait", "shared_p_cols"])
def test_backward_slips_are_caught(slip):
    rng = random.Random(4)
    assert any(Backward(rng, 4, slip=slip).check() for _ in range(40))


def test_decode_protocol():
    rng = random.Random(5)
    for S in (3, 4):
        for n in list(range(0, 9)) + [13]:
            for _ in range(40):
                errors = Decode(rng, n, S, rng.random() < 0.5, rng.choice([0.0, 0.5, 1.0])).check()
                assert not errors, (S, n, errors[:2])


class KeepRing(Protocol):
    """The keep-word ring of fa_fwd_wide.cu (dropout): four keep-word warps
    each write their 32 rows' words of tile t into buffer t & 1 once the four
    softmax warps have released the buffer's tile t - 2 (keep_empty, four
    arrivals), then arrive on keep_full (four arrivals); softmax warp c waits
    for keep_full of tile t, reads its rows (written by keep-word warp c) and
    arrives on keep_empty."""

    def __init__(self, rng, nt, slip=None):
        super().__init__(rng)
        self.nt, self.slip = nt, slip
        self.full = [Bar(f"keep_full{b}", 4) for b in range(2)]
        self.empty = [Bar(f"keep_empty{b}", 4) for b in range(2)]
        self.rows = [[None] * 4 for _ in range(2)]      # tile held by each warp's rows of a buffer
        self.unread = [set(), set()]                     # softmax warps that have not read the buffer's tile

    def producer(self, w):
        for t in range(self.nt):
            b = t & 1
            if t >= 2 and self.slip != "no_empty_wait":
                yield ("wait", self.empty[b], (t - 2) >> 1)
            yield None  # the Philox draw
            if self.rows[b][w] is not None and self.unread[b]:
                self.errors.append(f"keep warp {w} wrote tile {t} over tile {self.rows[b][w]} "
                                   f"not yet read by {sorted(self.unread[b])}")
            self.rows[b][w] = t
            if all(x == t for x in self.rows[b]):
                self.unread[b] = {0, 1, 2, 3}
            self.full[b].arrive()

    def softmax(self, c):
        for t in range(self.nt):
            b = t & 1
            yield ("wait", self.full[b], t >> 1)
            if self.rows[b][c] != t:
                self.errors.append(f"softmax warp {c} read tile {self.rows[b][c]} for tile {t}")
            self.unread[b].discard(c)
            yield None
            self.empty[b].arrive()

    def check(self):
        self.run([self.producer(w) for w in range(4)] + [self.softmax(c) for c in range(4)])
        return self.errors


@pytest.mark.parametrize("nt", [1, 2, 3, 9])
def test_wide_forward_keep_ring(nt):
    rng = random.Random(nt)
    for _ in range(200):
        assert KeepRing(rng, nt).check() == []


def test_wide_forward_keep_ring_slip_is_caught():
    rng = random.Random(7)
    assert any(KeepRing(rng, 6, slip="no_empty_wait").check() for _ in range(100))


@pytest.mark.parametrize("slip", ["no_refill_wait", "single_p_ready"])
def test_decode_slips_are_caught(slip):
    rng = random.Random(6)
    assert any(Decode(rng, 8, 3, False, 0.0, slip=slip).check() for _ in range(60))
