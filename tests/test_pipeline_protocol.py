"""Model check of the forward kernel's mbarrier protocol (CPU, no GPU).

Every role of the kernel (K producer, V producer, score / P.V issuers, softmax
warpgroups) is modelled as a generator that waits for barrier phases and
arrives on barriers in the same order as the CUDA code; copies and tensor-core
work complete asynchronously, in random order for copies and in issue order
for the tensor pipe.  Random interleavings are explored for random item sizes
(including one-chunk items), ring depths and both warp layouts (two issuing
threads, or one issuing the scores two chunks ahead of P.V).

A parity wait is sound only if, whenever the waiter polls, the barrier has
completed exactly the phase before the awaited one or the awaited one itself:
two phases late, the parity matches again and the waiter blocks on a phase
that may never come; a phase early, the parity matches the previous phase and
the wait passes at once.  The model flags both, and deadlock.
"""
from __future__ import annotations

import random

import pytest


class Bug(Exception):
    pass


class Bar:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.ph = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending > self.count:
            raise Bug(f"{self.name}: more arrivals than the count")
        if self.pending == self.count:
            self.pending = 0
            self.ph += 1


def wait(bar, k):
    """Wait for phase k of bar (generator); check parity soundness at every poll."""
    while True:
        if bar.ph < k:
            raise Bug(f"early wait on {bar.name}: phase {k} awaited, {bar.ph} completed")
        if bar.ph >= k + 2:
            raise Bug(f"late wait on {bar.name}: phase {k} awaited, {bar.ph} completed")
        if bar.ph == k + 1:
            return
        yield ("wait", bar.name, k)


def simulate(nchs, NK, NP, NSW, two_issuers, rng, need_p=0.3, mutant=None):
    KF = [Bar(f"k_full{i}") for i in range(NK)]
    KE = [Bar(f"k_empty{i}") for i in range(NK)]
    VF = [Bar(f"v_full{i}") for i in range(2)]
    QF, QE = Bar("q_full"), Bar("q_empty")
    SF = [Bar(f"s_full{i}") for i in range(2)]
    SR = [Bar(f"s_free{i}", NSW) for i in range(2)]
    PF = [Bar(f"p_full{i}", NSW) for i in range(NP)]
    OD = [Bar(f"o_done{i}") for i in range(2)]
    copies, pipe = [], []  # in-flight copies (complete in any order); tensor pipe (in order)
    stream = [(it, c, n) for it, n in enumerate(nchs) for c in range(n)]
    G = len(stream)

    def k_producer():
        g = 0
        for it, n in enumerate(nchs):
            if it > 0:
                yield from wait(QE, it - 1)
            copies.append(QF)
            for c in range(n):
                gc = g + c
                if gc >= NK:
                    yield from wait(KE[gc % NK], gc // NK - 1)
                copies.append(KF[gc % NK])
                yield ("step",)
            g += n

    def v_producer():
        for gc in range(G):
            if gc >= 2:
                k = (gc - 2) >> 1
                if mutant == "v_early":
                    k += 1
                yield from wait(OD[gc & 1], k)
            copies.append(VF[gc % 2])
            yield ("step",)

    def issue_s(gc):
        it, c, n = stream[gc]
        if c == 0:
            yield from wait(QF, it)
        yield from wait(KF[gc % NK], gc // NK)
        if gc >= 2 and mutant != "no_sfree":
            yield from wait(SR[gc & 1], (gc >> 1) - 1)
        pipe.append(("mma", f"S{gc}"))
        pipe.append(("commit", SF[gc & 1]))

    def issue_pv(g):
        yield from wait(VF[g % 2], g // 2)
        yield from wait(PF[g % NP], g // NP)
        pipe.append(("mma", f"PV{g}"))
        pipe.append(("commit", OD[g & 1]))

    def score_issuer():
        for gc in range(G):
            yield from issue_s(gc)

    def pv_issuer():
        for g in range(G):
            yield from issue_pv(g)

    def single_issuer():
        g = 0
        for it, n in enumerate(nchs):
            for c in range(min(n, 2)):
                yield from issue_s(g + c)
            for c in range(n):
                if c + 2 < n:
                    yield from issue_s(g + c + 2)
                yield from issue_pv(g + c)
            g += n

    def softmax(wg):
        g = 0
        for it, n in enumerate(nchs):
            for c in range(n):
                gc = g + c
                yield from wait(SF[gc & 1], gc >> 1)
                if wg == 0:
                    KE[gc % NK].arrive()
                    if c == n - 1:
                        QE.arrive()
                yield ("step",)
                SR[gc & 1].arrive()
                if rng.random() < need_p and c > 0:  # rescale: O must hold chunk gc-1
                    yield from wait(OD[(gc - 1) & 1], (gc - 1) >> 1)
                if gc >= NP and mutant != "no_pbuf":
                    yield from wait(OD[(gc - NP) & 1], (gc - NP) >> 1)
                yield ("step",)
                PF[gc % NP].arrive()
            e = g + n - 1
            yield from wait(OD[e & 1], e >> 1)
            g += n

    roles = {"K": k_producer(), "V": v_producer()}
    if two_issuers:
        roles["S"], roles["PV"] = score_issuer(), pv_issuer()
    else:
        roles["I"] = single_issuer()
    for wg in range(NSW):
        roles[f"W{wg}"] = softmax(wg)
    state = {r: None for r in roles}
    done = set()
    idle_rounds = 0
    for _ in range(500000):
        if len(done) == len(roles):
            return
        progressed = False
        if copies and rng.random() < 0.5:
            copies.pop(rng.randrange(len(copies))).arrive()
            progressed = True
        if pipe and rng.random() < 0.5:
            op = pipe.pop(0)
            if op[0] == "commit":
                op[1].arrive()
            progressed = True
        order = [r for r in roles if r not in done]
        rng.shuffle(order)
        for r in order:
            try:
                y = next(roles[r])
            except StopIteration:
                done.add(r)
                progressed = True
                continue
            if y != state[r] or y[0] != "wait":
                progressed = True
            state[r] = y
        idle_rounds = 0 if (progressed or copies or pipe) else idle_rounds + 1
        if idle_rounds > 3:
            raise Bug(f"deadlock: {dict((r, state[r]) for r in roles if r not in done)}")
    raise Bug("no termination")


CASES = [[1], [2], [3], [1, 1], [1, 1, 1, 1], [5, 1, 5], [2, 1, 1, 3], [8, 8], [1, 2, 1, 2, 1]]


def _random_cases(n, seed):
    rng = random.Random(seed)
    return [[rng.randint(1, 6) for _ in range(rng.randint(1, 5))] for _ in range(n)]


@pytest.mark.parametrize("two_issuers,NSW", [(True, 4), (True, 2), (False, 2)])
@pytest.mark.parametrize("NK,NP", [(3, 2), (4, 2), (3, 1), (2, 1)])
def test_protocol_is_deadlock_free_and_parity_sound(two_issuers, NSW, NK, NP):
    for i, nchs in enumerate(CASES + _random_cases(12, NK * 10 + NP)):
        for trial in range(6):
            simulate(nchs, NK, NP, NSW, two_issuers, random.Random(trial * 7919 + i))


@pytest.mark.parametrize("mutant", ["v_early", "no_pbuf", "no_sfree"])
def test_model_catches_planted_protocol_errors(mutant):
    """The checker itself is pinned: each planted protocol error is found."""
    caught = False
    for i, nchs in enumerate(CASES + _random_cases(20, 3)):
        for trial in range(10):
            try:
                simulate(nchs, 3, 2, 2, True, random.Random(trial * 31 + i), mutant=mutant)
            except Bug:
                caught = True
                break
        if caught:
            break
    assert caught, f"planted error {mutant} not detected"


# ---------------------------------------------------------------------------
# Query-major kernel (128-row query blocks): one softmax warpgroup, P in two
# TMEM buffers, O reused across items behind an "O read" barrier.  Besides
# deadlock and parity soundness, the model checks the three data hazards the
# barriers exist for: S(g) overwriting a slot the softmax still reads, P.V(g)
# reading a P buffer that the softmax has not finished writing or that a later
# chunk has overwritten, the first P.V of an item overwriting O before the
# previous item's epilogue has read it, and the epilogue reading O before the
# item's last P.V has executed.  (The "O read" barrier turns out to be implied
# by the softmax's own order -- the next item's first P.V needs that item's
# first P, written after the epilogue -- and is kept as a guard.)
# ---------------------------------------------------------------------------
class Rendezvous:
    """A named barrier among `n` roles: each instance (key) completes when all arrived."""

    def __init__(self, n):
        self.n, self.count = n, {}


def rendezvous(rv, key):
    rv.count[key] = rv.count.get(key, 0) + 1
    while rv.count[key] < rv.n:
        yield ("barrier", key)


def simulate_qm(nchs, NK, rng, need_p=0.3, mutant=None, halves=1):
    """halves = 2: two softmax warpgroups, each taking half of every chunk's keys
    (counts of two on the softmax barriers, a rendezvous per chunk to combine the
    row maxima and one per item before the epilogue)."""
    KF = [Bar(f"k_full{i}") for i in range(NK)]
    KE = [Bar(f"k_empty{i}") for i in range(NK)]
    VF = [Bar(f"v_full{i}") for i in range(2)]
    QF, QE = Bar("q_full"), Bar("q_empty")
    SF = [Bar(f"s_full{i}") for i in range(2)]
    SR = [Bar(f"s_free{i}", halves) for i in range(2)]
    single_p = mutant == "single_pfull"
    pcount = 1 if mutant == "pfull_count1" else halves
    PF = [Bar("p_full0", pcount)] * 2 if single_p else [Bar(f"p_full{i}", pcount) for i in range(2)]
    OD = [Bar(f"o_done{i}") for i in range(2)]
    OE = Bar("o_empty", halves)
    RV = Rendezvous(halves)
    copies, pipe = [], []
    stream = [(it, c, n) for it, n in enumerate(nchs) for c in range(n)]
    G = len(stream)
    need = [rng.random() < need_p for _ in range(G)]  # reference raised (the same in both halves)
    s_reading = [set(), set()]  # halves still reading the scores of slot i
    p_written = [{}, {}]        # P buffer i: half -> chunk whose probabilities it holds (complete)
    o_reading = set()           # (item, half) of epilogues reading O
    pv_done = [0] * len(nchs)   # P.V products executed per item

    def execute(op):
        kind, g = op
        it, c, n = stream[g]
        if kind == "S":
            if s_reading[g & 1]:
                raise Bug(f"S{g} overwrites slot {g & 1} while halves {s_reading[g & 1]} read it")
        else:  # P.V
            if any(p_written[g & 1].get(h) != g for h in range(halves)):
                raise Bug(f"PV{g} reads P buffer {g & 1} holding {p_written[g & 1]}")
            if c == 0 and o_reading:
                raise Bug(f"PV{g} (first of item {it}) overwrites O while {o_reading} read it")
            pv_done[it] += 1

    def k_producer():
        g = 0
        for it, n in enumerate(nchs):
            if it > 0:
                yield from wait(QE, it - 1)
            copies.append(QF)
            for c in range(n):
                gc = g + c
                if gc >= NK:
                    yield from wait(KE[gc % NK], gc // NK - 1)
                copies.append(KF[gc % NK])
                yield ("step",)
            g += n

    def v_producer():
        for gc in range(G):
            if gc >= 2:
                yield from wait(OD[gc & 1], (gc - 2) >> 1)
            copies.append(VF[gc % 2])
            yield ("step",)

    def issue_s(gc):
        it, c, n = stream[gc]
        if c == 0:
            yield from wait(QF, it)
        yield from wait(KF[gc % NK], gc // NK)
        if gc >= 2:
            yield from wait(SR[gc & 1], (gc >> 1) - 1)
        pipe.append(("mma", ("S", gc)))
        pipe.append(("commit", SF[gc & 1]))

    def issue_pv(gc):
        it, c, n = stream[gc]
        if c == 0 and it > 0 and mutant != "no_oempty":
            yield from wait(OE, it - 1)
        yield from wait(VF[gc % 2], gc // 2)
        yield from wait(PF[gc & 1], gc if single_p else gc >> 1)
        pipe.append(("mma", ("PV", gc)))
        pipe.append(("commit", OD[gc & 1]))

    def issuer():
        g = 0
        for it, n in enumerate(nchs):
            for c in range(min(n, 2)):
                yield from issue_s(g + c)
            for c in range(n):
                if c + 2 < n:
                    yield from issue_s(g + c + 2)
                yield from issue_pv(g + c)
            g += n

    def softmax(h):
        g = 0
        for it, n in enumerate(nchs):
            for c in range(n):
                gc = g + c
                yield from wait(SF[gc & 1], gc >> 1)
                s_reading[gc & 1].add(h)
                if h == 0:
                    KE[gc % NK].arrive()
                    if c == n - 1:
                        QE.arrive()
                yield ("step",)
                if halves > 1:
                    yield from rendezvous(RV, ("max", gc))
                if need[gc] and c > 0:  # rescale: O must hold chunk gc-1
                    yield from wait(OD[(gc - 1) & 1], (gc - 1) >> 1)
                if gc >= 2 and mutant != "no_pbuf":
                    yield from wait(OD[(gc - 2) & 1], (gc - 2) >> 1)
                p_written[gc & 1].pop(h, None)  # being overwritten
                yield ("step",)
                p_written[gc & 1][h] = gc
                s_reading[gc & 1].discard(h)
                SR[gc & 1].arrive()
                PF[gc & 1].arrive()
            e = g + n - 1
            if mutant != "no_epilogue_wait":
                yield from wait(OD[e & 1], e >> 1)
            if pv_done[it] != n:
                raise Bug(f"epilogue of item {it} reads O after {pv_done[it]} of {n} P.V products")
            if halves > 1:
                yield from rendezvous(RV, ("epilogue", it))
            o_reading.add((it, h))
            yield ("step",)
            o_reading.discard((it, h))
            OE.arrive()
            g += n

    roles = {"K": k_producer(), "V": v_producer(), "I": issuer()}
    for h in range(halves):
        roles[f"W{h}"] = softmax(h)
    state = {r: None for r in roles}
    done = set()
    idle_rounds = 0
    for _ in range(500000):
        if len(done) == len(roles):
            return
        progressed = False
        if copies and rng.random() < 0.5:
            copies.pop(rng.randrange(len(copies))).arrive()
            progressed = True
        if pipe and rng.random() < 0.5:
            op = pipe.pop(0)
            if op[0] == "commit":
                op[1].arrive()
            else:
                execute(op[1])
            progressed = True
        order = [r for r in roles if r not in done]
        rng.shuffle(order)
        for r in order:
            try:
                y = next(roles[r])
            except StopIteration:
                done.add(r)
                progressed = True
                continue
            if y != state[r] or y[0] not in ("wait", "barrier"):
                progressed = True
            state[r] = y
        idle_rounds = 0 if (progressed or copies or pipe) else idle_rounds + 1
        if idle_rounds > 3:
            raise Bug(f"deadlock: {dict((r, state[r]) for r in roles if r not in done)}")
    raise Bug("no termination")


@pytest.mark.parametrize("halves", [1, 2])
@pytest.mark.parametrize("NK", [2, 3, 4])
def test_query_major_protocol_is_sound(NK, halves):
    for i, nchs in enumerate(CASES + _random_cases(12, NK * 17)):
        for trial in range(6):
            simulate_qm(nchs, NK, random.Random(trial * 7919 + i), halves=halves)


@pytest.mark.parametrize("halves", [1, 2])
def test_query_major_o_read_barrier_is_implied(halves):
    for i, nchs in enumerate(CASES + _random_cases(12, 99)):
        for trial in range(6):
            simulate_qm(nchs, 3, random.Random(trial * 13 + i), mutant="no_oempty", halves=halves)


@pytest.mark.parametrize("mutant,halves", [("no_pbuf", 1), ("no_epilogue_wait", 1), ("single_pfull", 1),
                                           ("no_pbuf", 2), ("pfull_count1", 2)])
def test_query_major_model_catches_planted_errors(mutant, halves):
    caught = False
    for i, nchs in enumerate(CASES + _random_cases(20, 5)):
        for trial in range(10):
            try:
                simulate_qm(nchs, 4, random.Random(trial * 31 + i), mutant=mutant, halves=halves)
            except Bug:
                caught = True
                break
        if caught:
            break
    assert caught, f"planted error {mutant} not detected"
